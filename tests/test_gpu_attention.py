"""GPU parity of the single attention layer (nc_attention: RoPE + QK-norm,
then causal sliding-window attention) against the oracle.

Small shapes are compared element by element; the sweep shapes (B = 8,
H = 12, D = 128, T in {2048, 8192}, window in {1024, full}) are compared on
sampled (batch, position) outputs that the oracle evaluates one query at a
time.  Tolerance: 2e-2 absolute in bf16 (inputs and outputs are bf16, so the
output rounding alone is up to 2^-9 |o|), 1e-4 in fp32."""
import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc, synth
from oracle import nanochat_fwd as O

pytestmark = pytest.mark.gpu

ALPHA, BASE, EPS = 1.15, 100000.0, 1e-6


def _run(q, k, v, window, dtype):
    import torch
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    B, T, H, D = q.shape
    dq, dk, dv = (torch.from_numpy(a).cuda().to(tdt) for a in (q, k, v))
    out = torch.empty_like(dq)
    ws = torch.empty(nc.nc_attention_workspace_bytes(B, T, H, k.shape[2], D, dtype, 1),
                     dtype=torch.uint8, device="cuda")
    nc.nc_attention(dq, dk, dv, out, window, 1, ALPHA, D ** -0.5, BASE, EPS, ws)
    torch.cuda.synchronize()
    rc, _ = nc.nc_get_status()
    assert rc == 0
    return out.float().cpu().numpy()


def _ref(q, k, v, window, positions=None):
    T = q.shape[0]
    w = T if window <= 0 or window >= T else window
    return O.attention_layer(q, k, v, w, alpha=ALPHA, scale=q.shape[-1] ** -0.5, rope_base=BASE,
                             eps=EPS, positions=positions)


@pytest.mark.parametrize("B,T,H,window,dtype", [
    (1, 1, 1, 0, "bf16"), (2, 77, 2, 0, "bf16"), (1, 300, 3, 64, "bf16"), (2, 257, 1, 1, "bf16"),
    (1, 130, 2, 129, "fp32"), (2, 64, 1, 5, "fp32")])
def test_attention_small(B, T, H, window, dtype):
    q, k, v = synth.attention_inputs(500 + T, B, T, H, 128, bf16=(dtype == "bf16"))
    out = _run(q, k, v, window, dtype)
    tol = 2e-2 if dtype == "bf16" else 1e-4
    for b in range(B):
        ref = _ref(q[b], k[b], v[b], window)
        err = np.max(np.abs(out[b] - ref))
        assert err <= tol, (b, err)


@pytest.mark.parametrize("B,T,H,Hkv,window,dtype", [
    (2, 300, 4, 2, 96, "bf16"), (1, 200, 6, 3, 0, "bf16"), (2, 257, 4, 1, 1, "bf16"), (2, 130, 4, 2, 129, "fp32")])
def test_attention_grouped_query(B, T, H, Hkv, window, dtype):
    """H_kv < H: query head h attends with k/v head h / (H / H_kv)."""
    q, k, v = synth.attention_inputs(700 + T, B, T, H, 128, Hkv=Hkv, bf16=(dtype == "bf16"))
    out = _run(q, k, v, window, dtype)
    tol = 2e-2 if dtype == "bf16" else 1e-4
    for b in range(B):
        ref = _ref(q[b], k[b], v[b], window)
        err = np.max(np.abs(out[b] - ref))
        assert err <= tol, (b, err)


@pytest.mark.parametrize("T,window", synth.ATTN_SWEEP["cases"])
def test_attention_sweep_sampled(T, window):
    s = synth.ATTN_SWEEP
    B, H, D = s["B"], s["H"], s["D"]
    q, k, v = synth.attention_inputs(synth.SEED_BASE + s["index"], B, T, H, D)
    out = _run(q, k, v, window, "bf16")
    rng = np.random.default_rng(T + window)
    for b in (0, B - 1):
        pos = sorted(set([0, 1, 127, 128, T - 1] + list(rng.integers(0, T, 6))))
        ref = _ref(q[b], k[b], v[b], window, positions=pos)
        err = np.max(np.abs(out[b, pos] - ref))
        assert err <= 2e-2, (b, err)


@pytest.mark.parametrize("T,window", [(256, 0), (1000, 300), (129, 1), (2048, 1024)])
def test_tc_attention_matches_fp32_attention(T, window):
    """bf16 tensor-core attention vs the fp32 CUDA-core kernel on the same
    (bf16-valued) inputs: the only differences are bf16 P and output."""
    import torch
    B, H, D = 2, 2, 128
    q, k, v = synth.attention_inputs(900 + T, B, T, H, D)
    out_tc = _run(q, k, v, window, "bf16")
    out_32 = _run(q, k, v, window, "fp32")
    assert np.max(np.abs(out_tc - out_32)) <= 2e-2
    assert np.sqrt(np.mean((out_tc - out_32) ** 2)) <= 3e-3
