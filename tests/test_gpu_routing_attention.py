"""GPU parity of the pass-2 routing attention (nc_routing_attention) against
the oracle's routing_attention ("looped-nanochat-d24" card, routing loop):
logits (q2 . k2 + softplus(gate) q1 . k1) / sqrt(D) on the base model's
visibility rule.  Same shapes and tolerance as the base attention layer
(test_gpu_attention.py): bf16 inputs and output, 2e-2 absolute, since the
output is rounded to bf16 (up to 2^-9 |o|) and g q1 enters the tensor cores in
bf16.  Query and key features are the ones entering the attention (already
RoPE-applied and normalised in their pass), drawn N(0, 1)."""
import math

import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc, synth
from oracle import nanochat_fwd as O
from oracle import routing_attention as R

pytestmark = pytest.mark.gpu


def _inputs(seed, B, T, H, Hkv):
    q2, k2, v2 = synth.attention_inputs(seed, B, T, H, 128, Hkv=Hkv)
    q1, k1, _ = synth.attention_inputs(seed + 1, B, T, H, 128, Hkv=Hkv)
    return q2, k2, v2, q1, k1


def _run(q2, k2, v2, q1, k1, window, gate):
    import torch
    t = [torch.from_numpy(a).cuda().to(torch.bfloat16) for a in (q2, k2, v2, q1, k1)]
    out = torch.full_like(t[0], float("nan"))
    nc.nc_routing_attention(*t, out, window, gate)
    torch.cuda.synchronize()
    rc, _ = nc.nc_get_status()
    assert rc == 0
    assert nc.nc_last_launch_count() == 2  # g q1, then the attention kernel
    return out.float().cpu().numpy()


def _check(B, T, H, Hkv, window, gate, seed, positions=None):
    q2, k2, v2, q1, k1 = _inputs(seed, B, T, H, Hkv)
    out = _run(q2, k2, v2, q1, k1, window, gate)
    w = T if window <= 0 or window >= T else window
    for b in range(B):
        ref = R.routing_attention(q2[b], k2[b], v2[b], q1[b], k1[b], gate, w)
        got = out[b] if positions is None else out[b, positions]
        if positions is not None:
            ref = ref[positions]
        err = float(np.max(np.abs(got - ref)))
        assert err <= 2e-2, (b, err)


@pytest.mark.parametrize("B,T,H,window,gate", [
    (1, 1, 1, 0, 0.3), (2, 77, 2, 0, 1.5), (1, 300, 3, 64, -2.0), (2, 257, 1, 1, 0.0)])
def test_routing_attention_small(B, T, H, window, gate):
    _check(B, T, H, H, window, gate, 1500 + T)


@pytest.mark.parametrize("B,T,H,Hkv,window", [(2, 300, 4, 2, 96), (1, 200, 6, 3, 0), (2, 257, 4, 1, 1)])
def test_routing_attention_grouped_query(B, T, H, Hkv, window):
    _check(B, T, H, Hkv, window, 0.7, 1700 + T)


def test_routing_attention_prior_matters():
    """The prior changes the output (a closed gate gives the base attention)."""
    B, T, H = 1, 200, 2
    q2, k2, v2, q1, k1 = _inputs(1900, B, T, H, H)
    open_ = _run(q2, k2, v2, q1, k1, 0, 2.0)
    closed = _run(q2, k2, v2, q1, k1, 0, -80.0)      # softplus(-80) ~ 1.8e-35
    base = O.attention(q2[0], k2[0], v2[0], T, 128 ** -0.5)
    assert np.max(np.abs(closed[0] - base)) <= 2e-2
    assert np.max(np.abs(open_[0] - base)) > 0.1


@pytest.mark.parametrize("T,window", [(2048, 1024), (2048, 0)])
def test_routing_attention_sweep_sampled(T, window):
    s = synth.ATTN_SWEEP
    rng = np.random.default_rng(T + window)
    pos = sorted(set([0, 1, 127, 128, T - 1] + list(rng.integers(0, T, 6))))
    # R.routing_attention evaluates every query; restrict it to 2 heads of 2 rows
    B, H = 2, 2
    q2, k2, v2, q1, k1 = _inputs(synth.SEED_BASE + s["index"] + 10, B, T, H, H)
    out = _run(q2, k2, v2, q1, k1, window, 0.5)
    w = T if window <= 0 else window
    for b in range(B):
        ref = R.routing_attention(q2[b], k2[b], v2[b], q1[b], k1[b], 0.5, w)
        assert float(np.max(np.abs(out[b, pos] - ref[pos]))) <= 2e-2
        assert math.isfinite(float(np.abs(out[b]).max()))
