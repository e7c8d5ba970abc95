"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances.  fp32 mode: per-token loss and softcapped logits within 1e-4.
bf16 mode (bf16 GEMM operands, fp32 accumulation): per-token loss and
softcapped logits with rms error <= 6e-3 (over 256 or more values), per-token
loss max error <= 3e-2, logit max error <= 5e-2, mean-loss error <= 1e-3.  The per-token loss error is the error of the
target logit (the log-sum-exp term averages over 32768 logits), and the bf16
rounding of the GEMM operands alone puts it at rms ~4e-3 for these
random-init weights (test_bf16_rounding_budget.py reproduces this with an
emulation that rounds exactly where the kernels do), so a 1e-2 bound on the
maximum over thousands of tokens would fail for any bf16 implementation.
The logit errors have the same origin and size (rms ~4e-3); over one row's
33.5M logits the emulation's maximum is already 2.7e-2, so the stated 3e-2
is the edge of the bf16 noise rather than a bound on it.

Small cases are compared element by element; the d12 / d24
workloads run at full size on the GPU and are compared on whole sampled rows
(rows are independent sequences, so a row of the oracle is exact for that
row of the batch)."""
import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc, synth
from nc_cases import make_case, run_gpu
from oracle import nanochat_fwd as O

pytestmark = pytest.mark.gpu

TOL = {"bf16": dict(loss_rms=6e-3, loss_max=3e-2, mean=1e-3, logits=5e-2, logits_rms=6e-3),
       "fp32": dict(loss_rms=1e-4, loss_max=1e-4, mean=1e-4, logits=1e-4, logits_rms=1e-4)}


def _compare(gpu_loss, ref_loss, gpu_logits=None, ref_logits=None, dtype="bf16"):
    t = TOL[dtype]
    assert np.all(np.isfinite(gpu_loss))
    d = np.abs(gpu_loss - ref_loss)
    rms, mx = float(np.sqrt(np.mean(d ** 2))), float(d.max())
    assert mx <= t["loss_max"], f"loss max abs err {mx:.3e} > {t['loss_max']}"
    if d.size >= 256 or dtype == "fp32":
        assert rms <= t["loss_rms"], f"loss rms err {rms:.3e} > {t['loss_rms']}"
        assert abs(float(np.mean(gpu_loss)) - float(np.mean(ref_loss))) <= t["mean"]
    tz = t["logits"]
    if gpu_logits is not None:
        dz = np.abs(gpu_logits - ref_logits)
        zerr = float(dz.max())
        assert zerr <= tz, f"logit max abs err {zerr:.3e} > {tz}"
        zrms = float(np.sqrt(np.mean(dz.astype(np.float64) ** 2)))
        assert zrms <= t["logits_rms"], f"logit rms err {zrms:.3e} > {t['logits_rms']}"
        assert np.all(np.abs(gpu_logits) <= 15.0)


def test_d1_fp32_full():
    w = synth.WORKLOADS["d1"]
    seed = synth.SEED_BASE + w["index"]
    cfg, ocfg, p, tok, tgt = make_case(w["depth"], w["B"], w["T"], w["short"], w["dtype"], seed)
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, want_logits=True)
    _compare(loss, ref_loss, logits, ref_logits, "fp32")


@pytest.mark.parametrize("gemm_impl,attn_impl,gemm_pair", [(0, 0, 1), (0, 0, 0), (1, 1, 0)])
def test_d4_bf16_full(gemm_impl, attn_impl, gemm_pair):
    """gemm_pair selects the CTA-pair (cta_group::2) or the single-CTA tcgen05 GEMM."""
    w = synth.WORKLOADS["d4"]
    seed = synth.SEED_BASE + w["index"]
    cfg, ocfg, p, tok, tgt = make_case(w["depth"], w["B"], w["T"], w["short"], w["dtype"], seed)
    cfg.gemm_impl = gemm_impl
    cfg.attn_impl = attn_impl
    cfg.gemm_pair = gemm_pair
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    rows = [0, 3]
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, rows=rows, want_logits=True)
    _compare(loss[rows], ref_loss, logits[rows], ref_logits, "bf16")
    ref_all, _ = O.forward(ocfg, p, tok, tgt)
    _compare(loss, ref_all, dtype="bf16")


@pytest.mark.parametrize("depth,B,T,short,n_kv_head", [(4, 2, 512, 256, 1), (12, 1, 384, 128, 2), (12, 1, 256, 64, 3)])
def test_grouped_query_attention_forward(depth, B, T, short, n_kv_head):
    """H_kv < H: query head h reads k/v head h / (H / H_kv); the k/v and
    value-embedding widths shrink with H_kv (d4: H = 2; d12: H = 6)."""
    cfg, ocfg, p, tok, tgt = make_case(depth, B, T, short, "bf16", 300 + n_kv_head, n_kv_head=n_kv_head)
    assert cfg.n_kv_head == n_kv_head < cfg.n_head
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, rows=[0], want_logits=True)
    _compare(loss[:1], ref_loss, logits[:1], ref_logits, "bf16")


def test_tc_gemm_matches_cuda_core_gemm():
    """The tcgen05 and CUDA-core GEMMs round at the same points but sum in a
    different order; in bf16 that alone moves per-token losses by the bf16
    error level, so they are held to the same bounds as against the oracle."""
    cfg, ocfg, p, tok, tgt = make_case(4, 2, 384, 128, "bf16", 77)
    l0, z0, rc0, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    cfg.gemm_impl = 1
    l1, z1, rc1, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc0 == 0 and rc1 == 0
    _compare(l0, l1.astype(np.float64), z0, z1, "bf16")


@pytest.mark.parametrize("B,T", [(3, 200), (1, 1), (2, 129), (1, 77)])
def test_ragged_shapes_and_ignored_targets(B, T):
    cfg, ocfg, p, tok, tgt = make_case(4, B, T, 64, "bf16", 1000 + T, max_T=256)
    tgt = tgt.copy()
    tgt[0, ::3] = -1
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True, max_tokens=B * T + 5)
    assert rc == 0
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, want_logits=True)
    _compare(loss, ref_loss, logits, ref_logits, "bf16")
    assert np.all(loss[tgt == -1] == 0.0)


def test_fp32_ragged_window_one():
    cfg, ocfg, p, tok, tgt = make_case(2, 2, 70, 1, "fp32", 31, max_T=96)
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, want_logits=True)
    _compare(loss, ref_loss, logits, ref_logits, "fp32")


@pytest.mark.parametrize("name,rows,gemm_pair", [("d12", [0, 5], 1), ("d24", [2], 1), ("d24", [1], 2)])
def test_full_size_sampled_rows(name, rows, gemm_pair):
    """gemm_pair = 2 splits the partial last wave of FC2's tiles along K
    (partial sums through the workspace); at d24 that schedule is in use."""
    w = synth.WORKLOADS[name]
    seed = synth.SEED_BASE + w["index"]
    cfg, ocfg, p, tok, tgt = make_case(w["depth"], w["B"], w["T"], w["short"], w["dtype"], seed)
    cfg.gemm_pair = gemm_pair
    loss, _, rc, _ = run_gpu(cfg, p, tok, tgt)
    assert rc == 0
    ref_loss, _ = O.forward(ocfg, p, tok, tgt, rows=rows)
    _compare(loss[rows], ref_loss, dtype="bf16")


def test_out_of_range_ids_flag_data_error():
    cfg, ocfg, p, tok, tgt = make_case(1, 1, 16, 16, "bf16", 5)
    tok = tok.copy(); tgt = tgt.copy()
    tok[0, 3] = 40000
    tgt[0, 5] = -7
    loss, _, rc, _ = run_gpu(cfg, p, tok, tgt)
    assert rc == nc.STATUS_CODES["NC_ERR_DATA"]
    assert np.all(np.isfinite(loss))
    rc2, bits = nc.nc_get_status()
    assert rc2 == 0 and bits == 0  # reading clears the word


def test_loss_mean_and_host_entry_point():
    import torch
    cfg, ocfg, p, tok, tgt = make_case(4, 2, 256, 128, "bf16", 9)
    tgt = tgt.copy(); tgt[1, :10] = -1
    loss, _, rc, model = run_gpu(cfg, p, tok, tgt)
    assert rc == 0
    out = torch.empty(1, device="cuda")
    nc.nc_loss_mean(torch.from_numpy(loss.reshape(-1)).cuda(), torch.from_numpy(tgt.reshape(-1)).cuda(), out)
    valid = tgt != -1
    assert abs(out.item() - loss[valid].mean()) < 1e-5
    # host buffers in, host loss out: same numbers as the device entry point
    h_loss = torch.empty(tok.size, dtype=torch.float32).pin_memory()
    nc.nc_forward_host(model.params, torch.from_numpy(tok).pin_memory(),
                       torch.from_numpy(tgt).pin_memory(), h_loss)
    assert np.array_equal(h_loss.numpy().reshape(tok.shape), loss)
    # all targets ignored: the mean is NaN
    none = torch.full((8,), -1, dtype=torch.int32, device="cuda")
    nc.nc_loss_mean(torch.zeros(8, device="cuda"), none, out)
    assert np.isnan(out.item())


@pytest.mark.parametrize("B,T,short", [(4, 1024, 512), (2, 333, 100), (1, 128, 1)])
def test_tc_attention_forward(B, T, short):
    """The whole pass with the tcgen05 attention (attn_impl = 0) against the oracle."""
    cfg, ocfg, p, tok, tgt = make_case(4, B, T, short, "bf16", 4000 + T)
    cfg.attn_impl = 0
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=(B * T <= 1024))
    assert rc == 0
    rows = [0, B - 1] if B > 1 else [0]
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, rows=rows, want_logits=(B * T <= 1024))
    _compare(loss[rows], ref_loss, None if logits is None else logits[rows], ref_logits, "bf16")
