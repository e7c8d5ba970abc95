"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances.  fp32 mode: per-token loss and softcapped logits within 1e-4 of
the oracle, every value.  bf16 mode (bf16 GEMM operands and stored
activations, fp32 accumulation): the stated tolerances are 1e-2 on the
per-token loss and 3e-2 on the logits; bf16_parity.py applies them against
the emulation of the same bf16 roundings on the same inputs (the share of
values beyond them, the rms and the maximum may not exceed what rounding at
those points produces), because that rounding alone already exceeds both
numbers on some values of most cases.

Small cases are compared element by element; the d12 / d24
workloads run at full size on the GPU and are compared on whole sampled rows
(rows are independent sequences, so a row of the oracle is exact for that
row of the batch)."""
import numpy as np
import pytest

import bf16_emulation as E
import bf16_parity
from decoder_only_transformer_fwd_b200 import nc, synth
from nc_cases import make_case, run_gpu
from oracle import nanochat_fwd as O

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-4


def _compare_fp32(gpu_loss, ref_loss, gpu_logits=None, ref_logits=None):
    assert np.all(np.isfinite(gpu_loss))
    assert float(np.max(np.abs(gpu_loss - ref_loss))) <= FP32_TOL
    if gpu_logits is not None:
        assert float(np.max(np.abs(gpu_logits - ref_logits))) <= FP32_TOL
        assert np.all(np.abs(gpu_logits) <= 15.0)


def _compare_bf16(ocfg, p, tok, tgt, rows, gpu_loss, gpu_logits=None, cuda_core=(False, False)):
    """gpu_loss / gpu_logits hold the given rows; cuda_core = (gemm_impl, attn_impl) == 1."""
    want = gpu_logits is not None
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, rows=rows, want_logits=want)
    emu_loss, emu_logits = E.forward(ocfg, p, tok, tgt, rows=rows, want_logits=want,
                                     qkv_store=cuda_core[0], round_p=not cuda_core[1])
    stats = bf16_parity.check_forward(gpu_loss, ref_loss, emu_loss, gpu_logits, ref_logits, emu_logits)
    print({k: {"gpu": g, "emulation": e} for k, (g, e) in stats.items()})


def test_d1_fp32_full():
    w = synth.WORKLOADS["d1"]
    seed = synth.SEED_BASE + w["index"]
    cfg, ocfg, p, tok, tgt = make_case(w["depth"], w["B"], w["T"], w["short"], w["dtype"], seed)
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, want_logits=True)
    _compare_fp32(loss, ref_loss, logits, ref_logits)


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
    cc = (gemm_impl == 1, attn_impl == 1)
    _compare_bf16(ocfg, p, tok, tgt, [0, 3], loss[[0, 3]], logits[[0, 3]], cuda_core=cc)
    _compare_bf16(ocfg, p, tok, tgt, [1, 2], loss[[1, 2]], cuda_core=cc)


@pytest.mark.parametrize("depth,B,T,short,n_kv_head", [(4, 2, 512, 256, 1), (12, 1, 384, 128, 2), (12, 1, 256, 64, 3)])
def test_grouped_query_attention_forward(depth, B, T, short, n_kv_head):
    """H_kv < H: query head h reads k/v head h / (H / H_kv); the k/v and
    value-embedding widths shrink with H_kv (d4: H = 2; d12: H = 6)."""
    cfg, ocfg, p, tok, tgt = make_case(depth, B, T, short, "bf16", 300 + n_kv_head, n_kv_head=n_kv_head)
    assert cfg.n_kv_head == n_kv_head < cfg.n_head
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    _compare_bf16(ocfg, p, tok, tgt, [0], loss[:1], logits[:1])


def test_tc_gemm_matches_cuda_core_gemm():
    """The tcgen05 and CUDA-core GEMMs round at nearly the same points but sum
    in a different order; each is held to the oracle, and the two differ from
    each other by no more than two independent draws of the bf16 rounding
    noise (rms at most twice the emulation's error)."""
    cfg, ocfg, p, tok, tgt = make_case(4, 2, 384, 128, "bf16", 77)
    l0, z0, rc0, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    cfg.gemm_impl = 1
    l1, z1, rc1, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc0 == 0 and rc1 == 0
    _compare_bf16(ocfg, p, tok, tgt, [0, 1], l0, z0)
    _compare_bf16(ocfg, p, tok, tgt, [0, 1], l1, z1, cuda_core=(True, False))
    ref, _ = O.forward(ocfg, p, tok, tgt)
    emu, _ = E.forward(ocfg, p, tok, tgt)
    rms = lambda d: float(np.sqrt(np.mean(np.asarray(d, np.float64) ** 2)))
    assert rms(l0 - l1) <= 2.0 * rms(emu - ref)


@pytest.mark.parametrize("B,T", [(3, 200), (1, 1), (2, 129), (1, 77)])
def test_ragged_shapes_and_ignored_targets(B, T):
    cfg, ocfg, p, tok, tgt = make_case(4, B, T, 64, "bf16", 1000 + T, max_T=256)
    tgt = tgt.copy()
    tgt[0, ::3] = -1
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True, max_tokens=B * T + 5)
    assert rc == 0
    _compare_bf16(ocfg, p, tok, tgt, list(range(B)), loss, logits)
    assert np.all(loss[tgt == -1] == 0.0)


def test_fp32_ragged_window_one():
    cfg, ocfg, p, tok, tgt = make_case(2, 2, 70, 1, "fp32", 31, max_T=96)
    loss, logits, rc, _ = run_gpu(cfg, p, tok, tgt, want_logits=True)
    assert rc == 0
    ref_loss, ref_logits = O.forward(ocfg, p, tok, tgt, want_logits=True)
    _compare_fp32(loss, ref_loss, logits, ref_logits)


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
    _compare_bf16(ocfg, p, tok, tgt, rows, loss[rows])


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
    h_tok, h_tgt = torch.from_numpy(tok).pin_memory(), torch.from_numpy(tgt).pin_memory()
    nc.nc_forward_host(model.params, h_tok, h_tgt, h_loss)
    torch.cuda.synchronize()  # the call is asynchronous: the loss is on the host after a sync
    assert np.array_equal(h_loss.numpy().reshape(tok.shape), loss)
    # consecutive calls on one stream pipeline; each one's loss lands in its own buffer
    h_loss2 = torch.full((tok.size,), float("nan"), dtype=torch.float32).pin_memory()
    for buf in (h_loss2, h_loss, h_loss2):
        nc.nc_forward_host(model.params, h_tok, h_tgt, buf)
    torch.cuda.synchronize()
    assert np.array_equal(h_loss2.numpy().reshape(tok.shape), loss)
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
    _compare_bf16(ocfg, p, tok, tgt, rows, loss[rows], None if logits is None else logits[rows])
