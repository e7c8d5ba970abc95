"""GPU parity of one generation step ("The Mathematics of Karpathy's nanochat",
§Inference: Generating Text, §Sampling Controls) against the oracle.

* nc_last_logits: the softcapped logits of the last position of each row,
  compared element by element with the oracle's logits at that position
  (fp32: 1e-4; bf16: the stated 3e-2, applied against the emulation of the
  same bf16 roundings on the same inputs as for the full forward, see
  bf16_parity.py).
* nc_sample on given fp32 logits: greedy picks and the top-k kept set are
  decided on the same fp32 values on both sides and compared exactly; a
  multinomial draw is correct when the row's u lies in the drawn token's
  interval of the oracle's fp64 cumulative distribution, up to 2e-5 (fp32
  weights and a 1024-way prefix sum).  Where u is further than that from
  every interval edge, the token must equal the oracle's.
"""
import numpy as np
import pytest

import bf16_emulation as E
import bf16_parity
from decoder_only_transformer_fwd_b200 import nc, synth
from nc_cases import make_case
from oracle import nanochat_fwd as O
from oracle import sampling as S

pytestmark = pytest.mark.gpu

U_TOL = 2e-5
FP32_TOL = 1e-4


def _check_last_logits(ocfg, p, tok, z, dtype, rows=None):
    """z [len(rows), V]: the GPU's last-position logits of the given rows."""
    T = tok.shape[1]
    _, ref = O.forward(ocfg, p, tok, None, rows=rows, want_logits=True, positions=[T - 1])
    ref = ref[:, 0, :]
    if dtype == "fp32":
        assert float(np.max(np.abs(z - ref))) <= FP32_TOL
    else:
        _, emu = E.forward(ocfg, p, tok, None, rows=rows, want_logits=True, positions=[T - 1])
        bf16_parity.check("logits", z, ref, emu[:, 0, :])
    assert np.all(np.abs(z) <= 15.0)


def _sample(z, tau, k, u):
    import torch
    dz = torch.from_numpy(np.ascontiguousarray(z, dtype=np.float32)).cuda()
    du = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).cuda()
    out = torch.full((z.shape[0],), -7, dtype=torch.int32, device="cuda")
    nc.nc_sample(dz, tau, k, du, out)
    torch.cuda.synchronize()
    rc, _ = nc.nc_get_status()
    return out.cpu().numpy(), rc


def _check_draws(z, tau, k, u, got):
    z64 = z.astype(np.float64)
    exact = 0
    for b in range(z.shape[0]):
        v = int(got[b])
        assert 0 <= v < z.shape[1]
        if tau == 0:
            assert v == S.greedy(z64[b]), b
            continue
        assert np.isfinite(S.top_k_filter(z64[b], k)[v]), (b, v)   # in the kept set
        lo, hi = S.draw_interval(z64[b], tau, k, v)
        assert lo - U_TOL <= u[b] < hi + U_TOL, (b, v, lo, hi, u[b])
        ref = S.sample_next(z64[b], tau, k, float(u[b]))
        rlo, rhi = S.draw_interval(z64[b], tau, k, ref)
        if u[b] - rlo > U_TOL and rhi - u[b] > U_TOL:
            assert v == ref, (b, v, ref)
            exact += 1
    return exact


@pytest.mark.parametrize("V,ties", [(32768, 0), (1000, 3), (7, 0), (1, 0)])
def test_greedy_exact(V, ties):
    B = 16
    z = synth.sampling_logits(40 + V, B, V, ties=ties)
    if V > 10:
        z[:, V - 3] = z.max(axis=1)      # a later copy of each row's maximum
    u = synth.uniforms(40 + V, B)
    got, rc = _sample(z, 0.0, 50, u)
    assert rc == 0
    _check_draws(z, 0.0, 50, u, got)


@pytest.mark.parametrize("V,tau,k,ties", [
    (32768, 0.8, 50, 0), (32768, 1.0, 0, 0), (32768, 1.3, 1, 0), (32768, 0.7, 5, 6),
    (50000, 0.9, 40, 0),  # beyond the shared-memory row: read from global memory
    (1000, 1.0, 1000, 0), (1000, 2.0, 999, 2), (7, 2.0, 3, 0), (1, 1.0, 0, 0), (2049, 5.0, 0, 0)])
def test_sampling_matches_oracle(V, tau, k, ties):
    B = 64
    z = synth.sampling_logits(V + k, B, V, ties=ties)
    u = synth.uniforms(V + k, B)
    got, rc = _sample(z, tau, k, u)
    assert rc == 0
    exact = _check_draws(z, tau, k, u, got)
    assert exact >= B // 2 or V == 1


@pytest.mark.parametrize("V,k,lo", [(32768, 50, 1.0), (32768, 16384, 1.0), (32768, 16384, 0.5), (50000, 7, 4.0)])
def test_top_k_when_one_binade_holds_the_row(V, k, lo):
    """All logits in one binade put every key in the top digit's bin, far more
    than the 4096 candidates the select compacts: the lower digits are then
    counted over the whole row."""
    B = 8
    z = synth.binade_logits(3100 + k, B, V, lo)
    u = synth.uniforms(3100 + k, B)
    got, rc = _sample(z, 1.0, k, u)
    assert rc == 0
    exact = _check_draws(z, 1.0, k, u, got)
    # with thousands of near-equal weights most u fall within the tolerance of
    # an interval edge, where a draw is checked for validity only
    assert exact >= B // 2 or k > 1024


def test_top_k_ties_are_all_kept():
    # every row: 5th-largest value repeated 6 times; k = 5 keeps all of them,
    # and a u grid walks through every kept token
    V, B = 4096, 1
    z = synth.sampling_logits(77, B, V, ties=6)
    kept = np.nonzero(np.isfinite(S.top_k_filter(z[0].astype(np.float64), 5)))[0]
    assert len(kept) > 5
    n = 512
    zz = np.repeat(z, n, axis=0)
    u = ((np.arange(n) + 0.5) / n).astype(np.float32)
    got, rc = _sample(zz, 50.0, 5, u)    # high temperature: all kept tokens get a share
    assert rc == 0
    _check_draws(zz, 50.0, 5, u, got)
    assert set(got.tolist()) == set(kept.tolist())


def test_uniform_out_of_range_is_flagged_and_clamped():
    z = synth.sampling_logits(3, 2, 300)
    u = np.array([1.5, -0.25], dtype=np.float32)
    got, rc = _sample(z, 1.0, 0, u)
    assert rc == nc.STATUS_CODES["NC_ERR_DATA"]
    assert all(0 <= int(v) < 300 for v in got)


def _last_logits(cfg, p, tok):
    import torch
    B, T = tok.shape
    model = nc.NcModel(cfg, p, B * T)
    out = torch.empty(B, cfg.vocab, dtype=torch.float32, device="cuda")
    nc.nc_last_logits(model.params, torch.from_numpy(tok).cuda(), out)
    torch.cuda.synchronize()
    rc, _ = nc.nc_get_status()
    return out.cpu().numpy(), rc, model


@pytest.mark.parametrize("depth,B,T,short,dtype", [
    (4, 2, 300, 128, "bf16"), (4, 9, 64, 32, "bf16"), (1, 3, 77, 77, "fp32"), (12, 1, 200, 64, "bf16")])
def test_last_logits_match_oracle(depth, B, T, short, dtype):
    """bf16 runs the tensor-core form (up to 16 rows per launch, so B = 9 is
    one launch); fp32 runs the CUDA-core form (eight rows per launch)."""
    cfg, ocfg, p, tok, _ = make_case(depth, B, T, short, dtype, 600 + B * T)
    z, rc, _ = _last_logits(cfg, p, tok)
    assert rc == 0
    _check_last_logits(ocfg, p, tok, z, dtype)


@pytest.mark.parametrize("V,B", [(1000, 3), (50000, 17)])
def test_last_logits_vocab_shapes(V, B):
    """Vocabularies that are not a multiple of the 32-row unit the tensor-core
    head streams W_U in: V = 1000 (fewer units than SMs, a partial last unit)
    and V = 50000 (more than eight units per CTA, so the CTAs take two passes
    through their two TMEM buffers); B = 17 spans two launches of 16 rows."""
    import torch
    depth, T, short = 2, 48, 32
    cfg = nc.nc_init_config(depth, T, "bf16", "SSSL", short, -1)
    cfg.vocab = V
    cfg.vocab_padded = O.padded_vocab(V)
    ocfg = O.make_config(depth, T, short, vocab=V)
    seed = 900 + V + B
    p = synth.params(seed, n_layer=cfg.n_layer, n_embd=cfg.n_embd, n_head=cfg.n_head, n_kv_head=cfg.n_kv_head,
                     head_dim=cfg.head_dim, vocab=V, vocab_padded=cfg.vocab_padded, ve_layers=ocfg["ve_layers"],
                     bf16=True)
    tok = synth.tokens(seed, B, T, V)
    z, rc, _ = _last_logits(cfg, p, tok)
    assert rc == 0
    assert z.shape == (B, V)
    _check_last_logits(ocfg, p, tok, z, "bf16")


def test_last_logits_equal_full_forward_last_position():
    """The GEMV head and the tcgen05 head GEMM give the same logits at the last
    position, up to their different summation orders."""
    import torch
    cfg, ocfg, p, tok, tgt = make_case(4, 3, 256, 128, "bf16", 61)
    z, rc, model = _last_logits(cfg, p, tok)
    assert rc == 0
    _, full = model.forward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda(), want_logits=True)
    full = full.view(3, 256, -1)[:, -1, :].cpu().numpy()
    assert float(np.max(np.abs(z - full))) <= 2e-3


@pytest.mark.parametrize("tau,k", [(0.0, 0), (0.8, 50)])
def test_generate_next_d24(tau, k):
    """The generation step at d24 sizes (B = 4, T = 2048): the logits of row 3
    against the oracle, and the drawn tokens against the oracle's sampler on
    the GPU's own logits."""
    import torch
    w = synth.WORKLOADS["d24"]
    seed = synth.SEED_BASE + w["index"]
    cfg, ocfg, p, tok, _ = make_case(w["depth"], w["B"], w["T"], w["short"], w["dtype"], seed)
    model = nc.NcModel(cfg, p, w["B"] * w["T"])
    u = synth.uniforms(seed, w["B"])
    nxt, z = model.generate_next(torch.from_numpy(tok).cuda(), torch.from_numpy(u).cuda(), tau, k)
    torch.cuda.synchronize()
    rc, _ = nc.nc_get_status()
    assert rc == 0
    z = z.cpu().numpy()
    _check_draws(z, tau, k, u, nxt.cpu().numpy())
    if tau == 0.0:
        _check_last_logits(ocfg, p, tok, z[3:4], "bf16", rows=[3])
