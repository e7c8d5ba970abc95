"""GPU parity of the head backward (nc_head_backward) against the oracle's
head_backward: dL/dx of the final residual and dL/dW_U of the mean softcapped
cross-entropy.

The oracle takes the final residual x as its input.  Two kinds of cases:
  * identity blocks (W_O = W_2 = 0, the page's own initialisation of those
    matrices, "The Mathematics of Karpathy's nanochat" §Initialisation): every
    block then adds only the x0 re-injection, so the GPU's final residual is
    the oracle's up to fp32 rounding, and the comparison isolates the backward
    kernels.  Their own roundings are the bf16 operands (the normalised x as
    the forward's head consumes it, and dL/dz stored in bf16): tolerance 1e-2
    of the largest entry on every element, 3e-3 of the rms in rms;
  * random-init blocks, where the GPU's final residual also carries the bf16
    forward's noise (the logits move by ~4e-3 rms, so p = softmax moves by
    about that relative amount): 4e-2 / 1.5e-2.
The d24 case checks dL/dx on one sampled row (a row's dx depends on the other
rows only through the count of valid targets, which scales it)."""
import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc, synth
from nc_cases import make_case
from oracle import head_backward as HB
from oracle import nanochat_fwd as O

pytestmark = pytest.mark.gpu


def _final_residual(ocfg, p, tok_row):
    """The oracle's final residual of one row: the blocks, then backout."""
    x = O.embed(ocfg, p, tok_row.astype(np.int64))
    x0 = x.copy()
    x_bo = None
    for l in range(ocfg["n_layer"]):
        x = O.block(ocfg, p["layers"][l], l, x, tok_row.astype(np.int64), p["resid_lambdas"][l],
                    p["x0_lambdas"][l], x0)
        if l == ocfg["backout_layer"]:
            x_bo = x.copy()
    return x - float(p["backout_lambda"]) * x_bo


def _gpu(cfg, p, tok, tgt):
    import torch
    B, T = tok.shape
    model = nc.NcModel(cfg, p, B * T)
    t, y = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    loss, _ = model.forward(t, y)
    dx = torch.empty(B * T, cfg.n_embd, dtype=torch.float32, device="cuda")
    dw = torch.full((cfg.vocab, cfg.n_embd), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(nc.nc_head_backward_workspace_bytes(cfg, B * T), dtype=torch.uint8, device="cuda")
    nc.nc_head_backward(model.params, y, dx, dw, ws)
    torch.cuda.synchronize()
    rc, bits = nc.nc_get_status()
    assert rc == 0, bits
    return loss.cpu().numpy(), dx.cpu().numpy(), dw.cpu().numpy()


def _close(got, ref, max_frac, rms_frac, what):
    assert np.all(np.isfinite(got)), what
    d = np.abs(got.astype(np.float64) - ref)
    scale_max, scale_rms = float(np.abs(ref).max()), float(np.sqrt(np.mean(ref ** 2)))
    emax, erms = float(d.max()), float(np.sqrt(np.mean(d ** 2)))
    print(f"{what}: max err {emax:.3e} ({emax / scale_max:.2e} of max), rms err {erms:.3e} "
          f"({erms / scale_rms:.2e} of rms)")
    assert emax <= max_frac * scale_max, what
    assert erms <= rms_frac * scale_rms, what


@pytest.mark.parametrize("identity,B,T,ignore", [(True, 2, 256, False), (True, 3, 77, True), (False, 2, 256, True)])
def test_head_backward_d4(identity, B, T, ignore):
    cfg, ocfg, p, tok, tgt = make_case(4, B, T, 128, "bf16", 900 + T + B)
    if identity:
        for lp in p["layers"]:
            lp["w_o"] = np.zeros_like(lp["w_o"])
            lp["w_fc2"] = np.zeros_like(lp["w_fc2"])
    tgt = tgt.copy()
    if ignore:
        tgt[0, ::5] = -1
    loss, dx, dw = _gpu(cfg, p, tok, tgt)
    x = np.concatenate([_final_residual(ocfg, p, tok[b]) for b in range(B)])
    w_u = np.asarray(p["lm_head"][:cfg.vocab], np.float64)
    rdx, rdw, rloss = HB.head_backward(x, w_u, tgt.reshape(-1), cap=ocfg["softcap"], eps=ocfg["eps"])
    tol = (1e-2, 3e-3) if identity else (4e-2, 1.5e-2)
    _close(dx, rdx, *tol, "dL/dx")
    _close(dw, rdw, *tol, "dL/dW_U")
    valid = tgt.reshape(-1) != -1
    assert abs(float(loss[valid].mean()) - rloss) < 2e-3
    assert np.all(dx.reshape(B, T, -1)[tgt == -1] == 0.0)   # ignored rows get no gradient


def test_head_backward_no_valid_target_gives_zero():
    cfg, ocfg, p, tok, tgt = make_case(1, 1, 64, 64, "bf16", 17)
    _, dx, dw = _gpu(cfg, p, tok, np.full_like(tgt, -1))
    assert np.all(dx == 0.0) and np.all(dw == 0.0)


def test_head_backward_d24_sampled_row():
    w = synth.WORKLOADS["d24"]
    seed = synth.SEED_BASE + w["index"]
    cfg, ocfg, p, tok, tgt = make_case(w["depth"], w["B"], w["T"], w["short"], w["dtype"], seed)
    _, dx, _ = _gpu(cfg, p, tok, tgt)
    row = 1
    x = _final_residual(ocfg, p, tok[row])
    rdx, _, _ = HB.head_backward(x, np.asarray(p["lm_head"][:cfg.vocab], np.float64), tgt[row],
                                 cap=ocfg["softcap"], eps=ocfg["eps"])
    n_row, n_all = int((tgt[row] != -1).sum()), int((tgt != -1).sum())
    rdx *= n_row / n_all    # the oracle's mean over this row's targets -> over the whole batch's
    T = w["T"]
    _close(dx[row * T:(row + 1) * T], rdx, 4e-2, 1.5e-2, "d24 row dL/dx")
