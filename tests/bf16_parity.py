"""Parity check of the bf16 mode against the oracle, with the emulation of the
same bf16 roundings as the yardstick.

TEST INFRASTRUCTURE.

The stated bf16 tolerances are per-token loss within 1e-2 and softcapped
logits within 3e-2 of the fp64 oracle.  Rounding the GEMM operands and stored
activations to bf16 (and nothing else) already moves the per-token loss and
the logits by about 4e-3 rms for these random-init weights, and that noise has
heavy tails: the emulation in bf16_emulation.py, whose only difference from
the oracle is that rounding, exceeds 3e-2 on some logits and 1e-2 on a few
percent of the tokens in most seeded cases (test_bf16_rounding_budget.py pins
both facts).  No implementation that rounds at these points can hold the two
numbers as maxima, so they are applied as follows, per compared case:
  * the share of values beyond the stated tolerance may be at most twice the
    emulation's share on the same inputs (plus one value in a million, or two
    values, for the logits, and one token for the loss);
  * the rms error may be at most 1.25 times the emulation's, plus 2e-4;
  * the maximum error may exceed the stated tolerance only up to 1.5 times the
    emulation's maximum on the same inputs;
  * the mean loss is within 1e-3 of the oracle's.
A wiring or indexing fault gives errors of order one, far outside all four.
"""
from __future__ import annotations

import numpy as np

# the stated bf16 tolerances: per-token loss and softcapped logits, absolute
STATED_TOL = {"loss": 1e-2, "logits": 3e-2}


def _stats(err, tol):
    err = np.abs(np.asarray(err, np.float64)).ravel()
    return {"n": err.size, "max": float(err.max()), "rms": float(np.sqrt(np.mean(err ** 2))),
            "beyond": float(np.mean(err > tol))}


def check(kind, gpu, ref, emu):
    """Assert the rules above for one kind of output ('loss' or 'logits');
    returns the GPU's and the emulation's statistics."""
    tol = STATED_TOL[kind]
    assert np.all(np.isfinite(gpu)), f"{kind}: non-finite values"
    g = _stats(np.asarray(gpu, np.float64) - ref, tol)
    e = _stats(np.asarray(emu, np.float64) - ref, tol)
    slack = max(1e-6, 2.0 / g["n"]) if kind == "logits" else 1.0 / g["n"]
    assert g["beyond"] <= 2.0 * e["beyond"] + slack, \
        f"{kind}: {g['beyond']:.2e} of values beyond {tol} (emulation {e['beyond']:.2e})"
    assert g["rms"] <= 1.25 * e["rms"] + 2e-4, f"{kind}: rms {g['rms']:.3e} (emulation {e['rms']:.3e})"
    assert g["max"] <= max(tol, 1.5 * e["max"]), f"{kind}: max {g['max']:.3e} (emulation {e['max']:.3e})"
    return g, e


def check_forward(gpu_loss, ref_loss, emu_loss, gpu_logits=None, ref_logits=None, emu_logits=None):
    out = {"loss": check("loss", gpu_loss, ref_loss, emu_loss)}
    assert abs(float(np.mean(gpu_loss)) - float(np.mean(ref_loss))) <= 1e-3
    if gpu_logits is not None:
        out["logits"] = check("logits", gpu_logits, ref_logits, emu_logits)
        assert np.all(np.abs(gpu_logits) <= 15.0)
    return out
