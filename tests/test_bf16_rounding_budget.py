"""Evidence for how the bf16-mode tolerances are applied.

bf16_emulation.py applies the bf16 roundings of the tensor-core path (GEMM A
operands, q/k/v, the softmax weights entering P V, the attention output, the
ReLU^2 output) to the oracle's own fp64 steps; rounding is the only
difference between the two runs.  These tests pin what that rounding alone
does on the seeded random-init workloads:
  * the per-token loss error is about 4e-3 rms, unbiased;
  * its tails pass the stated per-value tolerances: the logit error exceeds
    3e-2 on seeded cases (on about one logit in ten million), and the loss
    error exceeds 1e-2 on one to three percent of the tokens of every case.
So no implementation that rounds at these points can hold 1e-2 and 3e-2 as
maxima; bf16_parity.py holds the GPU to the emulation's error on the same
inputs instead.
"""
import numpy as np
import pytest

import bf16_emulation as E
from decoder_only_transformer_fwd_b200 import synth
from oracle import nanochat_fwd as O


def _case(depth, B, T, short, seed, max_T):
    cfg = O.make_config(depth, max_T, short)
    p = synth.params(seed, n_layer=depth, n_embd=cfg["n_embd"], n_head=cfg["n_head"],
                     n_kv_head=cfg["n_kv_head"], head_dim=128, vocab=32768, vocab_padded=32768,
                     ve_layers=cfg["ve_layers"], bf16=True)
    return cfg, p, synth.tokens(seed, B, T, 32768), synth.targets(seed, B, T, 32768)


def test_bf16_operand_rounding_sets_the_loss_error():
    cfg, p, tok, y = _case(4, 1, 512, 256, 20261, 512)
    exact, _ = O.forward(cfg, p, tok, y)
    rounded, _ = E.forward(cfg, p, tok, y)
    err = rounded[0] - exact[0]
    rms = float(np.sqrt(np.mean(err ** 2)))
    assert 3e-3 < rms < 6e-3, rms
    assert abs(err.mean()) < 1e-3


@pytest.mark.parametrize("seed", [5004, 5005])
def test_rounding_alone_exceeds_the_stated_logit_tolerance(seed):
    """d4, three rows of 200 tokens, short window 64 (the ragged-shape GPU case)."""
    cfg, p, tok, y = _case(4, 3, 200, 64, seed, 256)
    ex_l, ex_z = O.forward(cfg, p, tok, y, want_logits=True)
    em_l, em_z = E.forward(cfg, p, tok, y, want_logits=True)
    dz = np.abs(em_z - ex_z)
    assert dz.max() > 3.4e-2
    assert 0 < np.mean(dz > 3e-2) < 1e-6       # a handful of the 19.7M logits
    dl = np.abs(em_l - ex_l)
    assert dl.max() > 1.3e-2
    assert 0.01 < np.mean(dl > 1e-2) < 0.05     # a few percent of the tokens
