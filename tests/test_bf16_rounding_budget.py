"""Evidence for the bf16-mode loss tolerance.

The bf16 path rounds to bf16 exactly at the GEMM operands and stored
activations: the normalised block inputs, q and k after RoPE + QK-norm and v
after the value-embedding mix (all three applied to the fp32 accumulator of
the QKV GEMM), the attention output, the ReLU^2 output and the head input; everything else (the residual stream,
accumulation, softmax, softcap, log-sum-exp) stays in fp32 or better.  This
test applies those roundings to the oracle's own fp64 steps and measures the
per-token loss error they cause: its rms sets the bound the GPU parity tests
use (rms <= 6e-3), and it is large enough that a bound on the maximum of 1e-2
over thousands of tokens (about 3.5 sigma) could not hold for any bf16
implementation.  Rounding is the only difference between the two runs here.
"""
import numpy as np

from decoder_only_transformer_fwd_b200 import synth
from oracle import nanochat_fwd as O

F64 = np.float64


def _rb(a):
    return synth.round_bf16(np.asarray(a, np.float32)).astype(F64)


def _forward_rounded(cfg, p, tok, y):
    T = tok.shape[0]
    H, D, eps = cfg["n_head"], cfg["head_dim"], cfg["eps"]
    x = O.embed(cfg, p, tok)
    x0 = x.copy()
    x_bo = None
    pos = np.arange(T)
    for l in range(cfg["n_layer"]):
        lp = p["layers"][l]
        x = p["resid_lambdas"][l] * x + p["x0_lambdas"][l] * x0
        a = O.rmsnorm(x, eps)
        qkv = _rb(a) @ np.asarray(lp["w_qkv"], F64).T
        q = qkv[:, :H * D].reshape(T, H, D)
        k = qkv[:, H * D:2 * H * D].reshape(T, H, D)
        v = qkv[:, 2 * H * D:].reshape(T, H, D)
        if lp["ve"] is not None:
            g = O.ve_gate(a[:, :12], lp["ve_gate"])
            v = v + g[:, :, None] * np.asarray(lp["ve"], F64)[tok].reshape(T, H, D)
        v = _rb(v)
        qh = _rb(O.qk_norm(O.rope(q, pos), cfg["qk_alpha"], eps))
        kh = _rb(O.qk_norm(O.rope(k, pos), cfg["qk_alpha"], eps))
        o = _rb(O.attention(qh, kh, v, cfg["windows"][l], cfg["softmax_scale"]))
        x = x + o.reshape(T, H * D) @ np.asarray(lp["w_o"], F64).T
        h = _rb(O.relu2(_rb(O.rmsnorm(x, eps)) @ np.asarray(lp["w_fc1"], F64).T))
        x = x + h @ np.asarray(lp["w_fc2"], F64).T
        if l == cfg["backout_layer"]:
            x_bo = x.copy()
    x = x - float(p["backout_lambda"]) * x_bo
    z = _rb(O.rmsnorm(x, eps)) @ np.asarray(p["lm_head"][: cfg["vocab"]], F64).T
    return O.cross_entropy_per_token(O.softcap(z), y)


def test_bf16_operand_rounding_sets_the_loss_error():
    depth, T = 4, 512
    cfg = O.make_config(depth, T, T // 2)
    p = synth.params(20261, n_layer=depth, n_embd=cfg["n_embd"], n_head=cfg["n_head"],
                     n_kv_head=cfg["n_kv_head"], head_dim=128, vocab=32768, vocab_padded=32768,
                     ve_layers=cfg["ve_layers"], bf16=True)
    tok = synth.tokens(20261, 1, T, 32768)
    y = synth.targets(20261, 1, T, 32768)
    exact, _ = O.forward(cfg, p, tok, y)
    rounded = _forward_rounded(cfg, p, tok[0].astype(np.int64), y[0])
    err = rounded - exact[0]
    rms = float(np.sqrt(np.mean(err ** 2)))
    # sigma of the bf16 per-token loss error: well above what a 1e-2 bound on
    # the max over >= 2048 tokens tolerates (1e-2 / 3.5), inside the 6e-3 bound
    assert 1e-2 / 3.5 < rms < 6e-3, rms
    assert abs(err.mean()) < 1e-3
    assert np.max(np.abs(err)) < 3e-2
