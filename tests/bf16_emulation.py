"""The oracle's forward pass with the bf16 roundings of the tensor-core path.

TEST INFRASTRUCTURE (imports the oracle; nothing here is used by the library).

The bf16 mode rounds to bf16 at exactly these points and keeps everything
else in fp32 or better:
  * the A operand of the QKV, FC1 and head GEMMs: bf16(x) of the fp32
    residual, the product then scaled by 1/rms(x) per row (RMSNorm without a
    weight, fused into the GEMM);
  * q and k after RoPE + QK-norm, and v after the value-embedding mix (all on
    the fp32 accumulator of the QKV GEMM);
  * the softmax weights p = exp(s - m) that enter the P V product (the row sum
    that normalises the output stays fp32, over the unrounded p);
  * the attention output o (the O-projection's A operand);
  * the ReLU^2 output h (the FC2's A operand).
The CUDA-core path (gemm_impl = 1, attn_impl = 1) rounds at slightly
different points: its QKV GEMM stores q, k and v in bf16 before RoPE +
QK-norm and the value-embedding mix round them again (qkv_store=True), and its
attention keeps p in fp32 (round_p=False).
This module applies those roundings to the oracle's own fp64 steps, so that
rounding is the only difference between its result and the oracle's.  The GPU
parity tests compare the GPU's error against this emulation's error on the
same inputs: both come from the same rounding points, so their sizes must
agree, while the particular values differ (a rounding that falls the other
way in one place moves everything downstream).
"""
from __future__ import annotations

import numpy as np

from decoder_only_transformer_fwd_b200 import synth
from oracle import nanochat_fwd as O

F64 = np.float64


def rb(a):
    """Round to the nearest bf16 (ties to even), returned as float64."""
    return synth.round_bf16(np.asarray(a, np.float32)).astype(F64)


def _normed_operand(x, eps):
    """bf16(x) * (1 / rms(x)): the fused-RMSNorm A operand, exactly as consumed."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return rb(x) * r


def _attention(q, k, v, window, scale, round_p):
    T, H, D = q.shape
    group = H // k.shape[1]
    mask = O.window_mask(T, window)
    out = np.empty((T, H, D), F64)
    for h in range(H):
        s = scale * (q[:, h, :] @ k[:, h // group, :].T)
        s = np.where(mask, s, -np.inf)
        p = np.exp(s - np.max(s, axis=1, keepdims=True))
        pv = rb(p) if round_p else p
        out[:, h, :] = (pv @ v[:, h // group, :]) / p.sum(axis=1, keepdims=True)
    return out


def forward_row(cfg, p, tok, y, positions=None, want_logits=False, qkv_store=False, round_p=True):
    """One row: (per-token loss or None, softcapped logits or None)."""
    tok = np.asarray(tok, np.int64)
    T = tok.shape[0]
    H, Hkv, D, eps = cfg["n_head"], cfg["n_kv_head"], cfg["head_dim"], cfg["eps"]
    x = O.embed(cfg, p, tok)
    x0 = x.copy()
    x_bo = None
    pos = np.arange(T)
    for l in range(cfg["n_layer"]):
        lp = p["layers"][l]
        x = p["resid_lambdas"][l] * x + p["x0_lambdas"][l] * x0
        a = O.rmsnorm(x, eps)
        qkv = _normed_operand(x, eps) @ np.asarray(lp["w_qkv"], F64).T
        if qkv_store:
            qkv = rb(qkv)
        q = qkv[:, :H * D].reshape(T, H, D)
        k = qkv[:, H * D:(H + Hkv) * D].reshape(T, Hkv, D)
        v = qkv[:, (H + Hkv) * D:].reshape(T, Hkv, D)
        if lp.get("ve") is not None:
            g = O.ve_gate(a[:, :cfg["gate_channels"]], lp["ve_gate"], cfg["ve_gate_scale"])
            v = v + g[:, :, None] * np.asarray(lp["ve"], F64)[tok].reshape(T, Hkv, D)
        v = rb(v)
        qh = rb(O.qk_norm(O.rope(q, pos, cfg["rope_base"]), cfg["qk_alpha"], eps))
        kh = rb(O.qk_norm(O.rope(k, pos, cfg["rope_base"]), cfg["qk_alpha"], eps))
        o = rb(_attention(qh, kh, v, cfg["windows"][l], cfg["softmax_scale"], round_p))
        x = x + o.reshape(T, H * D) @ np.asarray(lp["w_o"], F64).T
        h = rb(O.relu2(_normed_operand(x, eps) @ np.asarray(lp["w_fc1"], F64).T))
        x = x + h @ np.asarray(lp["w_fc2"], F64).T
        if l == cfg["backout_layer"]:
            x_bo = x.copy()
    if x_bo is not None:
        x = x - float(p["backout_lambda"]) * x_bo
    sel = pos if positions is None else np.asarray(positions, np.int64)
    z = _normed_operand(x[sel], eps) @ np.asarray(p["lm_head"][:cfg["vocab"]], F64).T
    zh = O.softcap(z, cfg["softcap"])
    loss = None if y is None else O.cross_entropy_per_token(zh, np.asarray(y)[sel])
    return loss, (zh if want_logits else None)


def forward(cfg, p, tokens, targets=None, rows=None, want_logits=False, positions=None, qkv_store=False,
            round_p=True):
    """Same calling convention and return shapes as the oracle's forward()."""
    tokens = np.asarray(tokens)
    rows = list(range(tokens.shape[0])) if rows is None else list(rows)
    losses, logits = [], []
    for b in rows:
        y = None if targets is None else np.asarray(targets)[b]
        l, z = forward_row(cfg, p, tokens[b], y, positions, want_logits, qkv_store, round_p)
        if l is not None:
            losses.append(l)
        if want_logits:
            logits.append(z)
    return (np.stack(losses) if losses else None), (np.stack(logits) if want_logits else None)
