"""Plain fp64 CPU definition of the nanochat GPT forward pass, from token ids to
per-token softcapped cross-entropy.

TEST INFRASTRUCTURE.  This module is the oracle the CUDA path is checked
against.  Only the test suite, the smoke check and the benchmark's CPU-baseline
leg may import it; the library itself never does, and nothing here is shared
with the CUDA kernels.

It is written straight from the equations of "The Mathematics of Karpathy's
nanochat" (cited below as [Math], with its section names) and the two pages
that describe the later nanochat commit: the "nanochat depth sweep" model card
([Sweep], Architecture list) and "Reading nanochat Source" ([Source], §5
Forward pass, shape by shape).  Every step is the definition itself in float64;
library routines (matmul, exp, tanh) serve as steps, with no blocking, fusion
or reordering.

Readings taken where the pages are silent or disagree (each also listed in
the design notes):
  * softmax scale: 1/sqrt(D) by default; [Math] omits it, the looped-nanochat
    card's formula and the FA3/SDPA call of [Source] §5.2 use it.  A parameter.
  * smear ([Sweep] "smear", [Source] §5.1 give no formula): additive,
    token-dependent scalar gate shaped like the value-embedding gate:
    s_t = sigmoid(w_sm . xhat_t[:12]), x_t = xhat_t + s_t * xhat_{t-1} (t >= 1).
    Parity unpinned beyond its own definition and its reductions.
  * x0 is the embedding after smear.
  * backout ([Sweep] "backout"): x_bo is the output of block L//2 (0-indexed);
    before the final norm x <- x - beta * x_bo.
  * value-embedding gate input: the normalised block input a = RMSNorm(x).
  * RMSNorm epsilon 1e-6 inside the square root, at every norm site.
  * window: key j is visible to query i iff j <= i and i - j < w.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# model shape  ([Math] §Architecture Overview; [Sweep] Models table notes)
# ---------------------------------------------------------------------------

def model_dims(depth: int, aspect_ratio: int = 64, head_dim: int = 128):
    """d_model = ceil(depth * aspect / head_dim) * head_dim, H = d_model / head_dim."""
    base = depth * aspect_ratio
    C = ((base + head_dim - 1) // head_dim) * head_dim
    return C, C // head_dim


def has_ve(layer: int, n_layer: int) -> bool:
    """[Math] §Value Embeddings: has_ve(l) = [l mod 2 == (L - 1) mod 2]."""
    return layer % 2 == (n_layer - 1) % 2


def layer_windows(n_layer: int, long_window: int, short_window: int, pattern: str = "SSSL"):
    """[Math] §Sliding Window Pattern: the pattern string is tiled over the layers,
    'L' = long (full context), 'S' = short; the last layer is always long."""
    w = [long_window if pattern[l % len(pattern)] == "L" else short_window for l in range(n_layer)]
    w[-1] = long_window
    return w


def padded_vocab(V: int, multiple: int = 64) -> int:
    """[Source] §5.4: the vocabulary is padded to a multiple of 64, then sliced back."""
    return ((V + multiple - 1) // multiple) * multiple


def make_config(depth: int, seq_len: int, short_window: int, *, vocab: int = 32768,
                pattern: str = "SSSL", backout_layer: int | None = None,
                n_kv_head: int | None = None, softmax_scale: float | None = None) -> dict:
    C, H = model_dims(depth)
    D = 128
    return {
        "n_layer": depth, "n_embd": C, "n_head": H,
        "n_kv_head": H if n_kv_head is None else n_kv_head, "head_dim": D,
        "vocab": vocab, "vocab_padded": padded_vocab(vocab),
        "windows": layer_windows(depth, seq_len, short_window, pattern),
        "ve_layers": [l for l in range(depth) if has_ve(l, depth)],
        "backout_layer": depth // 2 if backout_layer is None else backout_layer,
        "qk_alpha": 1.15,                    # [Math] §QK-Norm with Sharpening
        "softmax_scale": 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale,
        "rope_base": 100000.0,               # [Math] §Frequency Construction
        "eps": 1e-6,                         # [Math] §RMS Normalization, remark
        "softcap": 15.0,                     # [Math] §Logit Softcap
        "gate_channels": 12,                 # [Math] §Value Embeddings
        "ve_gate_scale": 3.0,                # [Math] §Value Embeddings
        "smear": True,                       # [Sweep] Architecture list
    }


def param_counts(depth: int, vocab: int = 32768):
    """Parameter counts in the [Sweep] Models table: (total, matrices + head).

    Matrices per block: W_Q, W_K, W_V, W_O (C x C each) and W_1, W_2 (4C x C):
    12 C^2.  Head: V x C (untied, [Math] §Untied Embeddings).  Embedding
    tables: token embedding V x C plus one value embedding V x C on every
    has_ve layer.  Gates and scalars (a few thousand values) are included in
    the total but are below the table's resolution.
    """
    C, H = model_dims(depth)
    mats = 12 * depth * C * C + vocab * C
    n_ve = sum(1 for l in range(depth) if has_ve(l, depth))
    gates = n_ve * H * 12 + 12 + 2 * depth + 1
    total = mats + vocab * C + n_ve * vocab * C + gates
    return total, mats


# ---------------------------------------------------------------------------
# building blocks
# ---------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """[Math] §RMS Normalization: x / sqrt(mean(x^2) + eps), no gain or bias,
    over the last axis."""
    x = np.asarray(x, F64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(z):
    z = np.asarray(z, F64)
    with np.errstate(over="ignore"):      # exp(-z) -> inf gives exactly 0
        return 1.0 / (1.0 + np.exp(-z))


def rope(u: np.ndarray, positions: np.ndarray, base: float = 100000.0) -> np.ndarray:
    """[Math] §Rotary Position Embeddings.  u has shape [T, D] or [T, n_heads, D],
    one position per row; omega_j = base^(-2j/D),
    phi_{t,j} = t * omega_j, halves u1 = u[:D/2], u2 = u[D/2:],
    RoPE(u) = (u1 cos + u2 sin, -u1 sin + u2 cos)."""
    u = np.asarray(u, F64)
    D = u.shape[-1]
    j = np.arange(D // 2, dtype=F64)
    omega = 1.0 / (base ** (2.0 * j / D))
    phi = np.asarray(positions, F64)[:, None] * omega[None, :]          # [T, D/2]
    if u.ndim == 3:                                                       # [T, H, D]
        phi = phi[:, None, :]
    cos, sin = np.cos(phi), np.sin(phi)
    u1, u2 = u[..., : D // 2], u[..., D // 2:]
    return np.concatenate([u1 * cos + u2 * sin, -u1 * sin + u2 * cos], axis=-1)


def qk_norm(u: np.ndarray, alpha: float = 1.15, eps: float = 1e-6) -> np.ndarray:
    """[Math] §QK-Norm with Sharpening: alpha * RMSNorm over the head dimension."""
    return alpha * rmsnorm(u, eps)


def ve_gate(a12: np.ndarray, w_gate: np.ndarray, scale: float = 3.0) -> np.ndarray:
    """[Math] §Value Embeddings: g = 3 * sigmoid(x[:, :12] W_gate^T), shape [T, H_kv]."""
    return scale * sigmoid(np.asarray(a12, F64) @ np.asarray(w_gate, F64).T)


def relu2(h: np.ndarray) -> np.ndarray:
    """[Math] §Feed-Forward Network: ReLU(h)^2."""
    h = np.asarray(h, F64)
    return np.maximum(h, 0.0) ** 2


def softcap(z: np.ndarray, cap: float = 15.0) -> np.ndarray:
    """[Math] §Logit Softcap: c * tanh(z / c); [Source] §5.4 takes the logits to fp32 first."""
    return cap * np.tanh(np.asarray(z, F64) / cap)


def logsumexp_rows(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, F64)
    m = np.max(z, axis=-1, keepdims=True)
    return (m + np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True)))[..., 0]


def cross_entropy_per_token(zhat: np.ndarray, y: np.ndarray) -> np.ndarray:
    """[Math] §Cross-Entropy Loss: -log softmax(zhat_t)[y_t] for y_t != -1, and 0
    where y_t == -1 (those positions are excluded from the mean)."""
    zhat = np.asarray(zhat, F64)
    y = np.asarray(y)
    valid = y != -1
    yi = np.where(valid, y, 0)
    lse = logsumexp_rows(zhat)
    picked = np.take_along_axis(zhat, yi[..., None].astype(np.int64), axis=-1)[..., 0]
    return np.where(valid, lse - picked, 0.0)


def mean_loss(loss_t: np.ndarray, y: np.ndarray) -> float:
    """Mean over T = {t : y_t != -1}; NaN when T is empty."""
    valid = np.asarray(y) != -1
    n = int(valid.sum())
    return float(np.asarray(loss_t, F64)[valid].sum() / n) if n else float("nan")


def window_mask(T: int, window: int) -> np.ndarray:
    """[Math] §Scaled Dot-Product Attention with Sliding Window: key j is
    visible to query i iff j <= i and i - j < w."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (i - j < window)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, window: int, scale: float) -> np.ndarray:
    """Masked softmax attention, one head at a time, as the dense definition:
    s_ij = scale * q_i . k_j on visible (i, j), -inf elsewhere; a_i = softmax(s_i);
    o_i = sum_j a_ij v_j.  q [T, H, D], k/v [T, H_kv, D]; query head h reads
    key/value head h // (H / H_kv).  Returns [T, H, D]."""
    q, k, v = (np.asarray(t, F64) for t in (q, k, v))
    T, H, D = q.shape
    Hkv = k.shape[1]
    group = H // Hkv
    mask = window_mask(T, window)
    out = np.empty((T, H, D), F64)
    for h in range(H):
        kh, vh = k[:, h // group, :], v[:, h // group, :]
        s = scale * (q[:, h, :] @ kh.T)
        s = np.where(mask, s, -np.inf)
        s = s - np.max(s, axis=1, keepdims=True)
        p = np.exp(s)
        p /= np.sum(p, axis=1, keepdims=True)
        out[:, h, :] = p @ vh
    return out


def attention_at(q, k, v, window: int, scale: float, positions) -> np.ndarray:
    """The same definition evaluated one query position at a time (for sampled
    outputs of long sequences): returns [len(positions), H, D]."""
    q, k, v = (np.asarray(t, F64) for t in (q, k, v))
    T, H, D = q.shape
    group = H // k.shape[1]
    out = np.empty((len(positions), H, D), F64)
    for n, i in enumerate(positions):
        lo = max(0, i - window + 1)
        for h in range(H):
            kh, vh = k[lo:i + 1, h // group, :], v[lo:i + 1, h // group, :]
            s = scale * (kh @ q[i, h, :])
            s = s - s.max()
            p = np.exp(s)
            out[n, h, :] = (p / p.sum()) @ vh
    return out


def attention_layer(q, k, v, window: int, *, alpha: float, scale: float, rope_base: float,
                    eps: float, positions=None) -> np.ndarray:
    """One attention layer from pre-projection q, k, v ([T, H, D]): RoPE, then
    QK-norm with alpha, then windowed attention ([Math] §QK-Norm, §Scaled
    Dot-Product Attention).  With `positions`, only those query rows."""
    T = q.shape[0]
    pos = np.arange(T)
    qh = qk_norm(rope(q, pos, rope_base), alpha, eps)
    kh = qk_norm(rope(k, pos, rope_base), alpha, eps)
    if positions is None:
        return attention(qh, kh, v, window, scale)
    return attention_at(qh, kh, v, window, scale, positions)


# ---------------------------------------------------------------------------
# the whole forward pass
# ---------------------------------------------------------------------------

def embed(cfg: dict, params: dict, tok: np.ndarray) -> np.ndarray:
    """Token embedding, RMSNorm and smear for one row ([Math] §High-Level Forward
    Pass step 1; [Sweep] "smear"; [Source] §5.1).  Returns x (= x0), [T, C]."""
    eps = cfg["eps"]
    xh = rmsnorm(np.asarray(params["wte"], F64)[tok], eps)
    x = xh.copy()
    if cfg.get("smear", True) and len(tok) > 1:
        gc = cfg["gate_channels"]
        s = sigmoid(xh[:, :gc] @ np.asarray(params["smear_gate"], F64))
        x[1:] = xh[1:] + s[1:, None] * xh[:-1]
    return x


def block(cfg: dict, lp: dict, layer: int, x: np.ndarray, tok: np.ndarray, lam: float,
          mu: float, x0: np.ndarray) -> np.ndarray:
    """One transformer block with its x0 re-injection ([Math] §Residual Stream
    with Learnable Scalars; §Causal Self-Attention; §Feed-Forward Network)."""
    eps = cfg["eps"]
    T = x.shape[0]
    H, Hkv, D = cfg["n_head"], cfg["n_kv_head"], cfg["head_dim"]
    x = lam * x + mu * x0
    a = rmsnorm(x, eps)
    qkv = a @ np.asarray(lp["w_qkv"], F64).T
    q = qkv[:, : H * D].reshape(T, H, D)
    k = qkv[:, H * D: (H + Hkv) * D].reshape(T, Hkv, D)
    v = qkv[:, (H + Hkv) * D:].reshape(T, Hkv, D)
    if lp.get("ve") is not None:
        g = ve_gate(a[:, : cfg["gate_channels"]], lp["ve_gate"], cfg["ve_gate_scale"])
        e = np.asarray(lp["ve"], F64)[tok].reshape(T, Hkv, D)
        v = v + g[:, :, None] * e
    o = attention_layer(q, k, v, cfg["windows"][layer], alpha=cfg["qk_alpha"],
                        scale=cfg["softmax_scale"], rope_base=cfg["rope_base"], eps=eps)
    x = x + o.reshape(T, H * D) @ np.asarray(lp["w_o"], F64).T
    h = relu2(rmsnorm(x, eps) @ np.asarray(lp["w_fc1"], F64).T)
    x = x + h @ np.asarray(lp["w_fc2"], F64).T
    return x


def forward(cfg: dict, params: dict, tokens: np.ndarray, targets: np.ndarray | None = None,
            rows=None, want_logits: bool = False, positions=None):
    """Per-token loss (and optionally the softcapped logits) for the given rows.

    tokens/targets are [B, T] int arrays; rows are independent sequences, so
    `rows` selects which ones to evaluate.  `positions` (default: all) limits
    the head to those positions of each row; the blocks still run over the
    whole row.  Returns (loss [R, P], logits [R, P, V] or None).
    """
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    rows = list(range(B)) if rows is None else list(rows)
    L, V = cfg["n_layer"], cfg["vocab"]
    lam = np.asarray(params["resid_lambdas"], F64)
    mu = np.asarray(params["x0_lambdas"], F64)
    beta = float(params["backout_lambda"])
    head = np.asarray(params["lm_head"][:V], F64)
    losses, logits = [], []
    for b in rows:
        tok = tokens[b].astype(np.int64)
        x = embed(cfg, params, tok)
        x0 = x.copy()
        x_bo = None
        for l in range(L):
            x = block(cfg, params["layers"][l], l, x, tok, lam[l], mu[l], x0)
            if l == cfg["backout_layer"]:
                x_bo = x.copy()
        if x_bo is not None:
            x = x - beta * x_bo
        pos = np.arange(T) if positions is None else np.asarray(positions, dtype=np.int64)
        z = rmsnorm(x[pos], cfg["eps"]) @ head.T
        zh = softcap(z, cfg["softcap"])
        if targets is not None:
            losses.append(cross_entropy_per_token(zh, np.asarray(targets)[b][pos]))
        if want_logits:
            logits.append(zh)
    loss = np.stack(losses) if losses else None
    return loss, (np.stack(logits) if want_logits else None)

