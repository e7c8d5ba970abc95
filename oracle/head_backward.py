"""Plain fp64 CPU definition of the backward pass of the model's head: the
gradient of the mean cross-entropy with respect to the final residual stream
and to the unembedding matrix.

TEST INFRASTRUCTURE.  Part of the oracle the CUDA path is checked against;
only the test suite, the smoke check and the benchmark's CPU legs may import
it, and nothing here is shared with the CUDA kernels.

Written from "The Mathematics of Karpathy's nanochat":
  * §RMS Normalization: xn = x / sqrt(mean(x^2) + eps) (no learned weight);
  * the head: z = xn W_U^T, then §Logit Softcap zhat = c tanh(z / c), whose
    derivative the section states as d zhat / d z = 1 - tanh^2(z / c);
  * §Cross-Entropy Loss: L = (1 / |T|) sum over valid t of
    (logsumexp(zhat_t) - zhat_t[y_t]), targets y_t = -1 ignored.
Each gradient is the chain rule through these steps, in the order of the
forward pass reversed; library matmul and exp serve as steps.  The forward
part is restated here (not imported) so that this module reads on its own.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def head_forward(x: np.ndarray, w_u: np.ndarray, targets: np.ndarray, *, cap: float = 15.0,
                 eps: float = 1e-6) -> float:
    """The mean loss L of the rows x [M, C] (final residual, before the norm)."""
    x = np.asarray(x, F64)
    w = np.asarray(w_u, F64)
    y = np.asarray(targets)
    xn = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    zh = cap * np.tanh((xn @ w.T) / cap)
    m = zh.max(axis=-1, keepdims=True)
    lse = (m + np.log(np.sum(np.exp(zh - m), axis=-1, keepdims=True)))[:, 0]
    valid = y >= 0
    n = int(valid.sum())
    if n == 0:
        return float("nan")
    picked = zh[np.arange(len(y)), np.where(valid, y, 0)]
    return float(np.sum((lse - picked)[valid]) / n)


def head_backward(x: np.ndarray, w_u: np.ndarray, targets: np.ndarray, *, cap: float = 15.0,
                  eps: float = 1e-6):
    """(dL/dx [M, C], dL/dW_U [V, C], L) for the rows x [M, C] (final residual,
    before the norm), W_U [V, C] and targets [M] (-1 = ignored)."""
    x = np.asarray(x, F64)
    w = np.asarray(w_u, F64)
    y = np.asarray(targets)
    M, C = x.shape
    # forward, keeping what the backward uses
    ms = np.mean(x * x, axis=-1, keepdims=True) + eps
    r = 1.0 / np.sqrt(ms)                     # 1 / rms, per row
    xn = x * r
    z = xn @ w.T
    th = np.tanh(z / cap)
    zh = cap * th
    m = zh.max(axis=-1, keepdims=True)
    e = np.exp(zh - m)
    p = e / e.sum(axis=-1, keepdims=True)     # softmax(zhat), per row
    valid = y >= 0
    n = int(valid.sum())
    if n == 0:
        return np.zeros_like(x), np.zeros_like(w), float("nan")
    lse = (m + np.log(e.sum(axis=-1, keepdims=True)))[:, 0]
    loss = float(np.sum((lse - zh[np.arange(M), np.where(valid, y, 0)])[valid]) / n)
    # dL/dzhat: (softmax - one-hot(y)) / |T| on valid rows, 0 on ignored ones
    dzh = p.copy()
    dzh[np.arange(M)[valid], y[valid]] -= 1.0
    dzh[~valid] = 0.0
    dzh /= n
    # through the softcap: d zhat / d z = 1 - tanh^2(z / c)
    dz = dzh * (1.0 - th * th)
    # through the head: z = xn W_U^T
    dxn = dz @ w
    dw = dz.T @ xn
    # through the norm: xn = x r with r = (mean(x^2) + eps)^(-1/2), so
    # dr/dx = -r^3 x / C and dL/dx = r dxn - x r^3 (x . dxn) / C
    dx = r * dxn - x * (r ** 3) * np.sum(x * dxn, axis=-1, keepdims=True) / C
    return dx, dw, loss
