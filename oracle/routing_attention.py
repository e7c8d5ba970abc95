"""Plain fp64 CPU definition of the pass-2 attention layer of the looped
(routing) nanochat variant.

TEST INFRASTRUCTURE.  Part of the oracle the CUDA path is checked against;
only the test suite, the smoke check and the benchmark's CPU legs may import
it, and nothing here is shared with the CUDA kernels.

Written from the "looped nanochat" model card (What is the routing loop?):
pass 2 re-runs the trunk, and each pass-2 layer adds a causal attention-logit
prior from one pass-1 layer,
    logits_ij = q2_i . k2_j / sqrt(D) + g q1_i . k1_j / sqrt(D),
    g = softplus(gate_logit)  (one learned gate per layer),
where q1, k1 are the normalised, RoPE-applied features captured in pass 1 and
q2, k2 those of pass 2; then the ordinary causal (windowed) softmax and the
sum over v2.  The card notes that the prior is computed through
augmented-width Q/K with ordinary attention, never as a T x T matrix; that
identity is a pin of this module, not its method.
Readings: the visibility rule is the base model's (key j visible to query i
iff j <= i and i - j < w); the 1/sqrt(D) scale applies to both terms as
printed, with D the head dimension of either pass.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def softplus(a: float) -> float:
    """log(1 + e^a), evaluated without overflow."""
    a = float(a)
    return a + np.log1p(np.exp(-a)) if a > 0 else float(np.log1p(np.exp(a)))


def routing_attention(q2, k2, v2, q1, k1, gate_logit: float, window: int, scale: float | None = None):
    """Pass-2 attention of one layer: q2, q1 [T, H, D]; k2, k1, v2 [T, H_kv, D]
    (query head h reads key/value head h // (H / H_kv)).  Returns [T, H, D]."""
    q2, k2, v2, q1, k1 = (np.asarray(t, F64) for t in (q2, k2, v2, q1, k1))
    T, H, D = q2.shape
    Hkv = k2.shape[1]
    group = H // Hkv
    sc = D ** -0.5 if scale is None else scale
    g = softplus(gate_logit)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    visible = (j <= i) & (i - j < window)
    out = np.empty((T, H, v2.shape[2]), F64)
    for h in range(H):
        kv = h // group
        s = sc * (q2[:, h] @ k2[:, kv].T) + g * sc * (q1[:, h] @ k1[:, kv].T)
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h] = p @ v2[:, kv]
    return out
