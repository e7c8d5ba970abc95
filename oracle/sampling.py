"""Plain fp64 CPU definition of one generation step's sampling: top-k
filtering, temperature, and one draw from the resulting distribution.

TEST INFRASTRUCTURE.  Part of the oracle the CUDA path is checked against;
only the test suite, the smoke check and the benchmark's CPU legs may import
it, and nothing here is shared with the CUDA kernels.

Written from "The Mathematics of Karpathy's nanochat", §Inference: Generating
Text (the logits of the last position only) and §Sampling Controls:
  * top-k: z_v is kept if v is among the k largest, else set to -inf; the
    page's code keeps every z_v that is not below the k-th largest value
    (counted with multiplicity), so ties at that value are all kept;
  * temperature tau > 0: P(v) = exp(z_v / tau) / sum_v' exp(z_v' / tau);
  * tau = 0: greedy decoding, the most likely token; among equal maxima the
    lowest index (argmax convention).
Reading where the page is silent: the draw from P is realised by inversion of
a caller-supplied uniform u in [0, 1): the index is the first v, in
vocabulary order, whose cumulative probability exceeds u.  For u uniform on
[0, 1) this picks v with probability P(v) exactly.
The page's worked example (five logits at tau = 0.8) lists probabilities that
follow exp(0.8 z) rather than exp(z / 0.8); the formula and the code on the
same page divide by tau, and so does this module.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def top_k_filter(z: np.ndarray, k: int | None) -> np.ndarray:
    """z with every entry below the k-th largest value set to -inf.  k None, 0
    or >= len(z) leaves z unchanged ([Math] §Sampling Controls, top-k)."""
    z = np.asarray(z, F64).copy()
    if not k or k >= z.shape[-1]:
        return z
    kth = np.sort(z)[::-1][k - 1]          # the k-th largest, ties counted
    z[z < kth] = -np.inf
    return z


def probabilities(z: np.ndarray, temperature: float, top_k: int | None = None) -> np.ndarray:
    """P(v) = exp(z_v / tau) / sum exp(z_v' / tau) over the kept entries."""
    zf = top_k_filter(z, top_k)
    a = zf / temperature
    a = a - np.max(a)                      # exact rescaling of numerator and denominator
    w = np.exp(a)
    return w / np.sum(w)


def greedy(z: np.ndarray) -> int:
    """The lowest index among the maxima of z (tau = 0)."""
    z = np.asarray(z, F64)
    best = 0
    for v in range(1, z.shape[-1]):
        if z[v] > z[best]:
            best = v
    return best


def sample_next(z: np.ndarray, temperature: float, top_k: int | None, u: float) -> int:
    """One token from the logits z [V]: greedy when temperature == 0, else the
    first v whose cumulative probability exceeds u."""
    if temperature == 0:
        return greedy(z)
    p = probabilities(z, temperature, top_k)
    c = np.cumsum(p)
    idx = int(np.searchsorted(c, u * c[-1], side="right"))
    return min(idx, int(np.nonzero(p > 0)[0][-1]))


def draw_interval(z: np.ndarray, temperature: float, top_k: int | None, v: int):
    """The sub-interval [lo, hi) of [0, 1) of the u values that draw token v."""
    p = probabilities(z, temperature, top_k)
    c = np.cumsum(p) / np.sum(p)
    lo = 0.0 if v == 0 else float(c[v - 1])
    return lo, float(c[v])
