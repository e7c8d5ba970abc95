"""Plain fp64 CPU definitions of the nesting pieces of StairFormer ("Fully
Nested Transformers" README): block lower triangular linear maps,
PrefixRMSNorm, and the prefix cross-entropy of the k-front submodels.

TEST INFRASTRUCTURE.  Part of the oracle; only the test suite may import it,
and nothing here is shared with the CUDA kernels.  There is no kernel for
these pieces yet: the README summarises the method and these are the parts it
fixes.

What the README fixes, and the readings taken where it is silent:
  * The residual stream of width C is cut into k nested blocks at head
    boundaries (its d24 run: 6 + 18 heads of 64, widths 384 + 1152).  The
    j-front submodel is the first j blocks, width C_j = sum of the first j
    widths; the smaller model is "the top-left corner of the network".
  * Block lower triangular weights: output block a of a linear map reads only
    input blocks b <= a, so the first C_j outputs depend only on the first C_j
    inputs ("the residual stream of smaller models is a prefix of larger
    models'").  Only the live (b <= a) blocks are weights.
  * PrefixRMSNorm "keeps normalization from leaking information backward down
    the hierarchy".  Reading: block a of the output is block a of the input
    divided by the RMS of the input prefix up to the end of block a,
    y_a = x_a / sqrt(mean(x[:C_a]^2) + eps); with one block it is RMSNorm.
    (Dividing by the block's own RMS would also preserve the filtration; the
    name says prefix.)
  * Every layer is then filtration-preserving: output prefixes depend only on
    input prefixes of the same width.
  * Prefix cross-entropy: every submodel has a loss.  Reading: submodel j's
    logits use the first C_j columns of the (untied) head on its normalised
    prefix, z_j = PrefixRMSNorm(x)[:, :C_j] W_U[:, :C_j]^T, then the base
    model's softcap and cross-entropy.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def block_bounds(widths):
    """Cumulative block ends [C_1, C_1 + C_2, ...] of the given block widths."""
    return list(np.cumsum(np.asarray(widths, dtype=np.int64)).tolist())


def head_blocks(head_counts, head_dim: int):
    """Block widths from heads per block (the README's --nested-block-head-counts)."""
    return [int(h) * head_dim for h in head_counts]


def block_lower_triangular_mask(out_widths, in_widths) -> np.ndarray:
    """[sum(out_widths), sum(in_widths)] boolean: True where output block a may
    read input block b, i.e. b <= a (the live blocks)."""
    assert len(out_widths) == len(in_widths)
    oe, ie = block_bounds(out_widths), block_bounds(in_widths)
    m = np.zeros((oe[-1], ie[-1]), dtype=bool)
    for a in range(len(out_widths)):
        o0 = oe[a] - out_widths[a]
        m[o0:oe[a], :ie[a]] = True
    return m


def btl_linear(x: np.ndarray, w: np.ndarray, out_widths, in_widths) -> np.ndarray:
    """y = x W^T with W [out, in] restricted to its live blocks."""
    mask = block_lower_triangular_mask(out_widths, in_widths)
    return np.asarray(x, F64) @ np.where(mask, np.asarray(w, F64), 0.0).T


def prefix_rmsnorm(x: np.ndarray, widths, eps: float = 1e-6) -> np.ndarray:
    """Block a of the output: x_a / sqrt(mean(x[..., :C_a]^2) + eps)."""
    x = np.asarray(x, F64)
    ends = block_bounds(widths)
    y = np.empty_like(x)
    for a, e in enumerate(ends):
        s = e - widths[a]
        r = np.sqrt(np.mean(x[..., :e] ** 2, axis=-1, keepdims=True) + eps)
        y[..., s:e] = x[..., s:e] / r
    return y


def prefix_logits(x: np.ndarray, w_u: np.ndarray, widths, j: int, *, cap: float = 15.0,
                  eps: float = 1e-6) -> np.ndarray:
    """Softcapped logits of the j-front submodel (j = 1..k) from the full
    residual x [M, C]: its normalised prefix times the head's first C_j columns."""
    cj = block_bounds(widths)[j - 1]
    xn = prefix_rmsnorm(x, widths, eps)[:, :cj]
    z = xn @ np.asarray(w_u, F64)[:, :cj].T
    return cap * np.tanh(z / cap)


def prefix_ce(x: np.ndarray, w_u: np.ndarray, targets: np.ndarray, widths, *, cap: float = 15.0,
              eps: float = 1e-6):
    """Per-token cross-entropy of every j-front submodel: list over j = 1..k of
    [M] arrays (0 where the target is -1)."""
    y = np.asarray(targets)
    valid = y != -1
    yi = np.where(valid, y, 0)
    out = []
    for j in range(1, len(widths) + 1):
        zh = prefix_logits(x, w_u, widths, j, cap=cap, eps=eps)
        m = zh.max(axis=-1, keepdims=True)
        lse = (m + np.log(np.sum(np.exp(zh - m), axis=-1, keepdims=True)))[:, 0]
        out.append(np.where(valid, lse - zh[np.arange(len(y)), yi], 0.0))
    return out
