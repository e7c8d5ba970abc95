"""Algorithmic FLOP accounting of the forward pass (for throughput reporting).

A GEMM of [M, K] x [K, N] counts 2 M N K.  Per token the matrix parameters
cost 2 FLOPs each: 12 L C^2 for the blocks (W_Q, W_K, W_V, W_O: C x C each;
W_1, W_2: 4C x C) plus V C for the untied head.  Attention costs 4 C per
visible key per layer (q.k and p.v, 2 FLOPs per multiply-add, H D = C), and
query i sees min(i + 1, w) keys.  The forward third of the training formula
in "The Mathematics of Karpathy's nanochat" (§FLOPs Estimation) uses
min(w, T) keys for every query instead; the StairFormer README's FLOPs/token
table uses T for every query.  Both conventions are provided.
"""
from __future__ import annotations


def gemm_flops_per_token(n_layer: int, n_embd: int, vocab: int) -> float:
    return 2.0 * (12 * n_layer * n_embd * n_embd + vocab * n_embd)


def mean_visible_keys(T: int, w: int) -> float:
    """(1/T) sum_{i<T} min(i + 1, w)."""
    w = min(w, T)
    # sum_{i=0}^{w-1} (i + 1) + (T - w) w
    return (w * (w + 1) / 2 + (T - w) * w) / T


def attention_flops_per_token(n_embd: int, windows, T: int) -> float:
    return sum(4.0 * n_embd * mean_visible_keys(T, w) for w in windows)


def forward_flops_per_token(n_layer: int, n_embd: int, vocab: int, windows, T: int) -> float:
    """Algorithmic forward FLOPs per token (masked attention work excluded)."""
    return gemm_flops_per_token(n_layer, n_embd, vocab) + attention_flops_per_token(n_embd, windows, T)


def nominal_window_flops_per_token(n_layer: int, n_embd: int, vocab: int, windows, T: int) -> float:
    """Forward third of the training estimate: 2 N_mat + sum_l 4 C min(w_l, T)."""
    return gemm_flops_per_token(n_layer, n_embd, vocab) + sum(4.0 * n_embd * min(w, T) for w in windows)


def dense_table_flops_per_token(n_layer: int, n_embd: int, vocab: int, T: int) -> float:
    """Convention of the StairFormer README's FLOPs/token table: 2 N_mat + 4 L C T."""
    return gemm_flops_per_token(n_layer, n_embd, vocab) + 4.0 * n_layer * n_embd * T


def attention_layer_flops(B: int, T: int, H: int, D: int, window: int) -> float:
    """One attention layer (QK^T and PV over the visible keys), whole batch."""
    w = T if window <= 0 or window >= T else window
    return 4.0 * B * T * H * D * mean_visible_keys(T, w)
