"""Seeded synthetic inputs for the nanochat forward pass.

This module only draws random numbers and converts storage formats.  It holds
none of the forward pass's arithmetic, so both the CUDA path and the CPU oracle
can take their inputs from it without sharing any of the method.

The pages train on ClimbMix text with a 32 768-token BPE vocabulary ("nanochat
depth sweep" model card, Training).  That corpus is not available here, so
token ids are drawn uniformly from [0, V): the worst case for gather locality,
and FLOP-neutral.

Weights follow the synthetic recipe: every Linear weight ~ N(0, 1/fan_in),
the token and value-embedding tables ~ N(0, 1), the gate weights ~ N(0, 1/12)
(gate logits ~ N(0, 1) on unit-RMS input), lambda = 1, mu = 0.1, beta = 0.5.

Every tensor has its own PCG64 stream keyed by (seed, tensor id), so a subset
of the tensors (one layer, one row) can be regenerated without drawing the
rest.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os as _os

import numpy as np

SEED_BASE = 20260  # seed of workload i is SEED_BASE + i

# tensor ids for the per-tensor streams
_ID_TOKENS, _ID_TARGETS, _ID_WTE, _ID_HEAD, _ID_SMEAR = 1, 2, 3, 4, 5
_ID_Q, _ID_K, _ID_V = 11, 12, 13
_ID_UNIFORM, _ID_LOGITS = 21, 22
_ID_NEST_X, _ID_NEST_W, _ID_NEST_WU, _ID_NEST_Y = 31, 32, 33, 34
_LAYER_BASE = 1000  # layer l uses ids _LAYER_BASE + 16*l + j


def _gen(seed: int, tid: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(tid)]))


def normal(seed: int, tid: int, shape, std: float) -> np.ndarray:
    """float32 N(0, std^2) array from the stream (seed, tid)."""
    a = _gen(seed, tid).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); the result
    is float32 holding bf16-representable values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # adding 0x7FFF + lsb carries into the upper half exactly when rounding up;
    # no finite value overflows 32 bits (the largest is 0xFF7FFFFF)
    r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) & np.uint32(0xFFFF0000)
    out = r.view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = np.float32("nan")
    return out.reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-exact."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def tokens(seed: int, B: int, T: int, V: int) -> np.ndarray:
    return _gen(seed, _ID_TOKENS).integers(0, V, size=(B, T), dtype=np.int64).astype(np.int32)


def targets(seed: int, B: int, T: int, V: int) -> np.ndarray:
    return _gen(seed, _ID_TARGETS).integers(0, V, size=(B, T), dtype=np.int64).astype(np.int32)


def uniforms(seed: int, B: int) -> np.ndarray:
    """float32 u_b in [0, 1): the random number each row's sampling step draws."""
    u = _gen(seed, _ID_UNIFORM).random(size=B, dtype=np.float32)
    return np.minimum(u, np.float32(0.99999994))


def sampling_logits(seed: int, B: int, V: int, cap: float = 15.0, ties: int = 0) -> np.ndarray:
    """float32 logits in the range of a softcapped head's output: a N(0, 2^2)
    bulk clipped to [-cap, cap], plus 8 entries per row drawn from [6, 8); with
    `ties`, that many entries of each row repeat the row's 5th-largest value."""
    g = _gen(seed, _ID_LOGITS)
    z = np.clip(g.standard_normal(size=(B, V)) * 2.0, -cap, cap).astype(np.float32)
    for b in range(B):
        hot = g.choice(V, size=min(V, 8), replace=False)
        z[b, hot] = (6.0 + 2.0 * g.random(len(hot))).astype(np.float32)
        if ties and V > 5:
            fifth = np.sort(z[b])[::-1][4]
            z[b, g.choice(V, size=min(ties, V), replace=False)] = fifth
    return z


def binade_logits(seed: int, B: int, V: int, lo: float = 1.0) -> np.ndarray:
    """float32 logits uniform in [lo, 2 lo): every entry shares one sign and
    exponent, i.e. one binade."""
    g = _gen(seed, _ID_LOGITS)
    return (lo * (1.0 + g.random(size=(B, V)))).astype(np.float32)


def params(seed: int, *, n_layer: int, n_embd: int, n_head: int, n_kv_head: int,
           head_dim: int, vocab: int, vocab_padded: int, ve_layers, gate_channels: int = 12,
           bf16: bool = True, layers=None) -> dict:
    """Synthetic parameter set.

    Shapes follow the nn.Linear [out, in] convention.  `ve_layers` lists the
    layers that carry a value embedding; `layers` optionally restricts which
    layers are drawn (the others are None).  With bf16=True every matrix and
    table is rounded to bf16 values (still stored as float32); gates and
    scalars stay float32.
    """
    C, Hq, Hkv, D, V = n_embd, n_head, n_kv_head, head_dim, vocab
    ve_layers = set(int(l) for l in ve_layers)
    want = set(range(n_layer)) if layers is None else set(layers)
    # (key, tensor id, shape, std, round to bf16); drawn in parallel threads
    jobs = [("wte", _ID_WTE, (V, C), 1.0, bf16),
            ("lm_head", _ID_HEAD, (vocab_padded, C), C ** -0.5, bf16),
            ("smear_gate", _ID_SMEAR, (gate_channels,), gate_channels ** -0.5, False)]
    nqkv = (Hq + 2 * Hkv) * D
    for l in sorted(want):
        b = _LAYER_BASE + 16 * l
        jobs += [((l, "w_qkv"), b + 0, (nqkv, C), C ** -0.5, bf16),
                 ((l, "w_o"), b + 1, (C, Hq * D), (Hq * D) ** -0.5, bf16),
                 ((l, "w_fc1"), b + 2, (4 * C, C), C ** -0.5, bf16),
                 ((l, "w_fc2"), b + 3, (C, 4 * C), (4 * C) ** -0.5, bf16)]
        if l in ve_layers:
            jobs += [((l, "ve"), b + 4, (V, Hkv * D), 1.0, bf16),
                     ((l, "ve_gate"), b + 5, (Hkv, gate_channels), gate_channels ** -0.5, False)]

    def draw(job):
        key, tid, shape, std, rnd = job
        a = normal(seed, tid, shape, std)
        return key, (round_bf16(a) if rnd else a)

    with _cf.ThreadPoolExecutor(max_workers=min(16, _os.cpu_count() or 4)) as ex:
        drawn = dict(ex.map(draw, jobs))
    p = {
        "wte": drawn["wte"],
        "lm_head": drawn["lm_head"],
        "smear_gate": drawn["smear_gate"],
        "resid_lambdas": np.ones(n_layer, np.float32),
        "x0_lambdas": np.full(n_layer, 0.1, np.float32),
        "backout_lambda": np.float32(0.5),
        "layers": [],
    }
    for l in range(n_layer):
        if l not in want:
            p["layers"].append(None)
            continue
        lp = {k: drawn[(l, k)] for k in ("w_qkv", "w_o", "w_fc1", "w_fc2")}
        lp["ve"] = drawn.get((l, "ve"))
        lp["ve_gate"] = drawn.get((l, "ve_gate"))
        p["layers"].append(lp)
    return p


def attention_inputs(seed: int, B: int, T: int, H: int, D: int, Hkv: int | None = None,
                     bf16: bool = True):
    """q, k, v ~ N(0, 1) shaped (B, T, H, D) / (B, T, Hkv, D)."""
    Hkv = H if Hkv is None else Hkv
    rnd = round_bf16 if bf16 else (lambda a: a)
    q = rnd(normal(seed, _ID_Q, (B, T, H, D), 1.0))
    k = rnd(normal(seed, _ID_K, (B, T, Hkv, D), 1.0))
    v = rnd(normal(seed, _ID_V, (B, T, Hkv, D), 1.0))
    return q, k, v


def nested_inputs(seed: int, M: int, C_in: int, C_out: int, V: int, V_pad: int):
    """Inputs of the nesting pieces: a residual x [M, C_in] ~ N(0, 1) (fp32),
    a dense weight W [C_out, C_in] ~ N(0, 1/C_in) and a head W_U [V_pad, C_in]
    ~ N(0, 1/C_in) (both bf16 values held as float32), targets [M] uniform in
    [0, V).  Zeroing the weight's dead blocks is left to the caller."""
    x = normal(seed, _ID_NEST_X, (M, C_in), 1.0)
    w = round_bf16(normal(seed, _ID_NEST_W, (C_out, C_in), C_in ** -0.5))
    w_u = round_bf16(normal(seed, _ID_NEST_WU, (V_pad, C_in), C_in ** -0.5))
    y = _gen(seed, _ID_NEST_Y).integers(0, V, size=M, dtype=np.int64).astype(np.int32)
    return x, w, w_u, y


# Workload shapes (model depth, batch, sequence length, short window, dtype).
# Workload i draws its inputs from seed SEED_BASE + i.
WORKLOADS = {
    "d1": dict(index=0, depth=1, B=1, T=256, short=256, dtype="fp32"),
    "d4": dict(index=1, depth=4, B=4, T=1024, short=512, dtype="bf16"),
    "d12": dict(index=2, depth=12, B=8, T=2048, short=1024, dtype="bf16"),
    "d24": dict(index=3, depth=24, B=4, T=2048, short=1024, dtype="bf16"),
}
# single attention layer sweep: 12 heads x 128, batch 8, T x window
ATTN_SWEEP = dict(index=4, H=12, D=128, B=8, cases=[(2048, 1024), (2048, 0), (8192, 1024), (8192, 0)])
