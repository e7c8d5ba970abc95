"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a worked
example printed on the pages (fixtures under tests/golden/), a closed form,
an invariant, a library routine, or brute force on tiny inputs.  The set is
chosen so that a dropped term, a wrong sign or index, or a transposed operand
in any oracle step fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

from golden_io import load
from oracle import nanochat_fwd as O
from decoder_only_transformer_fwd_b200 import synth

F64 = np.float64


# --------------------------------------------------------------------------
# worked examples
# --------------------------------------------------------------------------

def test_rmsnorm_worked_example():
    g = load("rmsnorm_example.txt")
    x = np.array(g["input"], F64)
    y = O.rmsnorm(x)
    assert np.allclose(y, g["output"], atol=g["tol"])
    assert abs(np.sqrt(np.mean(x * x)) - g["rms"]) < 1e-4


def test_rope_worked_example():
    g = load("rope_example.txt")
    u = np.array([g["input"]], F64)
    y = O.rope(u, np.array([g["position"]]), base=g["base"])[0]
    assert np.allclose(y, g["output"], atol=g["tol"])


def test_qknorm_worked_example():
    g = load("qknorm_example.txt")
    y = O.qk_norm(np.array(g["input"], F64), alpha=g["alpha"])
    assert np.allclose(y, g["output"], atol=g["tol"])


def test_ve_gate_worked_example():
    g = load("ve_gate_example.txt")
    # a 12-channel input whose dot with a one-hot gate row is the printed logit
    a12 = np.zeros((1, 12)); a12[0, 0] = g["logit"]
    w = np.zeros((1, 12)); w[0, 0] = 1.0
    gate = O.ve_gate(a12, w)[0, 0]
    assert abs(gate - g["gate"]) < g["tol"]
    v_new = np.array(g["v"]) + gate * np.array(g["ve"])
    assert np.allclose(v_new, g["v_new"], atol=g["tol"])


def test_relu2_worked_example():
    g = load("relu2_example.txt")
    assert np.allclose(O.relu2(np.array(g["input"])), g["output"], atol=g["tol"])


def test_softcap_worked_example():
    g = load("softcap_example.txt")
    for z, printed, tol in g["rows"]:
        assert abs(O.softcap(z, g["cap"]) - printed) < tol, (z, printed)


def test_softcap_bounds_and_linear_regime():
    z = np.linspace(-1e4, 1e4, 20001)
    zh = O.softcap(z)
    assert np.all(np.abs(zh) <= 15.0)
    small = np.linspace(-0.1, 0.1, 101)
    # tanh(u) = u - u^3/3 + ...: |c tanh(z/c) - z| <= |z|^3 / (3 c^2)
    assert np.all(np.abs(O.softcap(small) - small) <= np.abs(small) ** 3 / (3 * 225.0) + 1e-15)


def test_e2e_trace_embedding_rows():
    g = load("e2e_trace_example.txt")
    for r in (1, 2):
        y = O.rmsnorm(np.array(g[f"embed_row{r}"]))
        assert np.allclose(y, g[f"norm_row{r}"], atol=g["tol"])


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------

def test_rmsnorm_unit_rms():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 1536)) * rng.uniform(0.01, 100, (64, 1))
    y = O.rmsnorm(x)
    rms = np.sqrt(np.mean(y * y, axis=-1))
    # eps = 1e-6 perturbs the unit RMS by at most eps / (2 mean x^2)
    ms = np.mean(x * x, axis=-1)
    assert np.all(np.abs(rms - 1.0) <= 1e-6 / ms + 1e-12)


def test_rope_preserves_norm_and_is_relative():
    rng = np.random.default_rng(1)
    D = 128
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)
    for m, n in [(0, 0), (5, 3), (100, 7), (4000, 3990), (8191, 1)]:
        rq = O.rope(q[None], np.array([m]))[0]
        rk = O.rope(k[None], np.array([n]))[0]
        assert abs(np.linalg.norm(rq) - np.linalg.norm(q)) < 1e-9
        # the proposition: <RoPE(q, m), RoPE(k, n)> depends only on m - n
        rq0 = O.rope(q[None], np.array([m - n]))[0]
        assert abs(rq @ rk - rq0 @ k) < 1e-9 * (1 + abs(rq @ rk))
    # and explicitly against the printed closed form
    m, n = 37, 11
    omega = 1.0 / 100000.0 ** (2 * np.arange(D // 2) / D)
    phi = (m - n) * omega
    q1, q2, k1, k2 = q[:64], q[64:], k[:64], k[64:]
    closed = np.sum((q1 * k1 + q2 * k2) * np.cos(phi) + (q2 * k1 - q1 * k2) * np.sin(phi))
    got = O.rope(q[None], np.array([m]))[0] @ O.rope(k[None], np.array([n]))[0]
    assert abs(got - closed) < 1e-9


def test_rope_commutes_with_head_norm():
    # RoPE rotates each (j, j + D/2) pair, so it preserves the mean square and
    # norm(RoPE(u)) == RoPE(norm(u)).
    rng = np.random.default_rng(2)
    u = rng.standard_normal((9, 3, 128))
    pos = np.arange(9) * 13
    assert np.allclose(O.rmsnorm(O.rope(u, pos)), O.rope(O.rmsnorm(u), pos), atol=1e-12)


def test_cross_entropy_closed_forms():
    V = load("e2e_trace_example.txt")["vocab"]
    y = np.array([[0, 5, V - 1]])
    zero = np.zeros((1, 3, V))
    loss = O.cross_entropy_per_token(zero, y)
    assert np.allclose(loss, math.log(V), atol=1e-12)
    g = load("e2e_trace_example.txt")
    assert abs(math.log(V) - g["init_loss"]) < g["init_tol"]
    # one large logit at the target, capped at 15: log(e^15 + V - 1) - 15
    z = np.zeros((1, 1, V)); z[0, 0, 7] = 1e6
    zh = O.softcap(z)
    l = O.cross_entropy_per_token(zh, np.array([[7]]))[0, 0]
    assert abs(l - (math.log(math.exp(15.0) + V - 1) - 15.0)) < 1e-12
    # ignore index
    l = O.cross_entropy_per_token(zh, np.array([[-1]]))
    assert l[0, 0] == 0.0
    assert math.isnan(O.mean_loss(l, np.array([[-1]])))


def test_cross_entropy_matches_torch():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((2, 7, 1000)) * 5
    y = rng.integers(0, 1000, (2, 7)); y[0, 3] = -1
    zh = O.softcap(z)
    ours = O.cross_entropy_per_token(zh, y)
    ref = torch.nn.functional.cross_entropy(torch.from_numpy(zh).reshape(-1, 1000),
                                            torch.from_numpy(y).reshape(-1), ignore_index=-1,
                                            reduction="none").numpy().reshape(2, 7)
    assert np.allclose(ours, ref, atol=1e-12)
    assert abs(O.mean_loss(ours, y) - ref[y != -1].mean()) < 1e-12


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _sdpa_ref(q, k, v, window, scale):
    """torch SDPA in fp64 with an explicit boolean mask built from the
    definition of visibility: j <= i and i - j < w."""
    T = q.shape[0]
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & (i - j < window)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("T,window", [(1, 1), (7, 1), (33, 4), (33, 33), (40, 100), (64, 17)])
def test_attention_matches_sdpa(T, window):
    rng = np.random.default_rng(T * 101 + window)
    q, k, v = (rng.standard_normal((T, 3, 16)) for _ in range(3))
    ours = O.attention(q, k, v, window, 0.25)
    assert np.allclose(ours, _sdpa_ref(q, k, v, window, 0.25), atol=1e-12)
    # the per-position form agrees with the dense form
    pos = sorted(set([0, T // 2, T - 1]))
    assert np.allclose(O.attention_at(q, k, v, window, 0.25, pos), ours[pos], atol=1e-12)


def test_attention_full_window_is_causal_sdpa():
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((20, 2, 8)) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(t).permute(1, 0, 2)[None] for t in (q, k, v)), is_causal=True)
    ours = O.attention(q, k, v, 10 ** 6, 1 / math.sqrt(8))
    assert np.allclose(ours, ref[0].permute(1, 0, 2).numpy(), atol=1e-12)


def test_attention_single_position_returns_v():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((1, 2, 8)) for _ in range(3))
    assert np.allclose(O.attention(q, k, v, 1, 1.0), v, atol=0)


def test_attention_gqa_matches_repeated_heads():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((12, 4, 8))
    k, v = (rng.standard_normal((12, 2, 8)) for _ in range(2))
    rep = lambda t: np.repeat(t, 2, axis=1)
    assert np.allclose(O.attention(q, k, v, 5, 0.3), O.attention(q, rep(k), rep(v), 5, 0.3))


@pytest.mark.parametrize("window", [1, 3, 8, 32])
def test_attention_window_brute_force(window):
    """Changing k_j / v_j for j > t or j <= t - w leaves o_t bit-identical;
    changing a key inside the window changes it."""
    T = 32
    rng = np.random.default_rng(window)
    q, k, v = (rng.standard_normal((T, 1, 8)) for _ in range(3))
    base = O.attention(q, k, v, window, 0.5)
    for t in range(T):
        for j in range(T):
            k2, v2 = k.copy(), v.copy()
            k2[j] += 1.0; v2[j] -= 1.0
            o = O.attention(q, k2, v2, window, 0.5)[t]
            visible = (j <= t) and (t - j < window)
            if visible:
                assert not np.array_equal(o, base[t]), (t, j)
            else:
                assert np.array_equal(o, base[t]), (t, j)


# --------------------------------------------------------------------------
# model shape and parameter accounting
# --------------------------------------------------------------------------

def test_param_counts_match_depth_sweep_table():
    g = load("param_counts.txt")
    for depth, width, heads, total_m, mats_m in g["rows"]:
        C, H = O.model_dims(depth)
        assert (C, H) == (width, heads)
        total, mats = O.param_counts(depth)
        assert abs(total / 1e6 - total_m) < 0.05 + 1e-9, depth
        assert abs(mats / 1e6 - mats_m) < 0.05 + 1e-9, depth


def test_layer_rules():
    # [Math] window example: T = 2048, pattern SSSL, last layer long
    assert O.layer_windows(24, 2048, 1024)[:8] == [1024, 1024, 1024, 2048] * 2
    assert O.layer_windows(4, 1024, 512) == [512, 512, 512, 1024]
    assert O.layer_windows(6, 2048, 768)[-1] == 2048 and O.layer_windows(6, 2048, 768)[-2] == 768
    assert [l for l in range(24) if O.has_ve(l, 24)] == list(range(1, 24, 2))
    assert [l for l in range(1) if O.has_ve(l, 1)] == [0]
    assert O.has_ve(3, 4) and not O.has_ve(2, 4)
    assert O.padded_vocab(32768) == 32768 and O.padded_vocab(50257) == 50304


# --------------------------------------------------------------------------
# whole-model pins
# --------------------------------------------------------------------------

def _tiny_cfg(depth=2, T=16, short=8, **kw):
    cfg = O.make_config(depth, T, short, vocab=kw.pop("vocab", 300), **kw)
    return cfg


def _tiny_params(cfg, seed=7, bf16=False):
    return synth.params(seed, n_layer=cfg["n_layer"], n_embd=cfg["n_embd"], n_head=cfg["n_head"],
                        n_kv_head=cfg["n_kv_head"], head_dim=cfg["head_dim"], vocab=cfg["vocab"],
                        vocab_padded=cfg["vocab_padded"], ve_layers=cfg["ve_layers"], bf16=bf16)


def _identity_blocks(p):
    for lp in p["layers"]:
        lp["w_o"][:] = 0
        lp["w_fc2"][:] = 0


def _textbook_head_loss(x, head, y):
    """softcap(x W^T) then torch cross_entropy, for x already normalised."""
    z = torch.from_numpy(x @ head.T)
    zh = 15.0 * torch.tanh(z / 15.0)
    return torch.nn.functional.cross_entropy(zh, torch.from_numpy(y).long(),
                                             reduction="none", ignore_index=-1).numpy()


def test_identity_blocks_reduce_to_textbook_head():
    """W_O = W_2 = 0 makes every block the identity ([Math] §Weight
    Initialization); with per-layer (lambda, mu) the residual is c * x0 with
    c_l = lambda_l c_{l-1} + mu_l, and backout subtracts beta c_bo x0.  So the
    loss is a single textbook GEMM + softcap + CE on c x0 / sqrt(c^2 ms(x0) + eps),
    ms the mean square, eps = 1e-6."""
    cfg = _tiny_cfg(depth=4, T=12, short=4)
    p = _tiny_params(cfg)
    _identity_blocks(p)
    rng = np.random.default_rng(11)
    lam = rng.uniform(0.5, 1.5, 4); mu = rng.uniform(-0.3, 0.3, 4)
    for beta in (0.0, 0.5, 3.0):      # 3.0 makes the final coefficient negative
        p["resid_lambdas"] = lam; p["x0_lambdas"] = mu; p["backout_lambda"] = beta
        tok = rng.integers(0, cfg["vocab"], (2, 12)); y = rng.integers(0, cfg["vocab"], (2, 12))
        y[1, 5] = -1
        loss, _ = O.forward(cfg, p, tok, y)
        c = 1.0; c_bo = None
        for l in range(4):
            c = lam[l] * c + mu[l]
            if l == cfg["backout_layer"]:
                c_bo = c
        c_final = c - beta * c_bo
        head = np.asarray(p["lm_head"][: cfg["vocab"]], F64)
        for b in range(2):
            x0 = O.embed(cfg, p, tok[b])
            ms = np.mean(x0 * x0, axis=-1, keepdims=True)
            xf = c_final * x0 / np.sqrt(c_final ** 2 * ms + 1e-6)
            ref = _textbook_head_loss(xf, head, y[b])
            assert np.allclose(loss[b], ref, atol=1e-10)


def _one_layer_cfg(C=128, window=4, T=10):
    cfg = O.make_config(1, T, window, vocab=50)
    cfg["windows"] = [window]
    assert cfg["n_embd"] == C
    return cfg


def test_uniform_attention_block_is_windowed_moving_average():
    """With W_Q = W_K = 0 the scores are equal, so each query averages v over
    its window; with W_O = I the block adds that average to the residual.
    With W_2 = 0 the MLP vanishes.  The expected residual is built with a
    cumulative sum (a different route from the oracle's masked softmax)."""
    T, w = 10, 4
    cfg = _one_layer_cfg(window=w, T=T)
    p = _tiny_params(cfg)
    lp = p["layers"][0]
    C = cfg["n_embd"]
    lp["w_qkv"][: 2 * C] = 0            # q = k = 0
    lp["w_o"][:] = np.eye(C)
    lp["w_fc2"][:] = 0
    p["backout_lambda"] = 0.0
    rng = np.random.default_rng(12)
    tok = rng.integers(0, 50, (1, T)); y = rng.integers(0, 50, (1, T))
    loss, _ = O.forward(cfg, p, tok, y)
    x0 = O.embed(cfg, p, tok[0])
    x = p["resid_lambdas"][0] * x0 + p["x0_lambdas"][0] * x0
    a = O.rmsnorm(x)
    v = a @ np.asarray(lp["w_qkv"][2 * C:], F64).T
    g = 3.0 / (1.0 + np.exp(-(a[:, :12] @ np.asarray(lp["ve_gate"], F64).T)))   # [T, 1]
    v = v + g * np.asarray(lp["ve"], F64)[tok[0]]
    cs = np.vstack([np.zeros((1, C)), np.cumsum(v, axis=0)])
    avg = np.stack([(cs[t + 1] - cs[max(0, t - w + 1)]) / (t + 1 - max(0, t - w + 1)) for t in range(T)])
    ref = _textbook_head_loss(O.rmsnorm(x + avg), np.asarray(p["lm_head"][:50], F64), y[0])
    assert np.allclose(loss[0], ref, atol=1e-10)


def test_mlp_wiring_signed_square():
    """W_1 = [I; -I; 0], W_2 = [I, -I, 0] makes the MLP relu(a)^2 - relu(-a)^2
    = a |a| with a = RMSNorm(x); with W_O = 0 the block is x + a|a|."""
    cfg = _one_layer_cfg()
    p = _tiny_params(cfg)
    lp = p["layers"][0]
    C = cfg["n_embd"]
    lp["w_o"][:] = 0
    w1 = np.zeros((4 * C, C)); w1[:C] = np.eye(C); w1[C:2 * C] = -np.eye(C)
    w2 = np.zeros((C, 4 * C)); w2[:, :C] = np.eye(C); w2[:, C:2 * C] = -np.eye(C)
    lp["w_fc1"] = w1; lp["w_fc2"] = w2
    p["backout_lambda"] = 0.0
    rng = np.random.default_rng(13)
    tok = rng.integers(0, 50, (1, 10)); y = rng.integers(0, 50, (1, 10))
    loss, _ = O.forward(cfg, p, tok, y)
    x0 = O.embed(cfg, p, tok[0])
    x = 1.1 * x0
    a = O.rmsnorm(x)
    ref = _textbook_head_loss(O.rmsnorm(x + a * np.abs(a)), np.asarray(p["lm_head"][:50], F64), y[0])
    assert np.allclose(loss[0], ref, atol=1e-10)


def test_smear_reductions():
    """A very negative smear gate removes smear; position 0 never sees it."""
    cfg = _tiny_cfg(depth=2, T=10, short=4)
    p = _tiny_params(cfg)
    rng = np.random.default_rng(14)
    tok = rng.integers(0, cfg["vocab"], (1, 10)); y = rng.integers(0, cfg["vocab"], (1, 10))
    cfg_off = dict(cfg, smear=False)
    p_neg = dict(p, smear_gate=np.full(12, -1e4))
    # gate inputs are RMSNorm'd embedding channels; make them all positive so
    # the logit is strongly negative for every token
    p_neg["wte"] = np.abs(p["wte"])
    p_off = dict(p, wte=p_neg["wte"])
    l_neg, _ = O.forward(cfg, p_neg, tok, y)
    l_off, _ = O.forward(cfg_off, p_off, tok, y)
    assert np.allclose(l_neg, l_off, atol=1e-12)
    x_on = O.embed(cfg, p, tok[0]); x_off = O.embed(cfg_off, p, tok[0])
    assert np.array_equal(x_on[0], x_off[0]) and not np.allclose(x_on[1:], x_off[1:])


def test_backout_beta_invariance_at_depth_one():
    """At depth 1 the backout block is the last block, so x - beta x =
    (1 - beta) x and the final RMSNorm removes the factor for beta < 1."""
    cfg = O.make_config(1, 12, 12, vocab=80)
    p = _tiny_params(cfg)
    rng = np.random.default_rng(15)
    tok = rng.integers(0, 80, (1, 12)); y = rng.integers(0, 80, (1, 12))
    ref = None
    for beta in (0.0, 0.3, 0.9):
        p["backout_lambda"] = beta
        l, _ = O.forward(cfg, p, tok, y)
        ref = l if ref is None else ref
        assert np.allclose(l, ref, atol=1e-9)


def test_row_independence():
    cfg = _tiny_cfg(depth=2, T=9, short=4)
    p = _tiny_params(cfg)
    rng = np.random.default_rng(16)
    tok = rng.integers(0, cfg["vocab"], (3, 9)); y = rng.integers(0, cfg["vocab"], (3, 9))
    l, _ = O.forward(cfg, p, tok, y)
    perm = [2, 0, 1]
    lp, _ = O.forward(cfg, p, tok[perm], y[perm])
    assert np.array_equal(lp, l[perm])


def test_model_causality_and_window_reach():
    """In a one-layer model with window w, loss_t depends on tokens in
    [t - w, t] only (attention reaches t - w + 1, smear one further), and on
    the target y_t."""
    T, w = 16, 4
    cfg = O.make_config(1, T, w, vocab=60)
    cfg["windows"] = [w]
    p = _tiny_params(cfg)
    rng = np.random.default_rng(17)
    tok = rng.integers(0, 60, (1, T)); y = rng.integers(0, 60, (1, T))
    base, _ = O.forward(cfg, p, tok, y)
    t = 10
    for j in range(T):
        tok2 = tok.copy(); tok2[0, j] = (tok[0, j] + 17) % 60
        l2, _ = O.forward(cfg, p, tok2, y)
        if t - w <= j <= t:
            assert l2[0, t] != base[0, t], j
        else:
            assert l2[0, t] == base[0, t], j


def test_bf16_rounding_of_inputs():
    a = np.array([1.0, 1.00390625, 1.001953125, -3.14159, 1e-30, 65504.0], np.float32)
    r = synth.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(r, ref)
