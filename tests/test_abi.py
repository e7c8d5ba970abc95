"""The C ABI without a GPU: the library loads, exports every symbol declared in
include/nc.h, its struct layouts match the ctypes mirrors, and the host-side
logic (configuration, workspace sizing, argument checks) behaves as declared.
No test here launches a kernel."""
import ctypes as C
import os
import re

import pytest

from decoder_only_transformer_fwd_b200 import nc
from oracle import nanochat_fwd as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "nc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nc_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = nc.lib()
    names = _declared_functions()
    assert "nc_forward" in names and "nc_attention" in names and "nc_init_config" in names
    for n in names:
        assert hasattr(lib, n), n


def test_struct_sizes_match_mirrors():
    lib = nc.lib()
    assert lib.nc_sizeof(0) == C.sizeof(nc.nc_config)
    assert lib.nc_sizeof(1) == C.sizeof(nc.nc_layer_params)
    assert lib.nc_sizeof(2) == C.sizeof(nc.nc_params)
    assert lib.nc_sizeof(9) == 0


@pytest.mark.parametrize("depth,T,short", [(1, 256, 256), (4, 1024, 512), (12, 2048, 1024),
                                           (24, 2048, 1024), (7, 333, 100)])
def test_init_config_matches_pages(depth, T, short):
    cfg = nc.nc_init_config(depth, T, "bf16", "SSSL", short, -1)
    ref = O.make_config(depth, T, short)
    assert (cfg.n_layer, cfg.n_embd, cfg.n_head, cfg.n_kv_head, cfg.head_dim) == (
        ref["n_layer"], ref["n_embd"], ref["n_head"], ref["n_kv_head"], ref["head_dim"])
    assert cfg.vocab == ref["vocab"] and cfg.vocab_padded == ref["vocab_padded"]
    assert cfg.mlp_hidden == 4 * ref["n_embd"]
    assert list(cfg.window[:depth]) == ref["windows"]
    assert [l for l in range(depth) if cfg.has_ve[l]] == ref["ve_layers"]
    assert cfg.backout_layer == ref["backout_layer"]
    assert cfg.gate_channels == ref["gate_channels"] and cfg.smear == 1
    assert abs(cfg.qk_alpha - ref["qk_alpha"]) < 1e-7
    assert abs(cfg.softmax_scale - ref["softmax_scale"]) < 1e-7
    assert cfg.rope_base == ref["rope_base"] and abs(cfg.eps - ref["eps"]) < 1e-12
    assert cfg.softcap == ref["softcap"] and cfg.ve_gate_scale == ref["ve_gate_scale"]


def test_init_config_rejects_bad_arguments():
    lib = nc.lib()
    cfg = nc.nc_config()
    assert lib.nc_init_config(None, 4, 1024, 0, b"SSSL", 512, -1) == 1
    assert lib.nc_init_config(C.byref(cfg), 0, 1024, 0, b"SSSL", 512, -1) == 1
    assert lib.nc_init_config(C.byref(cfg), 65, 1024, 0, b"SSSL", 512, -1) == 1
    assert lib.nc_init_config(C.byref(cfg), 4, 1024, 7, b"SSSL", 512, -1) == 1
    assert lib.nc_init_config(C.byref(cfg), 4, 1024, 0, b"SSXL", 512, -1) == 1
    assert lib.nc_init_config(C.byref(cfg), 4, 1024, 0, b"", 512, -1) == 1
    assert lib.nc_init_config(C.byref(cfg), 4, 1024, 0, b"SSSL", 512, 4) == 1
    assert lib.nc_init_config(C.byref(cfg), 4, 1024, 0, b"L", 512, 1) == 0
    assert list(cfg.window[:4]) == [1024] * 4 and cfg.backout_layer == 1


def test_workspace_bytes():
    cfg = nc.nc_init_config(24, 2048, "bf16", "SSSL", 1024)
    w1 = nc.nc_workspace_bytes(cfg, 8192)
    w2 = nc.nc_workspace_bytes(cfg, 4096)
    assert w1 > w2 > 0 and w1 % 256 == 0
    # residual stream x, x0, x_bo in fp32 plus bf16 activations: at least this much
    C_ = cfg.n_embd
    assert w1 >= 8192 * C_ * (3 * 4 + 2 * (1 + 3 + 1 + 4))
    # bf16 mode never materialises the logits; fp32 mode may
    cfg32 = nc.nc_init_config(24, 2048, "fp32", "SSSL", 1024)
    assert nc.nc_workspace_bytes(cfg32, 8192) > w1 + 8192 * 32768 * 4
    cfg.n_kv_head = 4            # grouped-query attention: 3 query heads per k/v head
    w_gqa = nc.nc_workspace_bytes(cfg, 8192)
    assert 0 < w_gqa < w1
    cfg.n_kv_head = 5            # unsupported: H_kv does not divide H
    assert nc.nc_workspace_bytes(cfg, 8192) == 0


def test_forward_rejects_bad_arguments_without_launching():
    lib = nc.lib()
    cfg = nc.nc_init_config(1, 256, "fp32", "L", 256)
    p = nc.nc_params()
    assert lib.nc_params_init(C.byref(p), C.byref(cfg)) == 0
    buf = (C.c_byte * 4096)()
    addr = C.addressof(buf)
    a16 = C.c_void_p((addr + 15) & ~15)
    # null pointers
    assert lib.nc_forward(C.byref(p), None, a16, 1, 8, a16, None, None) == nc.STATUS_CODES["NC_ERR_ARG"]
    # shape beyond capacity (max_tokens == 0)
    assert lib.nc_forward(C.byref(p), a16, a16, 1, 8, a16, None, None) == nc.STATUS_CODES["NC_ERR_SHAPE"]
    # empty batches
    for B, T in ((0, 8), (1, 0), (-1, 8)):
        assert lib.nc_forward(C.byref(p), a16, a16, B, T, a16, None, None) == nc.STATUS_CODES["NC_ERR_SHAPE"]
        assert lib.nc_last_logits(C.byref(p), a16, B, T, a16, None) == nc.STATUS_CODES["NC_ERR_SHAPE"]
    p.max_tokens = 8
    assert lib.nc_forward(C.byref(p), a16, a16, 1, 300, a16, None, None) == nc.STATUS_CODES["NC_ERR_SHAPE"]
    # missing parameters
    assert lib.nc_forward(C.byref(p), a16, a16, 1, 8, a16, None, None) == nc.STATUS_CODES["NC_ERR_ARG"]
    # misaligned pointers
    for name in ("wte", "lm_head", "smear_gate", "resid_lambdas", "x0_lambdas"):
        setattr(p, name, a16.value)
    for l in range(1):
        L = p.layer[l]
        L.w_qkv = L.w_o = L.w_fc1 = L.w_fc2 = L.ve = L.ve_gate = a16.value
    mis = C.c_void_p(a16.value + 4)
    assert lib.nc_forward(C.byref(p), mis, a16, 1, 8, a16, None, None) == nc.STATUS_CODES["NC_ERR_ALIGN"]
    # missing workspace
    assert lib.nc_forward(C.byref(p), a16, a16, 1, 8, a16, None, None) == nc.STATUS_CODES["NC_ERR_WORKSPACE"]
    # invalid config
    p.cfg.head_dim = 64
    assert lib.nc_forward(C.byref(p), a16, a16, 1, 8, a16, None, None) == nc.STATUS_CODES["NC_ERR_SHAPE"]


def test_attention_rejects_bad_arguments():
    lib = nc.lib()
    buf = (C.c_byte * 4096)()
    a16 = C.c_void_p((C.addressof(buf) + 15) & ~15)
    args = lambda **kw: dict(dict(q=a16, k=a16, v=a16, o=a16, B=1, T=4, H=1, Hkv=1, D=128, w=0, rq=0,
                                  dt=0, ws=None, wsb=0), **kw)

    def call(a):
        return lib.nc_attention(a["q"], a["k"], a["v"], a["o"], a["B"], a["T"], a["H"], a["Hkv"],
                                a["D"], a["w"], a["rq"], 1.15, a.get("scale", 0.088), 1e5, 1e-6, a["dt"],
                                a["ws"], a["wsb"], None)
    assert call(args(q=None)) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert call(args(D=64)) == nc.STATUS_CODES["NC_ERR_SHAPE"]
    assert call(args(Hkv=3, H=4)) == nc.STATUS_CODES["NC_ERR_SHAPE"]  # H_kv must divide H
    assert call(args(Hkv=0, H=4)) == nc.STATUS_CODES["NC_ERR_SHAPE"]
    assert call(args(T=0)) == nc.STATUS_CODES["NC_ERR_SHAPE"]
    assert call(args(dt=5)) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert call(args(scale=0.0)) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert call(args(scale=-1.0)) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert call(args(k=C.c_void_p(a16.value + 2))) == nc.STATUS_CODES["NC_ERR_ALIGN"]
    assert call(args(rq=1)) == nc.STATUS_CODES["NC_ERR_WORKSPACE"]
    assert nc.nc_attention_workspace_bytes(2, 8, 4, 4, 128, "bf16", 1) >= 2 * 2 * 8 * 4 * 128 * 2
    assert nc.nc_attention_workspace_bytes(2, 8, 4, 4, 128, "bf16", 0) == 0


def test_generation_entry_points_reject_bad_arguments():
    lib = nc.lib()
    buf = (C.c_byte * 4096)()
    a16 = C.c_void_p((C.addressof(buf) + 15) & ~15)
    ARG, SHAPE = nc.STATUS_CODES["NC_ERR_ARG"], nc.STATUS_CODES["NC_ERR_SHAPE"]
    # nc_sample(logits, B, V, ldl, temperature, top_k, uniforms, out_next, stream)
    assert lib.nc_sample(None, 1, 8, 8, 1.0, 0, a16, a16, None) == ARG
    assert lib.nc_sample(a16, 1, 8, 8, 1.0, 0, None, a16, None) == ARG
    assert lib.nc_sample(a16, 0, 8, 8, 1.0, 0, a16, a16, None) == SHAPE
    assert lib.nc_sample(a16, 1, 0, 8, 1.0, 0, a16, a16, None) == SHAPE
    assert lib.nc_sample(a16, 1, 8, 7, 1.0, 0, a16, a16, None) == SHAPE
    assert lib.nc_sample(a16, 1, 8, 8, 1.0, -1, a16, a16, None) == SHAPE
    assert lib.nc_sample(a16, 1, 8, 8, -0.5, 0, a16, a16, None) == SHAPE
    assert lib.nc_sample(a16, 1, 8, 8, float("inf"), 0, a16, a16, None) == SHAPE
    assert lib.nc_sample(a16, 1, 8, 8, float("nan"), 0, a16, a16, None) == SHAPE
    cfg = nc.nc_init_config(1, 256, "fp32", "L", 256)
    p = nc.nc_params()
    assert lib.nc_params_init(C.byref(p), C.byref(cfg)) == 0
    assert lib.nc_last_logits(C.byref(p), a16, 1, 8, None, None) == ARG
    assert lib.nc_last_logits(C.byref(p), None, 1, 8, a16, None) == ARG
    assert lib.nc_last_logits(C.byref(p), a16, 1, 8, a16, None) == SHAPE  # max_tokens == 0
    p.max_tokens = 8
    assert lib.nc_last_logits(C.byref(p), a16, 1, 8, a16, None) == ARG    # no weights set
    assert lib.nc_generate_next(C.byref(p), a16, 1, 8, 1.0, 0, None, a16, a16, None) == ARG
    assert lib.nc_generate_next(C.byref(p), a16, 1, 8, 1.0, 0, a16, a16, None, None) == ARG
    assert lib.nc_generate_next(C.byref(p), a16, 1, 8, 1.0, -2, a16, a16, a16, None) == SHAPE
    assert lib.nc_generate_next(C.byref(p), a16, 1, 8, -1.0, 0, a16, a16, a16, None) == SHAPE


@pytest.mark.parametrize("dtype,C_ok,C_bad", [("bf16", 5120, 5248), ("fp32", 1280, 1408)])
def test_last_logits_width_limit(dtype, C_ok, C_bad):
    """The last-position head keeps the x rows in shared memory next to at
    least two stages of W_U: in bf16 (tensor-core form, C a multiple of 64)
    16 rows of x^T at 2 C bytes each and two 32 KB stages within 227 KB, so
    C <= 5168; in fp32 (CUDA-core form) eight fp32 rows next to two stages of
    16 W_U rows within 220 KB, so C <= 1280.  Past the limit the call is
    rejected before any launch; at the limit it gets as far as the (missing)
    workspace."""
    lib = nc.lib()
    buf = (C.c_byte * 4096)()
    a16 = C.c_void_p((C.addressof(buf) + 15) & ~15)
    for width, want in ((C_bad, "NC_ERR_SHAPE"), (C_ok, "NC_ERR_WORKSPACE")):
        cfg = nc.nc_init_config(1, 256, dtype, "L", 256)
        cfg.n_embd, cfg.n_head, cfg.n_kv_head = width, width // 128, width // 128
        cfg.mlp_hidden = 4 * width
        p = nc.nc_params()
        assert lib.nc_params_init(C.byref(p), C.byref(cfg)) == 0
        p.max_tokens = 8
        for name in ("wte", "lm_head", "smear_gate", "resid_lambdas", "x0_lambdas"):
            setattr(p, name, a16.value)
        L = p.layer[0]
        L.w_qkv = L.w_o = L.w_fc1 = L.w_fc2 = L.ve = L.ve_gate = a16.value
        assert lib.nc_last_logits(C.byref(p), a16, 1, 8, a16, None) == nc.STATUS_CODES[want], (width, want)


def test_status_strings():
    lib = nc.lib()
    for code in range(8):
        assert lib.nc_status_string(code)
    assert lib.nc_status_string(99) == b"unknown status"
    assert lib.nc_loss_mean(None, None, 4, None, None) == nc.STATUS_CODES["NC_ERR_ARG"]


def test_flop_accounting_matches_pages():
    """The FLOPs/token table of the StairFormer README (dense d9 and d23,
    head_dim 64, T = 2048) under its convention 2 N_mat + 4 L C T."""
    from golden_io import load
    from decoder_only_transformer_fwd_b200 import flops
    g = load("flops_per_token.txt")
    for depth, head_dim, printed in g["rows"]:
        C_, _ = O.model_dims(depth, head_dim=head_dim)
        f = flops.dense_table_flops_per_token(depth, C_, 32768, g["seq_len"])
        assert abs(f / printed - 1) < g["rtol"], (depth, f, printed)
    # algorithmic d24 count: 12.963 TFLOP per 8192-token step
    w = O.layer_windows(24, 2048, 1024)
    f24 = flops.forward_flops_per_token(24, 1536, 32768, w, 2048)
    assert abs(f24 * 8192 / 1e12 - 12.963) < 5e-3
    assert abs(flops.mean_visible_keys(2048, 1024) - 768.25) < 1e-9
    assert abs(flops.mean_visible_keys(2048, 2048) - 1024.5) < 1e-9
    # brute force of the closed form
    for T, wd in [(7, 3), (10, 10), (5, 9)]:
        assert abs(flops.mean_visible_keys(T, wd) - sum(min(i + 1, wd) for i in range(T)) / T) < 1e-12


def test_flag_wait_test_hook_argument_checks():
    lib = nc.lib()
    assert lib.nc_set_flag_wait_test(-1, 10.0) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert lib.nc_set_flag_wait_test(0, 0.0) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert lib.nc_set_flag_wait_test(0, 1000.5) == nc.STATUS_CODES["NC_ERR_ARG"]
    assert lib.nc_set_flag_wait_test(0, 1000.0) == 0   # normal operation


def test_head_backward_rejects_bad_arguments_without_launching():
    lib = nc.lib()
    buf = (C.c_byte * 4096)()
    a16 = C.c_void_p((C.addressof(buf) + 15) & ~15)
    ARG, SHAPE, WS = (nc.STATUS_CODES[k] for k in ("NC_ERR_ARG", "NC_ERR_SHAPE", "NC_ERR_WORKSPACE"))
    cfg = nc.nc_init_config(4, 256, "bf16", "SSSL", 128)
    p = nc.nc_params()
    assert lib.nc_params_init(C.byref(p), C.byref(cfg)) == 0
    call = lambda **kw: lib.nc_head_backward(C.byref(p), kw.get("y", a16), kw.get("B", 1), kw.get("T", 8),
                                             kw.get("dx", a16), kw.get("dw", a16), kw.get("ws", a16),
                                             kw.get("wsb", 16), None)
    assert call(y=None) == ARG and call(dx=None) == ARG and call(dw=None) == ARG
    assert call() == SHAPE                      # max_tokens == 0
    p.max_tokens = 8
    assert call(T=300) == SHAPE and call(B=0) == SHAPE
    assert call() == WS                         # no forward workspace
    need = lib.nc_head_backward_workspace_bytes(C.byref(cfg), 8)
    assert need >= 8 * cfg.vocab_padded * 2 + 8 * cfg.n_embd * 4
    p.cfg.gemm_impl = 1                         # tensor-core path only
    assert call() == SHAPE
    cfg32 = nc.nc_init_config(4, 256, "fp32", "SSSL", 128)
    assert lib.nc_params_init(C.byref(p), C.byref(cfg32)) == 0
    p.max_tokens = 8
    assert call() == SHAPE                      # bf16 mode only


def test_stairformer_entry_points_reject_bad_arguments():
    """Nested block widths must be 1..8 positive multiples of 64 summing to the
    width; BTL outputs a multiple of 256 wide; the prefix CE's padded vocabulary
    a multiple of 256 and its workspace large enough.  All rejected before any
    launch."""
    lib = nc.lib()
    buf = (C.c_byte * 4096)()
    a16 = C.c_void_p((C.addressof(buf) + 15) & ~15)
    mis = C.c_void_p(a16.value + 4)
    ARG, SHAPE = nc.STATUS_CODES["NC_ERR_ARG"], nc.STATUS_CODES["NC_ERR_SHAPE"]
    ALIGN, WS = nc.STATUS_CODES["NC_ERR_ALIGN"], nc.STATUS_CODES["NC_ERR_WORKSPACE"]

    def w(*v):
        return (C.c_int * len(v))(*v)

    ok = w(384, 1152)
    # nc_prefix_rmsnorm(x, M, C, widths, k, eps, out, out_bf16, stream)
    assert lib.nc_prefix_rmsnorm(None, 4, 1536, ok, 2, 1e-6, a16, 1, None) == ARG
    assert lib.nc_prefix_rmsnorm(a16, 4, 1536, ok, 2, -1.0, a16, 1, None) == ARG
    assert lib.nc_prefix_rmsnorm(a16, 4, 1536, w(384, 1088), 2, 1e-6, a16, 1, None) == SHAPE  # sum != C
    assert lib.nc_prefix_rmsnorm(a16, 4, 1536, w(400, 1136), 2, 1e-6, a16, 1, None) == SHAPE  # not x64
    assert lib.nc_prefix_rmsnorm(a16, 4, 1536, ok, 0, 1e-6, a16, 1, None) == SHAPE
    assert lib.nc_prefix_rmsnorm(a16, 4, 576, w(*([64] * 9)), 9, 1e-6, a16, 1, None) == SHAPE  # k > 8
    assert lib.nc_prefix_rmsnorm(a16, 4, 1536, ok, 2, 1e-6, mis, 1, None) == ALIGN
    assert lib.nc_prefix_rmsnorm(a16, 0, 1536, ok, 2, 1e-6, a16, 1, None) == 0  # nothing to do
    # nc_btl_linear(x, w, y, M, C_in, C_out, in_widths, out_widths, k, stream)
    assert lib.nc_btl_linear(a16, None, a16, 8, 1536, 1536, ok, ok, 2, None) == ARG
    assert lib.nc_btl_linear(a16, a16, a16, 8, 1536, 1152, ok, w(384, 768), 2, None) == SHAPE  # C_out % 256
    assert lib.nc_btl_linear(a16, a16, a16, 8, 1536, 1536, ok, w(512, 1024), 1, None) == SHAPE  # k mismatch
    assert lib.nc_btl_linear(mis, a16, a16, 8, 1536, 1536, ok, ok, 2, None) == ALIGN
    # nc_prefix_ce(x, w_u, targets, out_loss, M, C, V, V_pad, widths, k, eps, cap, ws, ws_bytes, stream)
    assert lib.nc_prefix_ce(a16, a16, None, a16, 8, 1536, 1000, 1024, ok, 2, 1e-6, 15.0, a16, 1 << 30, None) == ARG
    assert lib.nc_prefix_ce(a16, a16, a16, a16, 8, 1536, 1000, 1024, ok, 2, 1e-6, 0.0, a16, 1 << 30, None) == ARG
    assert lib.nc_prefix_ce(a16, a16, a16, a16, 8, 1536, 1000, 1000, ok, 2, 1e-6, 15.0, a16, 1 << 30, None) == SHAPE
    assert lib.nc_prefix_ce(a16, a16, a16, a16, 8, 1536, 1100, 1024, ok, 2, 1e-6, 15.0, a16, 1 << 30, None) == SHAPE
    need = nc.lib().nc_prefix_ce_workspace_bytes(8, 1536, 1024)
    assert need >= 8 * 1536 * 2
    assert lib.nc_prefix_ce(a16, a16, a16, a16, 8, 1536, 1000, 1024, ok, 2, 1e-6, 15.0, a16, need - 1, None) == WS
