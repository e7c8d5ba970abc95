"""ctypes binding of libnc.so (include/nc.h).

Argument marshalling only: device buffers are torch tensors (PyTorch is used
for allocation and streams), every step of the forward pass runs in the
library's CUDA kernels.  The library is loaded on first use and a missing
build raises immediately; there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

NC_MAX_LAYERS = 64
NC_BF16, NC_FP32 = 0, 1
STATUS = {0: "NC_OK", 1: "NC_ERR_ARG", 2: "NC_ERR_SHAPE", 3: "NC_ERR_ALIGN", 4: "NC_ERR_CUDA",
          5: "NC_ERR_DATA", 6: "NC_ERR_TIMEOUT", 7: "NC_ERR_WORKSPACE"}
STATUS_CODES = {v: k for k, v in STATUS.items()}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnc.so")


class nc_config(C.Structure):
    _fields_ = [("n_layer", C.c_int), ("n_embd", C.c_int), ("n_head", C.c_int),
                ("n_kv_head", C.c_int), ("head_dim", C.c_int), ("vocab", C.c_int),
                ("vocab_padded", C.c_int), ("mlp_hidden", C.c_int), ("max_T", C.c_int),
                ("dtype", C.c_int), ("window", C.c_int * NC_MAX_LAYERS),
                ("has_ve", C.c_int * NC_MAX_LAYERS), ("backout_layer", C.c_int),
                ("gate_channels", C.c_int), ("smear", C.c_int), ("gemm_impl", C.c_int),
                ("attn_impl", C.c_int), ("gemm_pair", C.c_int), ("qk_alpha", C.c_float), ("softmax_scale", C.c_float),
                ("rope_base", C.c_float), ("eps", C.c_float), ("softcap", C.c_float),
                ("ve_gate_scale", C.c_float)]


class nc_layer_params(C.Structure):
    _fields_ = [("w_qkv", C.c_void_p), ("w_o", C.c_void_p), ("w_fc1", C.c_void_p),
                ("w_fc2", C.c_void_p), ("ve", C.c_void_p), ("ve_gate", C.c_void_p)]


class nc_params(C.Structure):
    _fields_ = [("cfg", nc_config), ("wte", C.c_void_p), ("lm_head", C.c_void_p),
                ("smear_gate", C.c_void_p), ("resid_lambdas", C.c_void_p),
                ("x0_lambdas", C.c_void_p), ("backout_lambda", C.c_float),
                ("layer", nc_layer_params * NC_MAX_LAYERS), ("workspace", C.c_void_p),
                ("workspace_bytes", C.c_size_t), ("max_tokens", C.c_int)]


class NcError(RuntimeError):
    pass


_lib = None

_SIGS = {
    "nc_init_config": (C.c_int, [C.POINTER(nc_config), C.c_int, C.c_int, C.c_int, C.c_char_p, C.c_int, C.c_int]),
    "nc_workspace_bytes": (C.c_size_t, [C.POINTER(nc_config), C.c_int]),
    "nc_params_init": (C.c_int, [C.POINTER(nc_params), C.POINTER(nc_config)]),
    "nc_forward": (C.c_int, [C.POINTER(nc_params), C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                             C.c_void_p, C.c_void_p, C.c_void_p]),
    "nc_forward_host": (C.c_int, [C.POINTER(nc_params), C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                                  C.c_void_p, C.c_void_p]),
    "nc_loss_mean": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]),
    "nc_last_logits": (C.c_int, [C.POINTER(nc_params), C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "nc_sample": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_float, C.c_int, C.c_void_p, C.c_void_p,
                            C.c_void_p]),
    "nc_generate_next": (C.c_int, [C.POINTER(nc_params), C.c_void_p, C.c_int, C.c_int, C.c_float, C.c_int,
                                   C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "nc_attention_workspace_bytes": (C.c_size_t, [C.c_int] * 7),
    "nc_attention": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                               C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_float, C.c_float,
                               C.c_float, C.c_float, C.c_int, C.c_void_p, C.c_size_t, C.c_void_p]),
    "nc_get_status": (C.c_int, [C.c_void_p, C.POINTER(C.c_int)]),
    "nc_status_string": (C.c_char_p, [C.c_int]),
    "nc_last_error": (C.c_char_p, []),
    "nc_last_launch_count": (C.c_int, []),
    "nc_sizeof": (C.c_size_t, [C.c_int]),
    "nc_set_launch_timing": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_uint]),
    "nc_launch_timing_count": (C.c_int, []),
    "nc_kernel_name": (C.c_char_p, [C.c_int]),
    "nc_attention_noalloc": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                                       C.c_int, C.c_int, C.c_int, C.c_int, C.c_float, C.c_float, C.c_float,
                                       C.c_float, C.c_int, C.c_void_p]),
    "nc_attention_noalloc_max_bytes": (C.c_size_t, []),
    "nc_set_flag_wait_test": (C.c_int, [C.c_int, C.c_double]),
    "nc_prefix_rmsnorm": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_float, C.c_void_p,
                                    C.c_int, C.c_void_p]),
    "nc_btl_linear": (C.c_int, [C.c_void_p] * 3 + [C.c_int] * 3 + [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p]),
    "nc_prefix_ce_workspace_bytes": (C.c_size_t, [C.c_int] * 3),
    "nc_prefix_ce": (C.c_int, [C.c_void_p] * 4 + [C.c_int] * 4 + [C.c_void_p, C.c_int, C.c_float, C.c_float,
                                                                 C.c_void_p, C.c_size_t, C.c_void_p]),
    "nc_routing_attention_workspace_bytes": (C.c_size_t, [C.c_int] * 4),
    "nc_routing_attention": (C.c_int, [C.c_void_p] * 6 + [C.c_int] * 6 + [C.c_float, C.c_float, C.c_void_p,
                                                                         C.c_size_t, C.c_void_p]),
    "nc_head_backward_workspace_bytes": (C.c_size_t, [C.POINTER(nc_config), C.c_int]),
    "nc_head_backward": (C.c_int, [C.POINTER(nc_params), C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                                   C.c_void_p, C.c_size_t, C.c_void_p]),
}

KERNEL_KINDS = ["embed_norm_smear", "rmsnorm", "rope_table", "rope_qknorm", "gemm_tcgen05",
                "gemm_cuda_core", "attention_tcgen05", "attention_cuda_core", "ce_combine", "ce_rows",
                "loss_mean", "last_logits", "sample", "gemm_tcgen05_bwd", "head_bwd_rows", "prefix_rmsnorm"]


class LaunchTimer:
    """Per-launch CUDA-event timing of the library's kernels (nc_set_launch_timing).

    Events are created through torch (the library allocates nothing); use as
    a context manager around the calls to time, then read `per_kind()` after a
    synchronize: {kind name: (launches, total ms)}."""

    def __init__(self, capacity: int, kinds=None):
        import torch
        self.capacity = capacity
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:          # materialise the cudaEvent_t handles
            e.record()
        self._handles = (C.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self._kinds = (C.c_int * capacity)()
        mask = 0
        for k in (kinds or KERNEL_KINDS):
            mask |= 1 << KERNEL_KINDS.index(k)
        self.mask = mask
        self.n = 0

    def __enter__(self):
        _check(lib().nc_set_launch_timing(C.cast(self._handles, C.c_void_p), C.cast(self._kinds, C.c_void_p),
                                          self.capacity, self.mask), "nc_set_launch_timing")
        return self

    def __exit__(self, *exc):
        self.n = int(lib().nc_launch_timing_count())
        lib().nc_set_launch_timing(None, None, 0, 0)
        return False

    def per_kind(self) -> dict:
        out = {}
        for i in range(self.n):
            name = KERNEL_KINDS[self._kinds[i]]
            ms = self.events[2 * i].elapsed_time(self.events[2 * i + 1])
            c, t = out.get(name, (0, 0.0))
            out[name] = (c + 1, t + ms)
        return out


def lib():
    """Load libnc.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise NcError(f"{LIB_PATH} is missing: build it with "
                          "`python -m decoder_only_transformer_fwd_b200.build`")
        h = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        err = lib().nc_last_error().decode()
        raise NcError(f"{what}: {STATUS.get(rc, rc)} ({lib().nc_status_string(rc).decode()}) {err}")


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


# --------------------------------------------------------------------------
# the C calls, same names
# --------------------------------------------------------------------------

def nc_init_config(depth: int, max_T: int, dtype: str = "bf16", window_pattern: str = "SSSL",
                   short_window: int | None = None, backout_layer: int = -1) -> nc_config:
    cfg = nc_config()
    dt = NC_BF16 if dtype == "bf16" else NC_FP32
    sw = max_T // 2 if short_window is None else short_window
    _check(lib().nc_init_config(C.byref(cfg), depth, max_T, dt, window_pattern.encode(), sw,
                                backout_layer), "nc_init_config")
    return cfg


def nc_workspace_bytes(cfg: nc_config, max_tokens: int) -> int:
    return int(lib().nc_workspace_bytes(C.byref(cfg), max_tokens))


def nc_forward(params: nc_params, tokens, targets, out_loss, out_logits=None, stream=None):
    B, T = tokens.shape
    _check(lib().nc_forward(C.byref(params), _ptr(tokens), _ptr(targets), B, T, _ptr(out_loss),
                            _ptr(out_logits), _stream(stream)), "nc_forward")


def nc_last_logits(params: nc_params, tokens, out_logits, stream=None):
    """Softcapped logits [B, V] of the last position of each row of tokens [B, T]."""
    B, T = tokens.shape
    _check(lib().nc_last_logits(C.byref(params), _ptr(tokens), B, T, _ptr(out_logits), _stream(stream)),
           "nc_last_logits")


def nc_sample(logits, temperature: float, top_k: int, uniforms, out_next, stream=None):
    """One token per row of logits [B, V] (device fp32, rows may be strided),
    drawn with the row's uniform u in [0, 1) (uniforms: device fp32 [B])."""
    B, V = logits.shape
    _check(lib().nc_sample(_ptr(logits), B, V, logits.stride(0), float(temperature), int(top_k), _ptr(uniforms),
                           _ptr(out_next), _stream(stream)), "nc_sample")


def nc_generate_next(params: nc_params, tokens, temperature: float, top_k: int, uniforms, out_next, out_logits,
                     stream=None):
    B, T = tokens.shape
    _check(lib().nc_generate_next(C.byref(params), _ptr(tokens), B, T, float(temperature), int(top_k),
                                  _ptr(uniforms), _ptr(out_next), _ptr(out_logits), _stream(stream)),
           "nc_generate_next")


def nc_forward_host(params: nc_params, tokens: np.ndarray, targets: np.ndarray, out_loss: np.ndarray,
                    stream=None):
    """tokens/targets/out_loss are host arrays (pinned torch tensors or numpy).
    Asynchronous on `stream`: out_loss is valid after the stream synchronises."""
    B, T = tokens.shape
    ptr = lambda a: C.c_void_p(a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data)
    _check(lib().nc_forward_host(C.byref(params), ptr(tokens), ptr(targets), B, T, ptr(out_loss),
                                 _stream(stream)), "nc_forward_host")


def nc_head_backward_workspace_bytes(cfg: nc_config, max_tokens: int) -> int:
    return int(lib().nc_head_backward_workspace_bytes(C.byref(cfg), max_tokens))


def nc_head_backward(params: nc_params, targets, out_dx, out_dw, workspace, stream=None):
    """dL/dx [B*T, C] and dL/dW_U [V, C] (fp32 device tensors) of the mean CE,
    right after nc_forward on the same params and targets [B, T]."""
    B, T = targets.shape
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().nc_head_backward(C.byref(params), _ptr(targets), B, T, _ptr(out_dx), _ptr(out_dw), _ptr(workspace),
                                  nbytes, _stream(stream)), "nc_head_backward")


def nc_loss_mean(loss, targets, out_mean, stream=None):
    _check(lib().nc_loss_mean(_ptr(loss), _ptr(targets), loss.numel(), _ptr(out_mean),
                              _stream(stream)), "nc_loss_mean")


def nc_attention_workspace_bytes(B, T, H, Hkv, D, dtype="bf16", rope_qknorm=1) -> int:
    dt = NC_BF16 if dtype == "bf16" else NC_FP32
    return int(lib().nc_attention_workspace_bytes(B, T, H, Hkv, D, dt, rope_qknorm))


def nc_attention(q, k, v, out, window: int, rope_qknorm: int = 1, alpha: float = 1.15,
                 softmax_scale: float | None = None, rope_base: float = 100000.0, eps: float = 1e-6,
                 workspace=None, stream=None):
    import torch
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    dt = NC_BF16 if q.dtype == torch.bfloat16 else NC_FP32
    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().nc_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, T, H, Hkv, D, window,
                              rope_qknorm, alpha, scale, rope_base, eps, dt, _ptr(workspace),
                              nbytes, _stream(stream)), "nc_attention")


def nc_routing_attention(q2, k2, v2, q1, k1, out, window: int, gate_logit: float,
                         softmax_scale: float | None = None, workspace=None, stream=None):
    """Pass-2 routing attention (bf16 device tensors [B, T, heads, 128])."""
    import torch
    B, T, H, D = q2.shape
    Hkv = k2.shape[2]
    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    if workspace is None:
        workspace = torch.empty(int(lib().nc_routing_attention_workspace_bytes(B, T, H, D)), dtype=torch.uint8,
                                device=q2.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().nc_routing_attention(_ptr(q2), _ptr(k2), _ptr(v2), _ptr(q1), _ptr(k1), _ptr(out), B, T, H, Hkv, D,
                                      window, gate_logit, scale, _ptr(workspace), nbytes, _stream(stream)),
           "nc_routing_attention")


def _widths(widths):
    arr = (C.c_int * len(widths))(*[int(w) for w in widths])
    return arr, len(widths)


def nc_prefix_rmsnorm(x, widths, out, eps: float = 1e-6, stream=None):
    """PrefixRMSNorm of x [M, C] fp32 into out [M, C] (bf16 or fp32), nested block widths `widths`."""
    import torch
    M, Cw = x.shape
    w, k = _widths(widths)
    _check(lib().nc_prefix_rmsnorm(_ptr(x), M, Cw, w, k, eps, _ptr(out), int(out.dtype == torch.bfloat16),
                                   _stream(stream)), "nc_prefix_rmsnorm")


def nc_btl_linear(x, w, y, in_widths, out_widths, stream=None):
    """y [M, C_out] fp32 = x [M, C_in] bf16 @ W^T with W [C_out, C_in] bf16 block lower triangular."""
    M, C_in = x.shape
    C_out = w.shape[0]
    wi, k = _widths(in_widths)
    wo, k2 = _widths(out_widths)
    if k2 != k:
        raise NcError("nc_btl_linear: in_widths and out_widths differ in length")
    _check(lib().nc_btl_linear(_ptr(x), _ptr(w), _ptr(y), M, C_in, C_out, wi, wo, k, _stream(stream)),
           "nc_btl_linear")


def nc_prefix_ce(x, w_u, targets, out_loss, vocab: int, widths, eps: float = 1e-6, cap: float = 15.0,
                 workspace=None, stream=None):
    """Per-token softcapped CE of every j-front submodel: out_loss [k, M] fp32."""
    import torch
    M, Cw = x.shape
    V_pad = w_u.shape[0]
    wd, k = _widths(widths)
    if workspace is None:
        workspace = torch.empty(int(lib().nc_prefix_ce_workspace_bytes(M, Cw, V_pad)), dtype=torch.uint8,
                                device=x.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().nc_prefix_ce(_ptr(x), _ptr(w_u), _ptr(targets), _ptr(out_loss), M, Cw, vocab, V_pad, wd, k, eps,
                              cap, _ptr(workspace), nbytes, _stream(stream)), "nc_prefix_ce")


def nc_get_status(stream=None) -> tuple[int, int]:
    bits = C.c_int(0)
    rc = lib().nc_get_status(_stream(stream), C.byref(bits))
    return rc, bits.value


def nc_last_launch_count() -> int:
    return int(lib().nc_last_launch_count())


def nc_set_flag_wait_test(skew: int, wait_limit_ms: float):
    _check(lib().nc_set_flag_wait_test(int(skew), float(wait_limit_ms)), "nc_set_flag_wait_test")


# --------------------------------------------------------------------------
# parameter marshalling (allocation through torch)
# --------------------------------------------------------------------------

class NcModel:
    """Device copies of a parameter set (as produced by `synth.params`) plus a
    workspace, and the nc_params struct pointing at them."""

    def __init__(self, cfg: nc_config, host_params: dict, max_tokens: int, device="cuda"):
        import torch
        self.cfg = cfg
        self.device = torch.device(device)
        act = torch.bfloat16 if cfg.dtype == NC_BF16 else torch.float32
        keep = []

        def dev(a, dtype=act):
            t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(self.device).to(dtype)
            keep.append(t)
            return t

        p = nc_params()
        _check(lib().nc_params_init(C.byref(p), C.byref(cfg)), "nc_params_init")
        self.wte = dev(host_params["wte"])
        self.lm_head = dev(host_params["lm_head"])
        self.smear_gate = dev(host_params["smear_gate"], torch.float32)
        self.resid_lambdas = dev(host_params["resid_lambdas"], torch.float32)
        self.x0_lambdas = dev(host_params["x0_lambdas"], torch.float32)
        p.wte, p.lm_head = self.wte.data_ptr(), self.lm_head.data_ptr()
        p.smear_gate = self.smear_gate.data_ptr()
        p.resid_lambdas, p.x0_lambdas = self.resid_lambdas.data_ptr(), self.x0_lambdas.data_ptr()
        p.backout_lambda = float(host_params["backout_lambda"])
        for l, lp in enumerate(host_params["layers"]):
            if lp is None:
                raise ValueError(f"layer {l} missing from the parameter set")
            L = p.layer[l]
            L.w_qkv = dev(lp["w_qkv"]).data_ptr()
            L.w_o = dev(lp["w_o"]).data_ptr()
            L.w_fc1 = dev(lp["w_fc1"]).data_ptr()
            L.w_fc2 = dev(lp["w_fc2"]).data_ptr()
            if lp.get("ve") is not None:
                L.ve = dev(lp["ve"]).data_ptr()
                L.ve_gate = dev(lp["ve_gate"], torch.float32).data_ptr()
        nbytes = nc_workspace_bytes(cfg, max_tokens)
        if nbytes == 0:
            raise NcError("invalid configuration (nc_workspace_bytes returned 0)")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        p.workspace = self.workspace.data_ptr()
        p.workspace_bytes = nbytes
        p.max_tokens = max_tokens
        self._keep = keep
        self.params = p

    def forward(self, tokens, targets, want_logits: bool = False, stream=None):
        import torch
        B, T = tokens.shape
        loss = torch.empty(B * T, dtype=torch.float32, device=self.device)
        logits = (torch.empty(B * T, self.cfg.vocab, dtype=torch.float32, device=self.device)
                  if want_logits else None)
        nc_forward(self.params, tokens, targets, loss, logits, stream)
        return loss, logits

    def generate_next(self, tokens, uniforms, temperature: float = 1.0, top_k: int = 0, stream=None):
        """One generation step: (next tokens [B] int32, last-position logits [B, V])."""
        import torch
        B = tokens.shape[0]
        nxt = torch.empty(B, dtype=torch.int32, device=self.device)
        logits = torch.empty(B, self.cfg.vocab, dtype=torch.float32, device=self.device)
        nc_generate_next(self.params, tokens, temperature, top_k, uniforms, nxt, logits, stream)
        return nxt, logits
