"""nc_attention_noalloc: the attention layer for callers that cannot provide
a workspace (for example code inside a host program whose device memory is
owned by another runtime, or a loop that must not call cudaMalloc because it
can synchronise the device).  It keeps its scratch in a fixed array inside the
library.  Checked through the C ABI against nc_attention on the same inputs,
on two calls in a row (the array keeps the previous call's contents, which
must not leak into the next result).  The second call is smaller and has
another T and fewer k/v heads, so its RoPE tables and normalised q and k sit
at other offsets of the array than the first call's: a kernel that read a
byte the current call did not write would see the first call's data.  This
file sorts last so that a run that stops at the first failure has already run
every other test."""
import ctypes as C

import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc, synth

pytestmark = pytest.mark.gpu

ALPHA, BASE, EPS = 1.15, 100000.0, 1e-6


def _call_noalloc(q, k, v, out, window, dtype_code):
    import torch
    B, T, H, D = q.shape
    return nc.lib().nc_attention_noalloc(
        C.c_void_p(q.data_ptr()), C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
        C.c_void_p(out.data_ptr()), B, T, H, k.shape[2], D, window, ALPHA, D ** -0.5, BASE, EPS,
        dtype_code, C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _reference(q, k, v, window):
    import torch
    B, T, H, D = q.shape
    out = torch.empty_like(q)
    dt = "bf16" if q.dtype == torch.bfloat16 else "fp32"
    ws = torch.empty(nc.nc_attention_workspace_bytes(B, T, H, k.shape[2], D, dt, 1), dtype=torch.uint8,
                     device="cuda")
    nc.nc_attention(q, k, v, out, window, 1, ALPHA, D ** -0.5, BASE, EPS, ws)
    return out


# per case: dtype, window, tolerance, then (B, T, H, H_kv) of the first and of the second call
CASES = [("bf16", 96, 2e-2, (2, 300, 4, 4), (1, 131, 4, 2)),
         ("fp32", 0, 1e-4, (1, 200, 2, 2), (1, 77, 2, 1))]


@pytest.mark.parametrize("dtype,window,tol,first,second", CASES)
def test_noalloc_matches_workspace_entry_point_twice(dtype, window, tol, first, second):
    import torch
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    code = nc.NC_BF16 if dtype == "bf16" else nc.NC_FP32
    outs = []
    for call, (B, T, H, Hkv) in enumerate((first, second)):
        q, k, v = (torch.from_numpy(a).cuda().to(tdt)
                   for a in synth.attention_inputs(7100 + call, B, T, H, 128, Hkv=Hkv, bf16=(dtype == "bf16")))
        out = torch.full_like(q, float("nan"))
        rc = _call_noalloc(q, k, v, out, window, code)
        assert rc == 0, nc.STATUS.get(rc, rc)
        assert nc.nc_last_launch_count() == 3  # RoPE tables, RoPE + QK-norm, attention
        ref = _reference(q, k, v, window)
        torch.cuda.synchronize()
        assert nc.nc_get_status()[0] == 0
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= tol, (call, err)
        outs.append(out.float().cpu())
    assert outs[0].shape != outs[1].shape


def test_noalloc_rejects_sizes_beyond_its_array():
    import torch
    cap = nc.lib().nc_attention_noalloc_max_bytes()
    assert cap == 32 << 20
    B, T, H = 1, 8192, 12   # normalised q and k alone need 2 * 8192 * 12 * 128 * 2 bytes = 48 MiB
    q = torch.zeros(B, T, H, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    rc = _call_noalloc(q, q, q, out, 0, nc.NC_BF16)
    assert rc == nc.STATUS_CODES["NC_ERR_WORKSPACE"]
