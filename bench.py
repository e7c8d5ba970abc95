#!/usr/bin/env python
"""Throughput of the nanochat d24 forward pass + softcapped cross-entropy on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one call of the whole forward pass (embedding + norm + smear, 24
blocks, backout, head, softcap, per-token CE) over one batch of B = 4 rows of
T = 2048 synthetic tokens (8192 tokens), through the C ABI.  Inputs are
resident in HBM when the timed region starts.  The weights (1.46 GB of bf16
matrices plus 0.33 GB of gathered embedding rows per step) are far larger
than the 126 MB L2, so no flush is needed between steps.

Prints one JSON line (rank 0).  With N > 1 (launched by torch.distributed.run)
every rank runs an independent replica on its own 4 rows: the rows of a batch
are independent sequences and the forward pass has no exchange step, so there
is no data-path collective (weak scaling); the ranks only meet at the timing
barriers, the max-over-ranks reduction of the elapsed time and, after the
timed steps, one all-reduce of (loss sum, valid count) for the mean loss of
the global batch (reported as mean_loss).

--impl reference times the CPU oracle (fp64 numpy) on the host cores instead:
each step is a bounded sample of the same workload (the first 256 positions
of one row: by causality their losses equal those of the full row).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "d24"
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the tcgen05 GEMM
# kernel, from one ncu capture (caches flushed before each launch) of every
# GEMM mode at d24 sizes, weighted by a step's 97 launches; valid for the
# kernel build it was taken on and to be re-measured when the kernel changes
GEMM_DRAM_BYTES_PER_LAUNCH = 146.3e6
METRIC = "fwd+CE tokens/sec at d24 T=2048 on 1 B200; % of BF16 tensor peak"
CPU_SAMPLE_TOKENS = 256
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def workload_desc(n_layer, C, H, D, V, short_window, max_T, backout_layer, softcap, B, T):
    """The workload as the bench line names it; both arms describe it from
    their own configuration (plain numbers)."""
    head = "d24 nanochat GPT forward+CE" if n_layer == 24 else \
        f"profiling case: d24 dimensions cut to {n_layer} blocks, forward+CE"
    return (f"{head}: depth {n_layer}, C={C}, {H}x{D} heads, MLP {4 * C} ReLU^2, V={V}, SSSL windows "
            f"{short_window}/{max_T} (last block full), value embeddings on odd blocks, "
            f"backout from block {backout_layer}, softcap {softcap:g}, B={B}, T={T}")


def workload_config(desc, B, T, world, seed):
    return {"workload": desc, "global_batch": B * world, "seq_len": T, "tokens_per_step": B * T * world,
            "parallelism": f"replicas x{world} (independent rows; no collective on the data path)",
            "l2": "inputs larger than L2 (1.46 GB bf16 weights + 0.33 GB gathered rows per step)",
            "seed": seed}


def cpu_oracle_run(cfg_o, params, tok, tgt, ntok):
    from oracle import nanochat_fwd as O
    t0 = time.perf_counter()
    O.forward(cfg_o, params, tok[:1, :ntok], tgt[:1, :ntok])
    return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    import numpy as np  # noqa: F401
    from decoder_only_transformer_fwd_b200 import synth
    from oracle import nanochat_fwd as O
    w = synth.WORKLOADS[WORKLOAD]
    seed = synth.SEED_BASE + w["index"]
    ocfg = O.make_config(w["depth"], w["T"], w["short"])
    params = synth.params(seed, n_layer=ocfg["n_layer"], n_embd=ocfg["n_embd"], n_head=ocfg["n_head"],
                          n_kv_head=ocfg["n_kv_head"], head_dim=ocfg["head_dim"], vocab=ocfg["vocab"],
                          vocab_padded=ocfg["vocab_padded"], ve_layers=ocfg["ve_layers"], bf16=True)
    tok = synth.tokens(seed, w["B"], w["T"], ocfg["vocab"])
    tgt = synth.targets(seed, w["B"], w["T"], ocfg["vocab"])
    ntok = min(args.ref_tokens, w["T"])
    for _ in range(args.warmup):
        cpu_oracle_run(ocfg, params, tok, tgt, ntok)
    times = [cpu_oracle_run(ocfg, params, tok, tgt, ntok) for _ in range(args.steps)]
    total = sum(times)
    value = ntok * args.steps / total
    sample = (f"first {ntok} positions of row 0 of the d24 batch per step "
              f"(causal prefix: exact per-token losses), fp64 numpy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(
            workload_desc(ocfg["n_layer"], ocfg["n_embd"], ocfg["n_head"], ocfg["head_dim"], ocfg["vocab"],
                          ocfg["windows"][0], w["T"], ocfg["backout_layer"], ocfg["softcap"], w["B"], w["T"]),
            w["B"], w["T"], world, seed),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def attention_sweep(args, dev, stream):
    """The single attention layer sweep (RoPE + QK-norm, then causal sliding-window
    attention; B = 8, H = 12, D = 128) on the seeded inputs of the parity tests:
    per case the attention kernel's own device time (launch events, averaged
    over `steps` calls) and its algorithmic TFLOP/s, the RoPE + QK-norm
    kernel's time and GB/s (q and k read and written once, bf16, plus the
    cos/sin rows), and the whole nc_attention call."""
    import torch

    from decoder_only_transformer_fwd_b200 import flops, nc, synth
    peaks, _ = load_peaks()
    s = synth.ATTN_SWEEP
    B, H, D = s["B"], s["H"], s["D"]
    out = []
    for T, window in s["cases"]:
        q, k, v = (torch.from_numpy(a).to(dev).to(torch.bfloat16)
                   for a in synth.attention_inputs(synth.SEED_BASE + s["index"], B, T, H, D))
        o = torch.empty_like(q)
        ws = torch.empty(nc.nc_attention_workspace_bytes(B, T, H, H, D, "bf16", 1), dtype=torch.uint8,
                         device=dev)
        call = lambda: nc.nc_attention(q, k, v, o, window, 1, 1.15, D ** -0.5, 100000.0, 1e-6, ws, stream)
        for _ in range(3):
            call()
        timer = nc.LaunchTimer(2 * args.steps, kinds=["attention_tcgen05", "rope_qknorm"])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        with timer:
            for _ in range(args.steps):
                call()
        e1.record(stream)
        torch.cuda.synchronize()
        pk = timer.per_kind()
        n, kms = pk.get("attention_tcgen05", (0, 0.0))
        nr, rms_ = pk.get("rope_qknorm", (0, 0.0))
        f = flops.attention_layer_flops(B, T, H, D, window)
        us = 1e3 * kms / max(n, 1)
        tf = f / (us * 1e-6) / 1e12
        rope_us = 1e3 * rms_ / max(nr, 1)
        rope_bytes = 2 * (2 * B * T * H * D * 2) + 2 * T * (D // 2) * 4
        rope_gbs = rope_bytes / (rope_us * 1e-6) / 1e9 if rope_us > 0 else None
        out.append({"T": T, "window": window if window > 0 else "full", "kernel_us": us,
                    "call_us": 1e3 * e0.elapsed_time(e1) / args.steps, "gflop": f / 1e9, "tflops": tf,
                    "pct_bf16_peak": 100.0 * tf / peaks["bf16_tflops"],
                    "rope_qknorm": {"us": rope_us, "bytes": rope_bytes, "achieved_gbs": rope_gbs,
                                    "frac": rope_gbs / peaks["hbm_gbs"] if rope_gbs else None}})
        del q, k, v, o, ws
    return out


def head_backward_step(args, model, cfg, tok, tgt, M, stream, peaks):
    """The head backward (nc_head_backward) after a forward at the bench
    workload's sizes: device time per call and the TFLOP/s of its three head
    GEMMs (logits recomputed, dL/dxn, dL/dW_U: 3 x 2 M V C FLOPs)."""
    import torch

    from decoder_only_transformer_fwd_b200 import nc
    loss = torch.empty(M, dtype=torch.float32, device=tok.device)
    dx = torch.empty(M, cfg.n_embd, dtype=torch.float32, device=tok.device)
    dw = torch.empty(cfg.vocab, cfg.n_embd, dtype=torch.float32, device=tok.device)
    ws = torch.empty(nc.nc_head_backward_workspace_bytes(cfg, M), dtype=torch.uint8, device=tok.device)
    nc.nc_forward(model.params, tok, tgt, loss, None, stream)
    for _ in range(3):
        nc.nc_head_backward(model.params, tgt, dx, dw, ws, stream)
    torch.cuda.synchronize()
    timer = nc.LaunchTimer(8 * args.steps, kinds=["gemm_tcgen05_bwd", "head_bwd_rows"])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with timer:
        for _ in range(args.steps):
            nc.nc_head_backward(model.params, tgt, dx, dw, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    pk = timer.per_kind()
    ng, gms = pk.get("gemm_tcgen05_bwd", (0, 0.0))
    gemm_flops = 3 * 2.0 * M * cfg.vocab_padded * cfg.n_embd
    tf = gemm_flops * args.steps / (gms / 1e3) / 1e12 if gms > 0 else None
    return {"workload": f"head backward after the forward: dL/dx [{M}, {cfg.n_embd}] and dL/dW_U "
                        f"[{cfg.vocab}, {cfg.n_embd}] of the mean CE, B*T = {M}",
            "ms_per_call": e0.elapsed_time(e1) / args.steps, "gemm_ms_per_call": gms / args.steps,
            "gemm_tflops": tf, "gemm_frac_of_burst": tf / peaks["bf16_tflops"] if tf else None,
            "launches_per_call": nc.nc_last_launch_count()}


def routing_sweep(args, dev, stream, peaks):
    """The pass-2 routing attention (nc_routing_attention; 256-wide QK, 128-wide
    PV) at B = 8, H = 12, T = 2048, window 1024 and full: kernel time and
    algorithmic TFLOP/s (6 B T H D meankeys)."""
    import torch

    from decoder_only_transformer_fwd_b200 import flops, nc, synth
    s = synth.ATTN_SWEEP
    B, H, D = s["B"], s["H"], s["D"]
    out = []
    for T, window in [(2048, 1024), (2048, 0)]:
        t = [torch.from_numpy(a).to(dev).to(torch.bfloat16)
             for seed in (synth.SEED_BASE + s["index"], synth.SEED_BASE + s["index"] + 1)
             for a in synth.attention_inputs(seed, B, T, H, D)]
        q2, k2, v2, q1, k1 = t[0], t[1], t[2], t[3], t[4]
        o = torch.empty_like(q2)
        call = lambda: nc.nc_routing_attention(q2, k2, v2, q1, k1, o, window, 0.5, stream=stream)
        for _ in range(3):
            call()
        timer = nc.LaunchTimer(2 * args.steps, kinds=["attention_tcgen05"])
        torch.cuda.synchronize()
        with timer:
            for _ in range(args.steps):
                call()
        torch.cuda.synchronize()
        n, kms = timer.per_kind().get("attention_tcgen05", (0, 0.0))
        us = 1e3 * kms / max(n, 1)
        f = 1.5 * flops.attention_layer_flops(B, T, H, D, window)
        tf = f / (us * 1e-6) / 1e12
        out.append({"T": T, "window": window if window > 0 else "full", "kernel_us": us, "gflop": f / 1e9,
                    "tflops": tf, "pct_bf16_peak": 100.0 * tf / peaks["bf16_tflops"]})
        del t, q2, k2, v2, q1, k1, o
    return out


def nested_step(args, dev, stream, peaks):
    """The StairFormer nesting pieces at the README's d24 widths (384 + 1152,
    C = 1536) over M = 8192 rows: PrefixRMSNorm (bytes: x read, bf16 out
    written), the block lower triangular linear map C -> C (algorithmic FLOPs
    of the live blocks only: 2 M sum_a w_a C_a) and the prefix cross-entropy
    of both submodels at V = 32768 (2 M V (C_1 + C_2) FLOPs)."""
    import numpy as np
    import torch

    from decoder_only_transformer_fwd_b200 import nc, synth
    widths, M, V = [384, 1152], 8192, 32768
    Cw = sum(widths)
    x, w, w_u, y = synth.nested_inputs(synth.SEED_BASE + 90, M, Cw, Cw, V, V)
    ends = np.cumsum(widths)
    for a in range(len(widths)):  # dead blocks of the BTL weight are zero
        w[ends[a] - widths[a]:ends[a], ends[a]:] = 0.0
    xd = torch.from_numpy(x).to(dev)
    xb = xd.to(torch.bfloat16)
    wd = torch.from_numpy(w).to(dev).to(torch.bfloat16)
    wud = torch.from_numpy(w_u).to(dev).to(torch.bfloat16)
    yd = torch.from_numpy(y).to(dev)
    xn = torch.empty(M, Cw, dtype=torch.bfloat16, device=dev)
    out = torch.empty(M, Cw, dtype=torch.float32, device=dev)
    loss = torch.empty(len(widths), M, dtype=torch.float32, device=dev)
    ws = torch.empty(int(nc.lib().nc_prefix_ce_workspace_bytes(M, Cw, V)), dtype=torch.uint8, device=dev)
    res = {"workload": "StairFormer nesting pieces, widths 384 + 1152 (C = 1536), M = 8192, V = 32768"}

    def timed(call):
        for _ in range(3):
            call()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        return 1e3 * e0.elapsed_time(e1) / args.steps  # microseconds per call

    us = timed(lambda: nc.nc_prefix_rmsnorm(xd, widths, xn, stream=stream))
    nbytes = M * Cw * (4 + 2)
    res["prefix_rmsnorm"] = {"us": us, "bytes": nbytes, "achieved_gbs": nbytes / (us * 1e-6) / 1e9,
                             "frac": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    us = timed(lambda: nc.nc_btl_linear(xb, wd, out, widths, widths, stream=stream))
    f = 2.0 * M * sum(int(wa) * int(ea) for wa, ea in zip(widths, ends))
    res["btl_linear"] = {"us": us, "gflop": f / 1e9, "tflops": f / (us * 1e-6) / 1e12,
                         "dense_gflop": 2.0 * M * Cw * Cw / 1e9}
    us = timed(lambda: nc.nc_prefix_ce(xd, wud, yd, loss, V, widths, workspace=ws, stream=stream))
    f = 2.0 * M * V * float(sum(ends))
    res["prefix_ce"] = {"us": us, "gflop": f / 1e9, "tflops": f / (us * 1e-6) / 1e12,
                        "pct_bf16_peak": 100.0 * f / (us * 1e-6) / 1e12 / peaks["bf16_tflops"]}
    return res


def generation_step(args, model, cfg, tok, B, T, stream, peaks):
    """One generation step at the bench workload's sizes (nc_generate_next):
    the forward over [B, T], the last-position logits, one token per row drawn
    with temperature 0.8 and top-k 50.  Device time per step (CUDA events), and
    per-launch times of the two kernels that are specific to it."""
    import torch

    from decoder_only_transformer_fwd_b200 import nc, synth
    tau, k = 0.8, 50
    u = torch.from_numpy(synth.uniforms(synth.SEED_BASE, B)).to(tok.device)
    nxt = torch.empty(B, dtype=torch.int32, device=tok.device)
    z = torch.empty(B, cfg.vocab, dtype=torch.float32, device=tok.device)
    call = lambda: nc.nc_generate_next(model.params, tok, tau, k, u, nxt, z, stream)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    per_call = nc.nc_last_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    timer = nc.LaunchTimer(args.steps * 2, kinds=["last_logits", "sample"])
    with timer:
        for _ in range(args.steps):
            call()
    torch.cuda.synchronize()
    pk = timer.per_kind()
    n_ll, ms_ll = pk.get("last_logits", (0, 0.0))
    n_s, ms_s = pk.get("sample", (0, 0.0))
    us_ll = 1e3 * ms_ll / max(n_ll, 1)
    # algorithmic bytes of one k_last_logits launch: W_U [V, C] bf16 once, the
    # B final residual rows (fp32) and the B x V fp32 logits written
    nbytes = cfg.vocab * cfg.n_embd * 2 + B * cfg.n_embd * 4 + B * cfg.vocab * 4
    gbs = nbytes / (us_ll * 1e-6) / 1e9 if us_ll > 0 else None
    return {"workload": f"next-token step: forward over B={B} x T={T}, head on the last position only, "
                        f"temperature {tau}, top-k {k}",
            "ms_per_step": ms, "tokens_per_s": B / (ms / 1e3), "launches_per_step": per_call,
            "last_logits_us": us_ll, "sample_us": 1e3 * ms_s / max(n_s, 1),
            "last_logits_roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs / peaks["hbm_gbs"] if gbs else None, "bytes_per_launch": nbytes}}


def run_ours(args):
    import numpy as np
    import torch

    from decoder_only_transformer_fwd_b200 import flops, nc, replicas, synth

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = synth.WORKLOADS[WORKLOAD]
    B, T = (args.rows or w["B"]), w["T"]
    M = B * T
    seed = synth.SEED_BASE + w["index"]
    cfg = nc.nc_init_config(w["depth"], T, "bf16", "SSSL", w["short"], -1)
    if args.layers:
        # a shorter stack of the same blocks, for profiler captures of single launches
        L = args.layers
        cfg.n_layer = L
        cfg.window[L - 1] = T
        cfg.backout_layer = L // 2
        args.no_cpu_baseline = True
    ve_layers = [l for l in range(cfg.n_layer) if cfg.has_ve[l]]
    params = synth.params(seed, n_layer=cfg.n_layer, n_embd=cfg.n_embd, n_head=cfg.n_head,
                          n_kv_head=cfg.n_kv_head, head_dim=cfg.head_dim, vocab=cfg.vocab,
                          vocab_padded=cfg.vocab_padded, ve_layers=ve_layers, bf16=True)
    # each rank processes its own batch of B rows (rank-dependent tokens)
    tok_h = synth.tokens(replicas.rank_seed(seed, rank), B, T, cfg.vocab)
    tgt_h = synth.targets(replicas.rank_seed(seed, rank), B, T, cfg.vocab)
    model = nc.NcModel(cfg, params, M, device=dev)
    tok = torch.from_numpy(tok_h).to(dev)
    tgt = torch.from_numpy(tgt_h).to(dev)
    loss = torch.empty(M, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        nc.nc_forward(model.params, tok, tgt, loss, None, stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    max_over_ranks = replicas.max_over_ranks

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches_per_step = nc.nc_last_launch_count()
    rc, bits = nc.nc_get_status(stream)
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {nc.STATUS.get(rc)} bits={bits}")

    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    clocks = ClockSampler(ids[local] if local < len(ids) else local)
    clocks.start()
    time.sleep(0.3)

    # ---- timed region A: the whole step, device time, max over ranks ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1))

    # ---- timed region B: the same steps with per-launch events on every kernel ----
    timer = nc.LaunchTimer(launches_per_step * args.steps)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    b0.record(stream)
    with timer:
        for _ in range(args.steps):
            step()
    b1.record(stream)
    torch.cuda.synchronize()
    per_kind = timer.per_kind()
    ms_step_b = b0.elapsed_time(b1) / args.steps

    # ---- e2e: the host-buffer entry point, copies inside the timed region ----
    h_tok = torch.from_numpy(tok_h).pin_memory()
    h_tgt = torch.from_numpy(tgt_h).pin_memory()
    h_loss = torch.empty(M, dtype=torch.float32).pin_memory()
    nc.nc_forward_host(model.params, h_tok, h_tgt, h_loss, stream)
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        # each step copies its inputs in and its per-token loss out; the calls
        # are asynchronous, so the host enqueues the next step while the GPU
        # runs this one, and the clock stops once the last loss is on the host
        nc.nc_forward_host(model.params, h_tok, h_tgt, h_loss, stream)
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(time.perf_counter() - t0)
    attn = None if args.no_attention_sweep else attention_sweep(args, dev, stream)
    gen = None
    if not args.no_generation:
        gen = generation_step(args, model, cfg, tok, B, T, stream, load_peaks()[0])
    bwd = route = nest = None
    if not args.no_variants:
        bwd = head_backward_step(args, model, cfg, tok, tgt, M, stream, load_peaks()[0])
        route = routing_sweep(args, dev, stream, load_peaks()[0])
        nest = nested_step(args, dev, stream, load_peaks()[0])
    clk = clocks.stop()
    rc, bits = nc.nc_get_status(stream)
    if rc != 0:
        raise RuntimeError(f"device status after the timed steps: {nc.STATUS.get(rc)} bits={bits}")
    assert np.all(np.isfinite(h_loss.numpy()))
    # mean loss of the global batch: every rank's (sum, count), one all-reduce
    valid = tgt_h.reshape(-1) >= 0
    mean_loss = replicas.global_mean_loss(float(h_loss.numpy().astype(np.float64)[valid].sum()), int(valid.sum()))

    peaks, peak_src = load_peaks()
    windows = list(cfg.window[:cfg.n_layer])
    f_tok = flops.forward_flops_per_token(cfg.n_layer, cfg.n_embd, cfg.vocab, windows, T)
    ms_step = ms_total / args.steps
    tokens_all = M * world
    value = replicas.aggregate_throughput(M, world, args.steps, ms_total / 1e3)
    tflops = f_tok * M / (ms_step / 1e3) / 1e12

    gemm_flops_step = flops.gemm_flops_per_token(cfg.n_layer, cfg.n_embd, cfg.vocab) * M
    n_gemm, gemm_ms = per_kind.get("gemm_tcgen05", (0, 0.0))
    achieved = (gemm_flops_step * args.steps) / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    roofline = {
        "kernel": "gemm_tcgen05 (k_gemm_tc: QKV, O, FC1, FC2, head+CE)",
        "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
        "peak_kind": f"bf16 dense, burst ({peak_src}): the step is milliseconds long", "unit": "TFLOP/s",
        "frac": (achieved / peaks["bf16_tflops"]) if achieved else None,
        "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]) if achieved else None,
        "traffic": GEMM_DRAM_BYTES_PER_LAUNCH,
        "traffic_note": "cold-cache DRAM bytes (read + write) per GEMM launch, ncu capture of each GEMM "
                        "mode at d24 sizes weighted by the step's launch mix (12 QKV + 12 QKV-with-VE, "
                        "24 O, 24 FC1, 23 FC2 + 1 last-block FC2, 1 head per 97 launches)",
        "launches": n_gemm, "avg_launch_us": 1e3 * gemm_ms / max(n_gemm, 1),
        "share_of_step": gemm_ms / ms_total if ms_total > 0 else None,
        "instrumented_ms_per_step": ms_step_b,
        "timing_note": "avg_launch_us and achieved come from CUDA events recorded around every launch; those "
                       "events cut the programmatic-dependent-launch overlap between kernels, so the step with "
                       "them (instrumented_ms_per_step) runs longer than without (ms_per_step) and the per-launch "
                       "times are upper bounds",
    }

    # the embedding kernel is HBM-bound: per launch it gathers M rows of W_E
    # (bf16) and writes x, x0 (fp32) and bf16(x) for the first norm
    n_emb, ms_emb = per_kind.get("embed_norm_smear", (0, 0.0))
    emb_bytes = M * cfg.n_embd * (2 + 4 + 4 + 2)
    emb_gbs = emb_bytes / (ms_emb / max(n_emb, 1) / 1e3) / 1e9 if ms_emb > 0 else None
    embed_roofline = {"kernel": "k_embed_vec", "bound": "hbm", "achieved": emb_gbs, "peak": peaks["hbm_gbs"],
                      "unit": "GB/s", "frac": emb_gbs / peaks["hbm_gbs"] if emb_gbs else None,
                      "bytes_per_launch": emb_bytes}
    # the CE combine reads one partial sum per (row, 128-column tile half) and
    # the target logit, and writes the loss and the log-sum-exp of each row
    n_ce, ms_ce = per_kind.get("ce_combine", (0, 0.0))
    ce_bytes = M * (2 * ((cfg.vocab_padded + 127) // 128) * 4 + 4 + 4 + 4 + 4)
    ce_gbs = ce_bytes / (ms_ce / max(n_ce, 1) / 1e3) / 1e9 if ms_ce > 0 else None
    ce_roofline = {"kernel": "k_ce_combine", "bound": "hbm", "achieved": ce_gbs, "peak": peaks["hbm_gbs"],
                   "unit": "GB/s", "frac": ce_gbs / peaks["hbm_gbs"] if ce_gbs else None,
                   "bytes_per_launch": ce_bytes, "us": 1e3 * ms_ce / max(n_ce, 1)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import nanochat_fwd as O
        ocfg = O.make_config(w["depth"], T, w["short"])
        ntok = args.cpu_tokens
        dt = cpu_oracle_run(ocfg, params, tok_h, tgt_h, ntok)
        cpu = {"value": ntok / dt, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
               "sample": f"first {ntok} positions of row 0 (causal prefix: exact per-token losses), "
                         f"fp64 numpy oracle, {dt:.1f} s"}

    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(
                workload_desc(cfg.n_layer, cfg.n_embd, cfg.n_head, cfg.head_dim, cfg.vocab, cfg.window[0],
                              cfg.max_T, cfg.backout_layer, cfg.softcap, B, T),
                B, T, world, seed),
            "tflops": tflops, "pct_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
            "pct_bf16_peak_sustained": 100.0 * tflops / peaks["bf16_tflops_sustained"],
            "flops_per_token": f_tok,
            "mean_loss": mean_loss,
            "clocks": clk,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": tokens_all * args.steps / e2e_s, "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * M * 4, "d2h_bytes_per_step": M * 4},
            "gpu_launches": launches_per_step * args.steps,
            "kernel_ms_per_step": {k: v[1] / args.steps for k, v in per_kind.items()},
            # region B's step time minus the summed kernel times: launch gaps,
            # pipeline fill/drain between kernels and the timing events themselves
            "gap_ms_per_step": ms_step_b - sum(v[1] for v in per_kind.values()) / args.steps,
            "embed_roofline": embed_roofline,
            "ce_combine_roofline": ce_roofline,
            "attention_sweep": attn,
            "generation": gen,
            "head_backward": bwd,
            "routing_attention": route,
            "nested": nest,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=1024)
    ap.add_argument("--ref-tokens", type=int, default=CPU_SAMPLE_TOKENS,
                    help="--impl reference: positions of row 0 the oracle runs per step")
    ap.add_argument("--rows", type=int, default=0, help="rows per step (default: the workload's B = 4)")
    ap.add_argument("--no-attention-sweep", action="store_true")
    ap.add_argument("--no-generation", action="store_true", help="skip the generation-step measurement")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the head-backward and routing-attention measurements")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: keep the first N blocks of the d24 stack (1..24)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if not 0 <= args.layers <= 24:
        ap.error("--layers must be in 0..24 (0: all 24 blocks)")
    if args.ref_tokens < 1:
        ap.error("--ref-tokens must be >= 1")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
