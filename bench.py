#!/usr/bin/env python
"""Benchmark of the MoE token round trip (layout -> dispatch -> combine) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload deepseek] [--impl ours|reference]

One step = one pass of the whole path over one synthetic batch: layout (count, scan, host count
sync, assign), FP8 dispatch (with zero padding), BF16 combine, handle release.  The metric is
dispatch+combine algorithmic HBM bytes / step time (layout time counts against it).  N > 1 runs
one independent replica per GPU under torchrun (logical ranks live inside one GPU, so nothing
crosses GPUs); the value is the sum over GPUs of the bytes / max-over-ranks time.

--impl reference times the CPU oracle (single-threaded C, test infrastructure) on a bounded sample
of the same workload each step; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "dispatch+combine GB/s & % of B200 HBM peak at 4096×7168 top-8/256 experts"
UNIT = "GB/s"
WORKLOAD_NAMES = {"deepseek": "deepseek-v3-prefill", "decode": "decode-low-latency", "large": "large-capacity",
                  "skewed": "skewed-load", "tiny": "tiny"}
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------- byte model
def algorithmic_bytes(wl: W.Workload, valid_pairs: int, pad_rows: int, weighted: bool = False) -> dict:
    """Bytes the method must move (not what a kernel happens to move)."""
    T, H, k = wl.tokens, wl.hidden, wl.topk
    row = (H + 4 * (H // 128)) if wl.fp8 else 2 * H
    dispatch = T * H * 2 + valid_pairs * row + (pad_rows * row if wl.zero_padding else 0) + T * k * 8
    combine = valid_pairs * H * 2 + T * H * 2 + (T * H * 2 if wl.bias else 0) + T * k * 8 + (T * k * 4 if weighted else 0)
    layout = 2 * T * k * 8 + T * k * 4 + (valid_pairs + pad_rows) * 8
    return {"dispatch": dispatch, "combine": combine, "layout": layout}


def by_rank_bytes(wl: W.Workload, token_rank_rows: int) -> dict:
    """Non-expanded round trip: dispatch reads x once and writes one FP8 row with its scales and
    its top-k ids and weights per (token, rank) (BF16: a bf16 row), reading the routing and the
    token rows; combine reads every row once, writes the output and reads the token rows."""
    T, H, k, R = wl.tokens, wl.hidden, wl.topk, wl.ranks
    row = (H + 4 * (H // 128)) if wl.fp8 else 2 * H
    return {"dispatch_by_rank": T * H * 2 + token_rank_rows * (row + k * 8) + T * k * 12 + T * R * 4,
            "combine_by_rank": token_rank_rows * H * 2 + T * H * 2 + (T * H * 2 if wl.bias else 0) + T * R * 4}


def backward_bytes(wl: W.Workload, valid_pairs: int, pad_rows: int) -> dict:
    """Cached dispatch (the forward dispatch's bytes) and the combine's backward: grad_out read
    once, one bf16 grad row written per routed row, padding rows zeroed, the slots read."""
    T, H, k = wl.tokens, wl.hidden, wl.topk
    return {"dispatch_cached": algorithmic_bytes(wl, valid_pairs, pad_rows)["dispatch"],
            "combine_backward": T * H * 2 + (valid_pairs + (pad_rows if wl.zero_padding else 0)) * H * 2 + T * k * 8}


def kernel_source_digest(*files: str) -> str:
    """sha256 (first 12 hex digits) of the kernel's sources with comments and blank lines removed,
    so that a traffic record stays tied to the code it measured but survives comment edits."""
    h = hashlib.sha256()
    for f in files:
        src = open(os.path.join(ROOT, "combine_moe_layout_07_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:12]


KERNEL_SOURCES = {"combine": ("combine.cu", "moe_internal.cuh"), "dispatch": ("dispatch.cu", "moe_internal.cuh")}


def measured_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch recorded from an ncu capture of the same kernel source;
    None if no record or if the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_dispatch_combine_deepseek_v3_prefill.md")
    if not os.path.exists(path):
        return None
    digest = kernel_source_digest(*KERNEL_SOURCES[kernel])
    for line in open(path):
        m = re.match(r"\|\s*(\w+)\s*\|\s*([\w-]+)\s*\|\s*([0-9.e+]+)\s*\|\s*([0-9a-f]{12})\s*\|", line)
        if m and m.group(1) == kernel and m.group(2) == workload and m.group(4) == digest:
            return float(m.group(3))
    return None


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (with the GPU's own timestamps) taken while the benchmark runs; the
    summary keeps the samples inside [start, stop] of the timed region, widened by one sampling
    period on each side so that short regions still get a sample."""
    QUERY = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.sink = None
        self.out = ""
        self.t0 = self.t1 = None

    def start(self):
        import tempfile
        # samples go to a file: a pipe left unread until the end fills (64 KiB, about 30 s of
        # samples) and stalls the sampler
        self.sink = tempfile.TemporaryFile(mode="w+")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                                         stdout=self.sink, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.5)   # let the sampler come up before the timed region
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()

    def stop(self, log_path: str | None = None):
        if self.proc is not None:
            time.sleep(2 * self.PERIOD_MS / 1000)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.sink.seek(0)
            self.out = self.sink.read()
            self.sink.close()
        if log_path:
            with open(log_path, "w") as f:
                f.write(self.out)

    def summary(self, t0: float | None = None, t1: float | None = None):
        """Clock record of the window [t0, t1] (default: the marked timed region)."""
        import datetime
        t0 = self.t0 if t0 is None else t0
        t1 = self.t1 if t1 is None else t1
        rows = []
        for r in self.out.strip().splitlines():
            f = [c.strip() for c in r.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        pad = self.PERIOD_MS / 1000 * 1.5
        inside = [r for r in rows if t0 is not None and t0 - pad <= r[0] <= t1 + pad]
        if inside:
            use, where = inside, "timed region"
        elif t0 is not None:  # a gap in the sampler's output: the two samples nearest the window
            mid = 0.5 * (t0 + t1)
            use = sorted(rows, key=lambda r: abs(r[0] - mid))[:2]
            where = "nearest samples (none inside the timed region)"
        else:
            use, where = rows, "whole run (no timed region marked)"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(4) if r[3][i] == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "window": where}


# --------------------------------------------------------------------------- distributed plumbing
def dist_setup(backend: str):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(value: float, device) -> float:
    """Max of a scalar over all ranks (identity when not distributed)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# --------------------------------------------------------------------------- CPU oracle sample
def oracle_sample(wl: W.Workload, tokens: int):
    """Inputs for the CPU oracle (layout, dispatch, combine) on the first `tokens` tokens of the
    workload's batch, generated once; returns run() -> (seconds, algorithmic bytes, description),
    which times one oracle pass over them."""
    import oracle
    tpr = max(1, tokens // wl.ranks)
    sw = wl.with_(tokens_per_rank=tpr)
    idx, w = W.gen_routing(wl)
    idx, w = idx[: sw.tokens].numpy(), w[: sw.tokens].numpy()
    x = W.gen_x(sw)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    E, R, A = sw.experts, sw.ranks, sw.alignment
    lay = oracle.layout(idx, w, E, R, A)
    cap = int(lay.rows_per_rank.max())
    y = W.gen_y(sw, cap).view(torch.int16).numpy().view(np.uint16)
    bias = W.gen_bias(sw).view(torch.int16).numpy().view(np.uint16) if sw.bias else None
    desc = (f"first {sw.tokens} tokens ({tpr}/rank) of the {wl.name} batch, same E/R/k/H/A; "
            f"layout+dispatch+combine by the single-threaded C oracle")

    def run():
        t0 = time.perf_counter()
        lay = oracle.layout(idx, w, E, R, A, cap=cap)
        if sw.fp8:
            oracle.dispatch_fp8(lay, idx, w, xb, E, R, A, cap, sw.zero_padding, want_w=False)
        else:
            oracle.dispatch_bf16(lay, idx, w, xb, E, R, A, cap, sw.zero_padding, want_w=False)
        oracle.combine(idx, lay.slot, y, E, R, bias_bits=bias)
        dt = time.perf_counter() - t0
        valid = int(lay.cnt.sum())
        pad = int(lay.rows_per_rank.sum()) - valid
        b = algorithmic_bytes(sw, valid, pad)
        return dt, b["dispatch"] + b["combine"], desc

    return run


def host_cpu() -> dict:
    """The host the CPU numbers come from: logical CPUs and the model name."""
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "model": model}


def reference_tokens(wl: W.Workload, steps: int, warmup: int) -> int:
    """Tokens per step of the reference arm: 4096 for short runs, fewer for long ones, so that the
    whole run stays near a minute of oracle time (about 0.5 s per 1000 DeepSeek-V3 tokens)."""
    t = int(4096 * 30 / max(1, steps + warmup))
    t = max(16 * wl.ranks, min(4096, t))
    return t // wl.ranks * wl.ranks


def workload_config(wl: W.Workload, cap: int, extra: dict | None = None, step_bytes: int = 0) -> dict:
    cfg = {"workload": WORKLOAD_NAMES.get(wl.name, wl.name), "tokens": wl.tokens,
           "tokens_per_rank": wl.tokens_per_rank, "logical_ranks": wl.ranks, "hidden": wl.hidden,
           "experts": wl.experts, "topk": wl.topk, "expert_alignment": wl.alignment, "routing": wl.routing,
           "dispatch": "fp8_e4m3 1x128 block scales" if wl.fp8 else "bf16",
           "combine": "bf16 out, fp32 accumulate" + (", weighted" if wl.weighted_combine else ", pre-weighted rows")
                      + (", shared-expert bias" if wl.bias else ", no bias"),
           "do_cpu_sync": int(wl.cpu_sync), "do_zero_padding": int(wl.zero_padding),
           "num_sms": wl.num_sms or "all", "recv_capacity_rows": cap,
           "l2": (f"no flush: every step moves {step_bytes / 1e6:.0f} MB (> 126 MB L2)" if step_bytes
                  else "no flush: every step moves more than the 126 MB L2")}
    if extra:
        cfg.update(extra)
    return cfg


# --------------------------------------------------------------------------- reference arm
def run_reference(args) -> int:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = W.WORKLOADS[args.workload]
    tokens = args.ref_tokens or reference_tokens(wl, args.steps, args.warmup)
    run = oracle_sample(wl, tokens)
    times, nbytes, desc = [], 0, ""
    for i in range(args.warmup + args.steps):
        dt, nbytes, desc = run()
        if i >= args.warmup:
            times.append(dt)
    mean = sum(times) / len(times)
    value = nbytes / mean / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, 0, {"sample_tokens": tokens}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                             "host": host_cpu()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, world, dev, stream, step, step_bytes, x, idx, w, y, bias, out, x_c, idx_c, w_c, bias_c):
    """The same round trip with every step's inputs copied from pinned host memory (x, routing,
    expert outputs, bias) and the combined output copied back, timed on the device."""
    x_h = x_c.pin_memory()
    idx_h, w_h = idx_c.pin_memory(), w_c.pin_memory()
    y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    y_h.copy_(y)
    bias_h = bias_c.pin_memory() if bias_c is not None else None
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = x_h.numel() * 2 + idx_h.numel() * 8 + w_h.numel() * 4 + y_h.numel() * 2 + (bias_h.numel() * 2 if bias_h is not None else 0)
    d2h = out_h.numel() * 2

    def e2e_step():
        x.copy_(x_h, non_blocking=True)
        idx.copy_(idx_h, non_blocking=True)
        w.copy_(w_h, non_blocking=True)
        y.copy_(y_h, non_blocking=True)
        if bias_h is not None:
            bias.copy_(bias_h, non_blocking=True)
        step(False)
        out_h.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = reduce_max(a.elapsed_time(b), dev) / n
    return {"value": world * step_bytes / (ms * 1e-3) / 1e9, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n}


# --------------------------------------------------------------------------- workload extras
def decode_latency(step_parts, stream, dev, one_call: bool, n: int = 50) -> dict:
    """Per-call device time of layout, dispatch and combine, median over n steps, warm (the
    previous step's data still in L2) and cold (L2 flushed by writing a buffer of twice the L2
    size before every step).  Each step starts behind a device-side spin of about 200 us, so the
    host has enqueued the three calls before the first event fires: the intervals hold device
    time only, not the host's enqueue time (which an idle GPU would otherwise expose in the
    layout's interval)."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def run(cold: bool) -> dict:
        rec = {"layout": [], "dispatch": [], "combine": [], "total": []}
        for _ in range(n):
            if cold:
                flush.fill_(1)
            torch.cuda._sleep(400_000)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            step_parts(ev, stream)
            torch.cuda.synchronize()
            rec["layout"].append(ev[0].elapsed_time(ev[1]) * 1e3)
            rec["dispatch"].append(ev[1].elapsed_time(ev[2]) * 1e3)
            rec["combine"].append(ev[2].elapsed_time(ev[3]) * 1e3)
            rec["total"].append(ev[0].elapsed_time(ev[3]) * 1e3)
        med = {k: round(statistics.median(v), 2) for k, v in rec.items()}
        if one_call:  # layout and dispatch are one launch: its time is the first interval
            med = {"layout_dispatch": med["layout"], "combine": med["combine"], "total": med["total"]}
        return med

    res = {"unit": "us", "warm": run(False), "cold_l2_flushed": run(True), "samples": n}
    # the same round trip captured once in a CUDA graph (do_cpu_sync=0 path), replayed warm
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step_parts([torch.cuda.Event() for _ in range(4)], torch.cuda.current_stream())
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    res["graph_replay_total"] = round(e0.elapsed_time(e1) * 1e3 / n, 2)
    del g
    return res


def skewed_overlap(step, stream, dev, n_steps: int = 50) -> dict:
    """MoE round trips capped at the workload's num_sms on one stream while a second stream runs
    bf16 4096^3 matmuls: serial vs concurrent device time, and each side's slowdown."""
    a = torch.randn(4096, 4096, device=dev, dtype=torch.bfloat16)
    b = torch.randn(4096, 4096, device=dev, dtype=torch.bfloat16)
    side = torch.cuda.Stream(device=dev)

    def timed(fn, st):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        fn()
        e1.record(st)
        return e0, e1

    def moe_loop():
        for _ in range(n_steps):
            step(False)

    # size the GEMM loop to last about as long as the MoE loop (after cuBLAS warm-up)
    with torch.cuda.stream(side):
        for _ in range(3):
            torch.matmul(a, b)
    torch.cuda.synchronize()
    m0, m1 = timed(moe_loop, stream)
    torch.cuda.synchronize()
    moe_ms = m0.elapsed_time(m1)
    per_gemm = float("inf")
    for _ in range(2):  # twice; the faster run sets the per-call time
        with torch.cuda.stream(side):
            g0, g1 = timed(lambda: [torch.matmul(a, b) for _ in range(20)], side)
        torch.cuda.synchronize()
        per_gemm = min(per_gemm, g0.elapsed_time(g1) / 20)
    n_gemm = max(1, int(round(moe_ms / max(per_gemm, 1e-3))))

    def gemm_loop():
        for _ in range(n_gemm):
            torch.matmul(a, b)

    with torch.cuda.stream(side):
        g0, g1 = timed(gemm_loop, side)
    torch.cuda.synchronize()
    gemm_ms = g0.elapsed_time(g1)
    # concurrent: both streams start after one event
    start = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    side.wait_event(start)
    with torch.cuda.stream(side):
        ge = torch.cuda.Event(enable_timing=True)
        gemm_loop()
        ge.record(side)
    me = torch.cuda.Event(enable_timing=True)
    moe_loop()
    me.record(stream)
    torch.cuda.synchronize()
    moe_c, gemm_c = start.elapsed_time(me), start.elapsed_time(ge)
    wall = max(moe_c, gemm_c)
    return {"unit": "ms", "moe_steps": n_steps, "gemm_calls": n_gemm, "moe_alone": round(moe_ms, 3),
            "gemm_alone": round(gemm_ms, 3), "serial": round(moe_ms + gemm_ms, 3),
            "concurrent_wall": round(wall, 3), "moe_concurrent": round(moe_c, 3), "gemm_concurrent": round(gemm_c, 3),
            "moe_slowdown": round(moe_c / moe_ms, 3), "gemm_slowdown": round(gemm_c / gemm_ms, 3),
            "overlap_saving": round(1 - wall / (moe_ms + gemm_ms), 3)}


# --------------------------------------------------------------------------- our arm
def expert_gemm_measurement(moe, wl, h, x, cap: int, N: int, stream, dev, iters: int = 5) -> dict:
    """The first expert GEMM on this step's FP8 dispatch output, timed alone with CUDA events:
    out [R, cap, N] = per-expert E4M3 x E4M3 GEMM over K = H with 1x128 row scales and 128x128
    weight scales (synthetic weights).  FLOPs count every row the GEMM computes (routed rows and
    alignment padding); the peak is the measured bf16 burst x 2 (the FP8 / BF16 nominal ratio)."""
    E, R, H = wl.experts, wl.ranks, wl.hidden
    g = torch.Generator(device=dev).manual_seed(21)
    qw = torch.randint(0, 256, (E, N, H), generator=g, dtype=torch.uint8, device=dev)
    qw[(qw & 0x7F) == 0x7F] = 0x38
    sw = torch.rand((E, N // 128, H // 128), generator=g, device=dev) / 64 + 1 / 256
    recv = torch.empty(R, cap, H, dtype=torch.uint8, device=dev)
    sc = torch.empty(R, cap, H // 128, dtype=torch.float32, device=dev)
    out = torch.empty(R, cap, N, dtype=torch.bfloat16, device=dev)
    moe.moe_dispatch(h, x, moe.MOE_DTYPE_FP8_E4M3, recv, sc, None, cap=cap, stream=stream)
    rows = int(torch.clamp(h.rows_per_rank(), max=cap).sum())
    for _ in range(2):
        moe.moe_expert_gemm_fp8(h, recv, sc, qw, sw, out, cap=cap, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        moe.moe_expert_gemm_fp8(h, recv, sc, qw, sw, out, cap=cap, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    flops = 2.0 * rows * N * H
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    peak = 2.0 * bf16
    achieved = flops / (ms * 1e-3) / 1e12
    return {"kernel": "k_expert_gemm", "bound": "tensor", "N": N, "K": H, "rows": rows, "ms": ms,
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": ("measured bf16 burst x 2 (MEASURED_PEAKS.json bf16_tflops; fp8/bf16 nominal ratio 2)"
                            if "bf16_tflops" in peaks else "fallback 1.59 PFLOP/s bf16 x 2"),
            "iters": iters}


# steps and CPU-baseline sample of the configurations measured beside the headline one: each
# timed region lasts about 0.3 s (several clock samples), each oracle pass a few seconds at most
SIDE_WORKLOADS = {"decode": {"steps": 4000, "cpu_tokens": 1024},
                  "large": {"steps": 600, "cpu_tokens": 4096},
                  "skewed": {"steps": 300, "cpu_tokens": 8192}}


def measure_workload(moe, wl: W.Workload, args, world: int, rank: int, dev, stream, clk: ClockSampler,
                     steps: int, warmup: int, cpu_tokens: int, want_e2e: bool, headline: bool) -> dict:
    """Times `steps` round trips (layout -> dispatch -> combine -> handle free) of one workload
    after `warmup` untimed ones, bracketed by barrier + synchronize, max over ranks; returns the
    measurement with its per-kernel times, roofline, clocks, CPU-oracle baseline (rank 0, one
    GPU) and the workload's own extras (decode latency, skewed overlap)."""
    stream = torch.cuda.current_stream()
    idx_c, w_c = W.gen_routing(wl)
    x_c = W.gen_x(wl)
    bias_c = W.gen_bias(wl) if wl.bias else None
    idx, w, x = idx_c.to(dev), w_c.to(dev), x_c.to(dev)
    bias = bias_c.to(dev) if bias_c is not None else None
    weights_for_combine = w if wl.weighted_combine else None

    def make_params(cap_rows: int):
        return moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment,
                          recv_capacity_rows=cap_rows, num_sms=wl.num_sms, do_cpu_sync=wl.cpu_sync)

    # capacity: worst-case bound for the no-sync decode path, else the exact counts of this batch
    if wl.max_tokens_per_rank:
        cap = moe.moe_recv_capacity_hint(make_params(1), wl.max_tokens_per_rank)
    else:
        h0 = moe.moe_layout(make_params(0), idx, w)
        cap = int(h0.host_rows_per_rank.max())
        moe.moe_handle_free(h0)
    p_cap = 0 if wl.cpu_sync else cap
    h0 = moe.moe_layout(make_params(cap), idx, w)
    counts = h0.counts().cpu().numpy()
    rows = h0.rows_per_rank().cpu().numpy()
    moe.moe_handle_free(h0)
    valid_pairs = int(counts.sum())
    pad_rows = int(rows.sum()) - valid_pairs
    nb = algorithmic_bytes(wl, valid_pairs, pad_rows, weighted=wl.weighted_combine)
    step_bytes = nb["dispatch"] + nb["combine"]

    dtype_out = moe.MOE_DTYPE_FP8_E4M3 if wl.fp8 else moe.MOE_DTYPE_BF16
    if wl.fp8:
        recv = torch.empty(wl.ranks, cap, wl.hidden, dtype=torch.uint8, device=dev)
        scales = torch.empty(wl.ranks, cap, wl.hidden // 128, dtype=torch.float32, device=dev)
    else:
        recv = torch.empty(wl.ranks, cap, wl.hidden, dtype=torch.bfloat16, device=dev)
        scales = None
    y = W.gen_y_device(wl, cap, device=dev)
    out = torch.empty(wl.tokens, wl.hidden, dtype=torch.bfloat16, device=dev)

    ev = {k: [] for k in ("l0", "l1", "d1", "c1")}
    # without host sync the layout and the dispatch are one call (moe_layout_dispatch)
    one_call = not wl.cpu_sync
    prm = make_params(p_cap)  # made once, as a caller reusing its configuration would

    def step_parts(e, st):
        if e is not None:
            e[0].record(st)
        if one_call:
            h = moe.moe_layout_dispatch(prm, idx, w, x, dtype_out, recv, scales, None,
                                        do_zero_padding=wl.zero_padding, stream=st)
            if e is not None and e[1] is not None:
                e[1].record(st)
        else:
            h = moe.moe_layout(prm, idx, w, stream=st)
            if e is not None and e[1] is not None:
                e[1].record(st)
            moe.moe_dispatch(h, x, dtype_out, recv, scales, None, cap=cap, do_zero_padding=wl.zero_padding,
                             num_sms=wl.num_sms, stream=st)
        if e is not None:
            e[2].record(st)
        moe.moe_combine(h, y, out, topk_weights=weights_for_combine, bias=bias, cap=cap, num_sms=wl.num_sms,
                        stream=st)
        if e is not None:
            e[3].record(st)
        moe.moe_handle_free(h)

    tev = {k: [] for k in ("l0", "d1", "c1")}

    def step(record, timed: bool = False):
        # timed: events at the step's start, after the dispatch and after the combine, none between
        # the host's count wait and the dispatch launch (one there delays the dispatch)
        if not record:
            step_parts(None, stream)
            return
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        if timed:
            e[1] = None
        step_parts(e, stream)
        if timed:
            for key, val in zip(tev, (e[0], e[2], e[3])):
                tev[key].append(val)
        else:
            for key, val in zip(ev, e):
                ev[key].append(val)

    for _ in range(warmup):
        step(False)
    torch.cuda.synchronize()
    hc = moe.moe_layout(make_params(p_cap), idx, w)
    assert moe.moe_handle_status(hc) == moe.MOE_OK
    moe.moe_handle_free(hc)

    # the K timed steps record the combine's duration (the dominant kernel) and the layout +
    # dispatch span; the layout / dispatch split comes from a second, instrumented run, because an
    # event between the host's count wait and the dispatch launch would delay the dispatch
    barrier()
    torch.cuda.synchronize()
    launches0 = moe.moe_kernel_launch_count()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    t_start.record(stream)
    for _ in range(steps):
        step(True, timed=True)
    t_end.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier()
    launches = moe.moe_kernel_launch_count() - launches0
    ms = reduce_max(t_start.elapsed_time(t_end), dev) / steps
    # the per-kernel breakdown from a second, instrumented run of the same step
    for _ in range(max(3, min(steps, 50))):
        step(True)
    torch.cuda.synchronize()
    layout_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(ev["l0"], ev["l1"]))
    dispatch_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(ev["l1"], ev["d1"]))
    combine_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(tev["d1"], tev["c1"]))  # timed steps
    front_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(tev["l0"], tev["d1"]))   # layout + dispatch
    value = world * step_bytes / (ms * 1e-3) / 1e9

    kernels_ms = ({"layout_dispatch": front_ms, "combine": combine_ms} if one_call else
                  {"layout": layout_ms, "dispatch": dispatch_ms, "combine": combine_ms})
    rec = {"value": value, "ms_per_step": ms, "steps": steps, "warmup": warmup, "cap": cap,
           "kernel_times": ("combine and layout+dispatch: CUDA events over the timed steps" if one_call else
                            "combine: CUDA events over the timed steps (layout + dispatch there: "
                            f"{front_ms:.4f} ms); layout and dispatch apart: an instrumented run of the "
                            "same step after them"),
           "window": (w0, w1), "launches": launches, "nb": nb, "valid_pairs": valid_pairs, "pad_rows": pad_rows,
           "rows": rows, "kernels_ms": kernels_ms, "one_call": one_call}
    # end to end through the public API: pinned host inputs -> device, round trip, result -> host
    rec["e2e"] = run_e2e(args, world, dev, stream, step, step_bytes, x, idx, w, y, bias, out, x_c, idx_c, w_c,
                         bias_c) if want_e2e else None
    extras = {}
    if args.expert_gemm and headline:
        if not wl.fp8 or wl.alignment % 128 or wl.hidden % 128 or args.expert_gemm % 128:
            raise SystemExit("--expert-gemm needs an FP8 workload, expert_alignment and N multiples of 128")
        hg = moe.moe_layout(make_params(cap), idx, w, stream=stream)
        extras["expert_gemm"] = expert_gemm_measurement(moe, wl, hg, x, cap, args.expert_gemm, stream, dev)
        moe.moe_handle_free(hg)
    if wl.name == "decode":
        extras["latency"] = decode_latency(step_parts, stream, dev, one_call)
    if wl.name == "skewed":
        extras["overlap"] = skewed_overlap(step, stream, dev)
        extras["rows_per_rank"] = {"max": int(rows.max()), "mean": float(rows.mean()), "min": int(rows.min())}
    rec["extras"] = extras

    peak, peak_kind = hbm_peak()
    kern = {("layout_dispatch" if one_call else "dispatch"): (kernels_ms.get("layout_dispatch", dispatch_ms),
                                                              nb["dispatch"]),
            "combine": (combine_ms, nb["combine"])}
    dom = max(kern, key=lambda k: kern[k][0])
    achieved = kern[dom][1] / (kern[dom][0] * 1e-3) / 1e9
    rec["peak"] = peak
    rec["roofline"] = {"bound": "hbm", "kernel": f"k_{dom}", "achieved": achieved, "peak": peak, "unit": "GB/s",
                       "frac": achieved / peak,
                       "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                       if peak_kind == "measured" else "fallback 6.65 TB/s",
                       "algorithmic_bytes_per_launch": kern[dom][1],
                       "traffic": measured_traffic(dom, wl.name) if dom in KERNEL_SOURCES else None}

    cpu = None
    if world == 1 and rank == 0 and cpu_tokens > 0:
        run = oracle_sample(wl, cpu_tokens)
        passes = [run() for _ in range(3)]
        dt, cb, desc = min(passes)
        cpu = {"value": cb / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": desc + "; best of 3 passes", "host": host_cpu()}
    rec["cpu_baseline"] = cpu
    del recv, scales, y, out, x, idx, w, bias
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def next_rows_measurement(moe, wl: W.Workload, args, world: int, rank: int, dev, clk: ClockSampler,
                          steps: int = 100, warmup: int = 5, cpu_tokens: int = 2048) -> dict:
    """The two widened paths at the headline shape, each timed like the headline step (warm-up,
    barrier-bracketed CUDA events, max over ranks) with its per-kernel times, roofline fraction,
    timed window (the caller adds its clock record) and the oracle on a sample:
      by_rank   non-expanded round trip: layout with the token rows -> by-rank FP8 dispatch (rows
                plus the per-row top-k views) -> by-rank combine of per-rank partial sums;
      backward  cached dispatch (a second dispatch with the step's handle, no layout) -> backward
                of the combine (grad_out scattered to every routed row, padding rows zeroed)."""
    import oracle
    stream = torch.cuda.current_stream()
    T, H, k, E, R, A = wl.tokens, wl.hidden, wl.topk, wl.experts, wl.ranks, wl.alignment
    idx_c, w_c = W.gen_routing(wl)
    idx, w, x = idx_c.to(dev), w_c.to(dev), W.gen_x(wl).to(dev)
    peak, _ = hbm_peak()
    out = {}

    def timed(step, parts):
        for _ in range(warmup):
            step(None)
        torch.cuda.synchronize()
        ev = []
        barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.time()
        t0.record(stream)
        for _ in range(steps):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(parts + 1)]
            step(e)
            ev.append(e)
        t1.record(stream)
        torch.cuda.synchronize()
        w1 = time.time()
        barrier()
        ms = reduce_max(t0.elapsed_time(t1), dev) / steps
        part_ms = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev) for i in range(parts)]
        return ms, part_ms, (w0, w1)

    def record(names, part_ms, part_bytes, ms, window, cpu):
        kern = {n: (t, b) for n, t, b in zip(names, part_ms, part_bytes) if b}
        dom = max(kern, key=lambda n: kern[n][0])
        achieved = kern[dom][1] / (kern[dom][0] * 1e-3) / 1e9
        total = sum(part_bytes)
        return {"value": world * total / (ms * 1e-3) / 1e9, "unit": UNIT, "us_per_step": ms * 1e3, "steps": steps,
                "warmup": warmup, "kernels_us": {n: t * 1e3 for n, t in zip(names, part_ms)},
                "kernels_gbs": {n: b / (t * 1e-3) / 1e9 for n, t, b in zip(names, part_ms, part_bytes) if b},
                "bytes_per_step": dict(zip(names, part_bytes)),
                "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "algorithmic_bytes_per_launch": kern[dom][1], "traffic": None},
                "cpu_baseline": cpu, "timed_window_unix_s": [round(v, 3) for v in window]}

    def oracle_rate(run):
        if not (world == 1 and rank == 0 and cpu_tokens > 0):
            return None
        best = min(run() for _ in range(3))
        return {"value": best[1] / best[0] / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": best[2] + "; best of 3 passes", "host": host_cpu()}

    n_s = cpu_tokens // R * R
    idx_s, w_s = idx_c[:n_s].numpy(), w_c[:n_s].numpy()
    xb_s = W.gen_x(wl.with_(tokens_per_rank=n_s // R)).view(torch.int16).numpy().view(np.uint16)

    # ---- by rank
    pr = moe.params(T, R, E, k, H, A, recv_capacity_rows=0, do_cpu_sync=True, by_rank=True)
    h0 = moe.moe_layout(pr, idx, w)
    tpr = h0.tokens_per_rank().cpu().numpy()
    moe.moe_handle_free(h0)
    cap_r, nr = int(tpr.max()), int(tpr.sum())
    recv = torch.empty(R, cap_r, H, dtype=torch.uint8, device=dev)
    sc = torch.empty(R, cap_r, H // 128, dtype=torch.float32, device=dev)
    ti = torch.empty(R, cap_r, k, dtype=torch.int32, device=dev)
    tw = torch.empty(R, cap_r, k, dtype=torch.float32, device=dev)
    y = W.gen_y_device(wl, cap_r, device=dev)
    o = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

    def step_by_rank(e):
        if e is not None:
            e[0].record(stream)
        h = moe.moe_layout(pr, idx, w, stream=stream)
        if e is not None:
            e[1].record(stream)
        moe.moe_dispatch_by_rank(h, x, moe.MOE_DTYPE_FP8_E4M3, recv, sc, topk_idx=idx, recv_topk_idx=ti,
                                 recv_topk_weights=tw, cap=cap_r, stream=stream)
        if e is not None:
            e[2].record(stream)
        moe.moe_combine_by_rank(h, y, o, cap=cap_r, stream=stream)
        if e is not None:
            e[3].record(stream)
        moe.moe_handle_free(h)

    ms, part, win = timed(step_by_rank, 3)
    bb = by_rank_bytes(wl.with_(bias=False), nr)

    def run_by_rank():
        t0 = time.perf_counter()
        st, tr, rows = oracle.layout_by_rank(idx_s, E, R)
        c = int(rows.max())
        oracle.dispatch_by_rank(idx_s, w_s, tr, xb_s, E, R, c, True)
        yb = np.zeros((R, c, H), np.uint16)
        oracle.combine_by_rank(idx_s, tr, yb, E, R)
        dt = time.perf_counter() - t0
        b = sum(by_rank_bytes(wl.with_(tokens_per_rank=n_s // R, bias=False), int(rows.sum())).values())
        return dt, b, (f"first {n_s} tokens ({n_s // R}/rank) of the batch; by-rank layout + dispatch + combine by "
                       f"the single-threaded C oracle (zero expert outputs)")

    out["by_rank"] = record(["layout", "dispatch_by_rank", "combine_by_rank"], part,
                            [0, bb["dispatch_by_rank"], bb["combine_by_rank"]], ms, win, oracle_rate(run_by_rank))
    out["by_rank"]["rows"] = {"token_rank_rows": nr, "expanded_rows": int((idx_c >= 0).sum()),
                              "max_per_rank": cap_r}
    del recv, sc, ti, tw, y, o
    torch.cuda.empty_cache()

    # ---- cached dispatch + backward of the combine
    p = moe.params(T, R, E, k, H, A, recv_capacity_rows=0, do_cpu_sync=True)
    h = moe.moe_layout(p, idx, w)
    cap = int(h.host_rows_per_rank.max())
    counts = h.counts().cpu().numpy()
    rows = h.rows_per_rank().cpu().numpy()
    valid, pad = int(counts.sum()), int(rows.sum()) - int(counts.sum())
    recv = torch.empty(R, cap, H, dtype=torch.uint8, device=dev)
    sc = torch.empty(R, cap, H // 128, dtype=torch.float32, device=dev)
    g_out = W.gen_x(wl.with_(seed=wl.seed + 7)).to(dev)
    g_y = torch.empty(R, cap, H, dtype=torch.bfloat16, device=dev)

    def step_backward(e):
        if e is not None:
            e[0].record(stream)
        moe.moe_dispatch(h, x, moe.MOE_DTYPE_FP8_E4M3, recv, sc, None, cap=cap, do_zero_padding=True, stream=stream)
        if e is not None:
            e[1].record(stream)
        moe.moe_combine_backward(h, g_out, g_y, cap=cap, do_zero_padding=True, stream=stream)
        if e is not None:
            e[2].record(stream)

    ms, part, win = timed(step_backward, 2)
    bw = backward_bytes(wl.with_(zero_padding=True), valid, pad)

    def run_backward():
        t0 = time.perf_counter()
        lay = oracle.layout(idx_s, w_s, E, R, A)
        c = int(lay.rows_per_rank.max())
        lay = oracle.layout(idx_s, w_s, E, R, A, cap=c)
        oracle.dispatch_fp8(lay, idx_s, w_s, xb_s, E, R, A, c, True, want_w=False)
        oracle.combine_backward(lay, idx_s, xb_s, E, R, A, c)
        dt = time.perf_counter() - t0
        v = int(lay.cnt.sum())
        b = sum(backward_bytes(wl.with_(tokens_per_rank=n_s // R, zero_padding=True), v,
                               int(lay.rows_per_rank.sum()) - v).values())
        return dt, b, (f"first {n_s} tokens ({n_s // R}/rank) of the batch; layout + FP8 dispatch + combine "
                       f"backward by the single-threaded C oracle")

    out["backward"] = record(["dispatch_cached", "combine_backward"], part,
                             [bw["dispatch_cached"], bw["combine_backward"]], ms, win, oracle_rate(run_backward))
    moe.moe_handle_free(h)
    del recv, sc, g_out, g_y, x, idx, w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def side_record(wl: W.Workload, rec: dict, clk: ClockSampler) -> dict:
    """The compact record of a configuration measured beside the headline one."""
    k = rec["kernels_ms"]
    nb = rec["nb"]
    out = {"value": rec["value"], "unit": UNIT, "us_per_step": rec["ms_per_step"] * 1e3, "steps": rec["steps"],
           "warmup": rec["warmup"], "frac_of_hbm_peak": rec["value"] / rec["peak"],
           "kernels_us": {key: val * 1e3 for key, val in k.items()}, "kernel_times": rec["kernel_times"],
           "kernels_gbs": {("layout_dispatch" if rec["one_call"] else "dispatch"):
                           nb["dispatch"] / k["layout_dispatch" if rec["one_call"] else "dispatch"] / 1e6,
                           "combine": nb["combine"] / k["combine"] / 1e6},
           "bytes_per_step": nb, "valid_rows": rec["valid_pairs"], "padding_rows": rec["pad_rows"],
           "rows_per_rank_max_over_mean": float(rec["rows"].max() / max(rec["rows"].mean(), 1e-9)),
           "roofline": rec["roofline"], "cpu_baseline": rec["cpu_baseline"],
           "clocks": clk.summary(*rec["window"]), "timed_window_unix_s": [round(v, 3) for v in rec["window"]],
           "config": workload_config(wl, rec["cap"], step_bytes=nb["dispatch"] + nb["combine"]), **rec["extras"]}
    return out


def run_ours(args) -> int:
    world, rank, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import combine_moe_layout_07_b200 as moe

    wl = W.WORKLOADS[args.workload]
    if args.tokens_per_rank:
        wl = wl.with_(tokens_per_rank=args.tokens_per_rank)
    stream = torch.cuda.current_stream()
    clk = ClockSampler(local).start()
    rec = measure_workload(moe, wl, args, world, rank, dev, stream, clk, args.steps, args.warmup,
                           0 if args.no_cpu_baseline else args.cpu_tokens, want_e2e=not args.no_e2e, headline=True)
    side = {}
    if not args.no_side_workloads:
        for name, spec in SIDE_WORKLOADS.items():
            if name == wl.name:
                continue
            swl = W.WORKLOADS[name]
            srec = measure_workload(moe, swl, args, world, rank, dev, stream, clk, spec["steps"],
                                    max(3, args.warmup), 0 if args.no_cpu_baseline else spec["cpu_tokens"],
                                    want_e2e=False, headline=False)
            side[name] = srec
    next_rows = None
    if not args.no_side_workloads and wl.name == "deepseek":
        next_rows = next_rows_measurement(moe, wl, args, world, rank, dev, clk,
                                          cpu_tokens=0 if args.no_cpu_baseline else 2048)
    clk.stop(args.clock_log)
    clk.t0, clk.t1 = rec["window"]

    if rank == 0:
        nb, k = rec["nb"], rec["kernels_ms"]
        rows, peak = rec["rows"], rec["peak"]
        line = {"metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "data_types": {"x": "bf16", "recv": "e4m3 + f32 scales" if wl.fp8 else "bf16", "y,out": "bf16"},
                "config": workload_config(wl, rec["cap"], {"parallelism": f"{world} independent replica(s), "
                                                                          f"{wl.ranks} logical EP ranks each"},
                                          step_bytes=nb["dispatch"] + nb["combine"]),
                "frac_of_hbm_peak": rec["value"] / world / peak,
                "frac_of_8tbs_nominal": rec["value"] / world / 8000.0,
                "kernels_ms": k, "kernel_times": rec["kernel_times"],
                "kernels_gbs": {("layout_dispatch" if rec["one_call"] else "dispatch"):
                                nb["dispatch"] / k["layout_dispatch" if rec["one_call"] else "dispatch"] / 1e6,
                                "combine": nb["combine"] / k["combine"] / 1e6},
                "bytes_per_step": nb, "valid_rows": rec["valid_pairs"], "padding_rows": rec["pad_rows"],
                "A_pad": (rec["valid_pairs"] + rec["pad_rows"]) / max(rec["valid_pairs"], 1),
                "rows_per_rank_max_over_mean": float(rows.max() / max(rows.mean(), 1e-9)),
                "roofline": rec["roofline"], "cpu_baseline": rec["cpu_baseline"],
                "e2e": rec["e2e"],
                "gpu_launches": rec["launches"], "clocks": clk.summary(*rec["window"]),
                "library": os.path.relpath(moe.library_path(), ROOT), **rec["extras"]}
        if side:
            line["workloads"] = {WORKLOAD_NAMES[name]: side_record(W.WORKLOADS[name], srec, clk)
                                 for name, srec in side.items()}
        if next_rows:
            for r in next_rows.values():  # the sampler's records are read once it has stopped
                r["clocks"] = clk.summary(*r["timed_window_unix_s"])
            line["next_rows"] = next_rows
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(W.WORKLOADS), default="deepseek")
    ap.add_argument("--cpu-tokens", type=int, default=16384, help="tokens in the CPU-oracle baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="tokens per step of the reference arm (0: 4096, fewer for long runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--expert-gemm", type=int, default=0, metavar="N",
                    help="also time the first expert GEMM (E4M3, K = hidden, N output columns) on the dispatch output")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--clock-log", default=None, metavar="FILE", help="write the raw nvidia-smi clock samples to FILE")
    ap.add_argument("--no-side-workloads", action="store_true",
                    help="measure only the headline workload (not decode, large and skewed beside it)")
    ap.add_argument("--tokens-per-rank", type=int, default=0, help="override the workload's tokens per rank "
                    "(smaller cases for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
