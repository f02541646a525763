"""Benchmark of the fused NVFP4 + binary-sign low-rank GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: the activation
quantiser and the fused GEMM (two kernels, the second launched with
programmatic dependent launch), i.e. one `biloco_gemm` call.  The default
workload is the decode shape (M=1, N=K=5120, r=512).  Steps are replayed from
a CUDA graph; each step reads a different copy of the weight so that the copies
together exceed the L2 cache, and the device time of exactly K steps is taken
with CUDA events on the launching stream, bracketed by a barrier and
synchronisation, max over ranks.

Multi-GPU (torchrun): every rank runs an independent replica of the workload
(the operation has no exchange step); `value` is the bytes of all ranks over
the slowest rank's time ("scaling": "weak").

`--impl reference` times the CPU oracle (NumPy/FP64) on a bounded row slice
of the same workload; only rank 0 runs it.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused FP4+binary-lowrank GEMM µs and HBM GB/s (% of peak), M=1–32, r=512"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0


def algo_bytes(M, N, K, r):
    """Algorithmic HBM bytes of one call: weight codes + E4M3 scales + sign bits +
    BF16 activation + BF16 output + FP32 alpha."""
    return N * K // 2 + N * K // 16 + (N + K) * r // 8 + M * K * 2 + M * N * 2 + 4 * r


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------- ncu traffic

KERNEL_SOURCES = os.path.join(ROOT, "nvfp4_binary_rank_b200", "csrc")


def kernel_source_digest() -> str:
    """sha256 over the library's CUDA/C++ sources (names and contents, sorted)."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(os.listdir(KERNEL_SOURCES)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            with open(os.path.join(KERNEL_SOURCES, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, M: int):
    """DRAM bytes (read + write) per launch of the GEMM kernel that serves this
    workload (decode_kernel for M <= 128 under the default schedule), from the
    committed ncu summary, or None when there is none or the kernel sources changed
    since it was captured."""
    kernel = "decode_kernel" if M <= 128 else "fused_kernel"
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("source_digest") != kernel_source_digest():
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(mx)) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm

def setup_problem(w, n_copies, device):
    import torch
    import nvfp4_binary_rank_b200 as nb
    d = workloads.make_inputs(w)
    x = torch.from_numpy(d["x_bf16"].astype(np.int16)).view(torch.bfloat16).to(device)
    R = torch.from_numpy(d["R"]).to(device)
    W, sf, g = nb.pack_weight(R)
    copies = [(W, sf, g)] + [(W.clone(), sf.clone(), g.clone()) for _ in range(n_copies - 1)]
    del R
    if w.r:
        Ub = nb.pack_signs(torch.from_numpy(d["U"].astype(np.float32)).to(device))
        Vb = nb.pack_signs(torch.from_numpy(np.ascontiguousarray(d["V"].T).astype(np.float32)).to(device))
        alpha = torch.from_numpy(d["alpha"]).to(device)
    else:
        Ub = Vb = alpha = None
    y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=device)
    torch.cuda.synchronize()
    return dict(x=x, copies=copies, Ub=Ub, Vb=Vb, alpha=alpha, y=y, host=d)


def n_copies_for(w, l2_bytes):
    per = w.N * w.K // 2 + w.N * w.K // 16
    return max(2, int(np.ceil(1.25 * l2_bytes / per)))


def time_graph(prob, steps, warmup, stream, dist_ctx, spread_pass=True):
    """Device time of exactly `steps` calls replayed from CUDA graphs."""
    import torch
    import nvfp4_binary_rank_b200 as nb
    copies = prob["copies"]
    nc = len(copies)

    def call(i):
        W, sf, g = copies[i % nc]
        nb.gemm(prob["x"], W, sf, g, prob["Ub"], prob["Vb"], prob["alpha"], out=prob["y"])

    with torch.cuda.stream(stream):
        for i in range(max(warmup, 3)):
            call(i)
    stream.synchronize()
    st = nb.last_error(stream)
    if st != 0:
        raise RuntimeError(f"warm-up failed: {nb.status_string(st)}")

    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                call(i)
        return g

    chunk = nc * max(1, 64 // nc)
    full, rem = divmod(steps, chunk)
    g_full = capture(chunk) if full else None
    g_rem = capture(rem) if rem else None
    # warm replay of the graphs themselves
    with torch.cuda.stream(stream):
        if g_full:
            g_full.replay()
        if g_rem:
            g_rem.replay()
    stream.synchronize()

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(full):
            g_full.replay()
        if g_rem:
            g_rem.replay()
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    dist_ctx.barrier()
    ms = start.elapsed_time(end)
    st = nb.last_error(stream)
    if st != 0:
        raise RuntimeError(f"timed region failed: {nb.status_string(st)}")
    del g_full, g_rem
    time_graph.per_step_us, time_graph.chunk = [], chunk
    if not spread_pass:
        return ms
    # The spread, outside the timed region: SPREAD_REPLAYS replays of a graph of
    # `chunk` calls, each bracketed by events; per-step median and 10th percentile.
    g_sp = capture(chunk)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(SPREAD_REPLAYS + 1)]
    with torch.cuda.stream(stream):
        g_sp.replay()
        evs[0].record(stream)
        for i in range(SPREAD_REPLAYS):
            g_sp.replay()
            evs[i + 1].record(stream)
    evs[-1].synchronize()
    time_graph.per_step_us = [evs[i].elapsed_time(evs[i + 1]) * 1e3 / chunk for i in range(SPREAD_REPLAYS)]
    time_graph.chunk = chunk
    if nb.last_error(stream) != 0:
        raise RuntimeError("spread pass failed")
    del g_sp
    return ms


SPREAD_REPLAYS = 30


def spread(per_step_us, chunk):
    """Median and 10th percentile of the per-step times of the spread pass."""
    a = np.asarray(per_step_us, dtype=np.float64)
    if a.size == 0:
        return {"median_us": None, "p10_us": None, "replays": 0}
    return {"median_us": round(float(np.median(a)), 3), "p10_us": round(float(np.percentile(a, 10)), 3),
            "replays": int(a.size), "calls_per_replay": int(chunk)}


def time_isolated(prob, calls, stream):
    """One call at a time, not overlapped with another: each call is bracketed by
    events with a synchronisation before it, and reads a weight copy the calls
    before it did not touch.  Returns the median device time of one call (us)."""
    import torch
    import nvfp4_binary_rank_b200 as nb
    copies = prob["copies"]
    nc = len(copies)
    times = []
    with torch.cuda.stream(stream):
        for i in range(calls + 3):
            W, sf, g = copies[i % nc]
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            stream.synchronize()
            a.record(stream)
            nb.gemm(prob["x"], W, sf, g, prob["Ub"], prob["Vb"], prob["alpha"], out=prob["y"])
            b.record(stream)
            b.synchronize()
            if i >= 3:
                times.append(a.elapsed_time(b) * 1e3)
    if nb.last_error(stream) != 0:
        raise RuntimeError("isolated calls failed")
    return round(float(np.median(times)), 3)


def time_e2e(prob, steps, stream):
    """Same call from pinned host buffers: H2D of x, the call, D2H of y, per step."""
    import torch
    import nvfp4_binary_rank_b200 as nb
    x_host = prob["x"].cpu().pin_memory()
    y_host = torch.empty(prob["y"].shape, dtype=torch.bfloat16).pin_memory()
    copies = prob["copies"]
    nc = len(copies)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(3):
            prob["x"].copy_(x_host, non_blocking=True)
            W, sf, g = copies[i % nc]
            nb.gemm(prob["x"], W, sf, g, prob["Ub"], prob["Vb"], prob["alpha"], out=prob["y"])
            y_host.copy_(prob["y"], non_blocking=True)
        stream.synchronize()
        start.record(stream)
        for i in range(steps):
            prob["x"].copy_(x_host, non_blocking=True)
            W, sf, g = copies[i % nc]
            nb.gemm(prob["x"], W, sf, g, prob["Ub"], prob["Vb"], prob["alpha"], out=prob["y"])
            y_host.copy_(prob["y"], non_blocking=True)
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / steps, x_host.numel() * 2, y_host.numel() * 2


class DistCtx:
    """One process per GPU (torchrun env vars).  NCCL between GPUs; `gloo`
    serves the CPU tests of the rank logic."""

    def __init__(self, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = False

    def init(self):
        import datetime
        import torch
        import torch.distributed as dist
        if self.world > 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            kw = {"timeout": datetime.timedelta(seconds=120)}
            if self.backend == "nccl":
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, **kw)
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def step_metrics(bytes_per_step: int, ms_max: float, steps: int, world: int):
    """(us per step, GB/s of one rank, whole-job GB/s): every rank moves the same
    bytes; the slowest rank's time (ms for `steps` steps) bounds the job."""
    us = ms_max * 1e3 / steps
    gbs_rank = bytes_per_step / (us * 1e-6) / 1e9
    return us, gbs_rank, gbs_rank * world


def measure_config(w, steps, warmup, stream, dist_ctx, l2):
    import torch
    import nvfp4_binary_rank_b200 as nb
    prob = setup_problem(w, n_copies_for(w, l2), torch.device("cuda", torch.cuda.current_device()))
    ms = dist_ctx.max(time_graph(prob, steps, warmup, stream, dist_ctx))
    us = ms * 1e3 / steps
    b = algo_bytes(w.M, w.N, w.K, w.r)
    peak, _ = hbm_peak()
    out = {"us": round(us, 3), "GBps": round(b / (us * 1e-6) / 1e9, 1),
           "frac": round(b / (us * 1e-6) / 1e9 / peak, 4), "bytes": b,
           "M": w.M, "N": w.N, "K": w.K, "r": w.r,
           "kernels": nb.gemm_kernel_count(w.M, w.N, w.K, w.r)}
    out.update(spread(time_graph.per_step_us, time_graph.chunk))
    del prob
    torch.cuda.empty_cache()
    return out


EXTRA_CONFIGS = [
    ("mlp_up", workloads.CONFIGS["mlp_up"]),
    ("mlp_down", workloads.CONFIGS["mlp_down"]),
    ("sweep_M8_r512", workloads.sweep_config(8, 512)),
    ("sweep_M16_r512", workloads.sweep_config(16, 512)),
    ("sweep_M32_r512", workloads.sweep_config(32, 512)),
    ("sweep_M1_r0", workloads.sweep_config(1, 0)),
    ("sweep_M32_r1024", workloads.sweep_config(32, 1024)),
    ("sweep_M64_r512", workloads.sweep_config(64, 512)),
    ("sweep_M128_r512", workloads.sweep_config(128, 512)),
]


def selected_workload(args):
    """The timed workload: a named configuration, or a sweep point (--sweep M,r)."""
    if args.sweep:
        M, r = (int(v) for v in args.sweep.split(","))
        return workloads.sweep_config(M, r)
    return workloads.CONFIGS[args.workload]


def workload_config(w, world):
    """The `config` object of both arms: the workload and how it is laid out."""
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "r": w.r, "seed": w.seed,
            "parallelism": f"replicas x{world}", "l2": "inputs larger than L2"}


def metric_range(head_us, head_frac, extra):
    """The metric over its stated batch range at r = 512, K = 5120: the headline
    (M = 1) and the sweep points M = 8, 16, 32, with the worst of them."""
    pts = {"M1": {"us": round(head_us, 3), "frac": round(head_frac, 4)}}
    for m in (8, 16, 32):
        e = extra.get(f"sweep_M{m}_r512")
        if e:
            pts[f"M{m}"] = {"us": e["us"], "frac": e["frac"]}
    worst = min(pts.items(), key=lambda kv: kv[1]["frac"])
    return {"points": pts, "worst": {"M": int(worst[0][1:]), **worst[1]}}


def run_ours(args):
    import torch
    import nvfp4_binary_rank_b200 as nb
    from nvfp4_binary_rank_b200 import build as _b
    ctx = DistCtx()
    torch.cuda.set_device(ctx.local)
    ctx.init()
    if ctx.rank == 0:
        _b.build()
    ctx.barrier()
    nb.load()
    stream = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(ctx.local).L2_cache_size
    w = selected_workload(args)
    peak, peak_kind = hbm_peak()

    prob = setup_problem(w, n_copies_for(w, l2), torch.device("cuda", ctx.local))
    with ClockSampler(ctx.local) as clk:
        ms_local = time_graph(prob, args.steps, args.warmup, stream, ctx, spread_pass=not args.timed_only)
    head_spread = spread(time_graph.per_step_us, time_graph.chunk)
    ms = ctx.max(ms_local)
    b = algo_bytes(w.M, w.N, w.K, w.r)
    us, gbs_rank, value = step_metrics(b, ms, args.steps, ctx.world)
    isolated_us = None if args.timed_only else time_isolated(prob, 200, stream)

    e2e_steps = 3 if args.timed_only else min(args.steps, 2000)
    e2e_ms, h2d, d2h = time_e2e(prob, e2e_steps, stream)
    e2e_ms = ctx.max(e2e_ms)
    e2e_val = b * ctx.world / (e2e_ms * 1e-3) / 1e9
    del prob
    torch.cuda.empty_cache()

    extra = {}
    rng_line = None
    if not args.no_extra:
        sub_steps = max(2000, args.steps // 20)
        for name, ww in EXTRA_CONFIGS:
            extra[name] = measure_config(ww, sub_steps, args.warmup, stream, ctx, l2)
        rng_line = metric_range(us, gbs_rank / peak, extra)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ctx.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6),
        "us_per_call": round(us, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": workload_config(w, ctx.world),
        "timing": {"l2": f"{n_copies_for(w, l2)} weight copies rotated (> L2 {l2 >> 20} MiB)",
                   "launch": f"CUDA graph replay, {nb.gemm_kernel_count(w.M, w.N, w.K, w.r)} kernel(s) per step",
                   "spread": head_spread,
                   "isolated_us": isolated_us,
                   "isolated": "one call at a time (synchronised before it, not overlapped), median of 200"},
        "roofline": {"bound": "hbm", "achieved": round(gbs_rank, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(gbs_rank / peak, 4),
                     "traffic": ncu_traffic(w.name, w.M),
                     "peak_kind": peak_kind, "per": "step (all kernels of one call)"},
        "e2e": {"value": round(e2e_val, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "us_per_step": round(e2e_ms * 1e3, 3),
                "api": "nvfp4_binary_rank_b200.gemm, eager, pinned host x/y"},
        "gpu_launches": nb.gemm_kernel_count(w.M, w.N, w.K, w.r) * args.steps,
        "clocks": clk.summary(),
        "extra_configs": extra,
        "range_M1_32_r512_K5120": rng_line,
    }
    if ctx.world == 1 and ctx.rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=12.0)
        line["cpu_baseline_1thread"] = cpu_baseline(w, budget_s=6.0, threads=1)
    if ctx.rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_sample(w, rows, kk=None, rr=None):
    """Inputs for the oracle on output rows [0, rows), the first kk elements of K and
    the first rr ranks of the workload: the same problem at a smaller size."""
    from oracle import nvfp4 as on
    kk = w.K if kk is None else kk
    rr = w.r if rr is None else rr
    d = workloads.make_inputs(w)
    wq, ws, g = on.quant_weight(d["R"])
    return dict(x=d["x"][:, :kk], wq=wq[:rows, :kk // 2], ws=ws[:rows, :kk // 16], g=g,
                U=d["U"][:rows, :rr], V=d["V"][:kk, :rr], alpha=d["alpha"][:rr])


def _oracle_step(s):
    from oracle import biloco as ob
    from oracle import nvfp4 as on
    xq, xs = on.quant_act(s["x"])
    y = ob.gemm_part(xq, xs, s["wq"], s["ws"], s["g"])
    if s["alpha"].size:
        y = y + ob.correction_part(s["x"], s["U"], s["V"], s["alpha"])
    return y


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, budget_s=12.0, rows=None, threads=None):
    """The oracle as it stands, timed on the host's cores: NumPy's BLAS threads
    (all cores by default), or `threads` of them."""
    import contextlib
    rows = w.N if rows is None else rows
    s = _oracle_sample(w, rows)
    b = algo_bytes(w.M, rows, w.K, w.r)
    limit = contextlib.nullcontext()
    if threads is not None:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(threads)
    with limit:
        cores = _threads()
        t0 = time.perf_counter()
        n = 0
        while True:
            _oracle_step(s)
            n += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = (time.perf_counter() - t0) / n
    return {"value": round(b / dt / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} full oracle passes (quantise x, FP64 GEMM part from packed weight, "
                      f"FP64 correction) over {w.name} rows 0..{rows}, {dt * 1e3:.1f} ms each"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = selected_workload(args)
    # Each step is a bounded sample of the workload (output rows, a K slice in
    # multiples of 256, a rank slice), shrunk by halving until one step fits
    # 100 s / (steps + warm-up), so that the whole run stays within about 2 minutes.
    target = 100.0 / max(args.steps + args.warmup, 1)
    rows, kk, rr = min(w.N, 128), w.K, w.r

    def step_time(rows, kk, rr):
        smp = _oracle_sample(w, rows, kk, rr)
        _oracle_step(smp)
        t0 = time.perf_counter()
        n = 0
        while n < 3 or time.perf_counter() - t0 < 0.05:
            _oracle_step(smp)
            n += 1
        return (time.perf_counter() - t0) / n

    t = step_time(rows, kk, rr)
    while t > target:
        if rows > 1:
            rows = max(1, rows // 2)
        elif kk > 256:
            kk = max(256, (kk // 2) // 256 * 256)
        elif rr > 1:
            rr = max(1, rr // 2)
        else:
            break
        t = step_time(rows, kk, rr)
    if t < target / 4 and rows == min(w.N, 128) and kk == w.K and rr == w.r:
        rows = int(max(1, min(w.N, rows * 0.5 * target / max(t, 1e-9))))
    s = _oracle_sample(w, rows, kk, rr)
    for _ in range(args.warmup):
        _oracle_step(s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(s)
    dt = (time.perf_counter() - t0) / args.steps
    b = algo_bytes(w.M, rows, kk, rr)
    val = b / dt / 1e9
    sample = f"oracle on output rows 0..{rows}, K elements 0..{kk}, ranks 0..{rr} of {w.name} per step"
    line = {
        "metric": METRIC, "value": round(val, 4), "unit": UNIT, "n_gpus": int(args.gpus),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": workload_config(w, int(args.gpus)),
        "sample": {"rows_per_step": rows, "k_per_step": kk, "ranks_per_step": rr,
                   "whole_problem": bool(rows == w.N and kk == w.K and rr == w.r)},
        "cpu_baseline": {"value": round(val, 4), "unit": UNIT, "cores": _threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(workloads.CONFIGS), default="decode")
    ap.add_argument("--sweep", metavar="M,r", default=None,
                    help="time the sweep point with M rows and rank r at N = K = 5120 instead of --workload "
                         "(for profiler runs of one batch class)")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--timed-only", action="store_true",
                    help="setup and the timed region only (for profiler runs): no spread pass, isolated "
                         "calls, end-to-end loop, other workloads or CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.timed_only:
        args.no_extra = args.no_cpu_baseline = True
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
