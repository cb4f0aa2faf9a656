"""Benchmark of the A16W4 per-group matmul on B200.

One step = one pass of the whole hot path over one batch: the MSD matmul
(expansion pre-pass + tcgen05 int8 GEMM with the fused combine) and the
direct-dequant matmul (tcgen05 fp16 GEMM), both on the same inputs.  The
default workload is the M=1 decode GEMV (K=4096, N=4096, g=128).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Rank 0 prints one JSON line.  `value` is whole-job throughput in GB/s of
algorithmic bytes (weights + scales + x + y of both variants per step),
inputs resident in HBM; the timed steps replay a CUDA graph of the library's
launches (kernel launches of ~2-5 us would otherwise be host-bound).  Weights
rotate over enough copies that every read misses the 126 MB L2.

`--impl reference` times the CPU oracle instead (the only other place this
file runs it), on a bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from inputs import WORKLOADS, make_workload, workload as get_workload  # noqa: E402

METRIC = "W4A16 GEMM TFLOP/s and weight GB/s (M≤16) vs B200 roofline, 1 GPU"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------- workload accounting

def step_bytes(wl) -> dict:
    """Algorithmic bytes of one call of each variant: int4 W + fp16 scales + fp16 x + fp16 y."""
    E = wl.E
    w = E * wl.K * wl.N // 2
    s = E * (wl.K // wl.g) * wl.N * 2
    x = wl.M * wl.K * 2
    y = wl.M * wl.N * 2
    return {"w": w, "scale": s, "x": x, "y": y, "total": w + s + x + y}


def step_flops(wl) -> int:
    """Useful flops of one variant call (2*M*N*K; grouped: 2*T*N*K)."""
    return 2 * wl.M * wl.N * wl.K


def kernel_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_int4_a16w4_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def recorded_traffic(workload_name, kernel_name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it is now (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[workload_name][kernel_name]
        if e.get("kernel_sha") != kernel_sha():
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend):
    import datetime
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity for one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job GB/s: the bytes every replica processed in `steps` steps over
    the slowest rank's timed region (`ms_max`, already the max over ranks)."""
    return bytes_per_step * steps * world / (ms_max * 1e-3) / 1e9


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples: W4A16_CLOCKS_DIR if set, else the system temp dir
        out = os.environ.get("W4A16_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out, f"w4a16_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return None
        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- GPU arm

class GpuWorkload:
    """Device-resident inputs for one workload, with weight copies rotated
    so that every call reads its weights from HBM."""

    def __init__(self, w4, torch, wl, case, device):
        self.w4, self.torch, self.wl, self.c = w4, torch, wl, case
        self.grouped = wl.E > 1
        b = step_bytes(wl)
        big = b["w"] + b["scale"] + (b["x"] if wl.M > 16 else 0)
        # distinct copies so consecutive calls never find their operands in L2
        self.copies = 1 if self.grouped else max(2, int(np.ceil(2.2 * L2_BYTES / max(big, 1))))
        if wl.M > 16 and not self.grouped:
            self.copies = min(self.copies, 6)
        if not self.grouped:
            self.copies += self.copies % 2
        self.x = [torch.from_numpy(case.x).to(device)]
        if wl.M > 16 and not self.grouped:
            self.x += [self.x[0].clone() for _ in range(self.copies - 1)]
        wp_logical = [torch.from_numpy(w).to(device) for w in case.wp]
        self.wp = []
        self.sc = []
        for i in range(self.copies):
            self.wp.append([w4.repack(wl_e, wl.K, wl.N) for wl_e in wp_logical])
            self.sc.append([torch.from_numpy(s).to(device) for s in case.scale])
        del wp_logical
        self.offsets = torch.from_numpy(case.offsets).to(device) if self.grouped else None
        # both results in one buffer, so the end-to-end step reads them back in one copy
        self.y_both = torch.empty((2, wl.M, wl.N), dtype=torch.float16, device=device)
        self.y = {op: self.y_both[v] for v, op in enumerate((w4.OP_MSD, w4.OP_DEQUANT))}
        self.ws = {op: w4.alloc_workspace(op, wl.M, wl.K, wl.N, wl.g, E=wl.E, device=device)
                   for op in (w4.OP_MSD, w4.OP_DEQUANT)}

    def call(self, op, i, x=None, y=None):
        w4, wl = self.w4, self.wl
        k = i % self.copies
        x = self.x[k % len(self.x)] if x is None else x
        y = self.y[op] if y is None else y
        if self.grouped:
            w4.w4a16_grouped_matmul(op, x, self.wp[k], self.sc[k], self.offsets, wl.E, wl.M, wl.K, wl.N, wl.g,
                                    y, self.ws[op])
        elif op == w4.OP_MSD:
            w4.w4a16_msd_matmul(x, self.wp[k][0], self.sc[k][0], wl.M, wl.K, wl.N, wl.g, y, self.ws[op])
        else:
            w4.w4a16_dequant_matmul(x, self.wp[k][0], self.sc[k][0], wl.M, wl.K, wl.N, wl.g, y, self.ws[op])

    def step(self, s):
        """One step: MSD then dequant, each on its own weight copy."""
        w4 = self.w4
        for v, op in enumerate((w4.OP_MSD, w4.OP_DEQUANT)):
            self.call(op, 2 * s + v)


def launches_per_step(grouped):
    # MSD: expansion pre-pass + GEMM; dequant: GEMM
    return 3


def run_gpu(args, wl, rank, world, local):
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        init_dist("nccl")
    import weight_only_int4_a16w4_b200 as w4

    case = make_workload(args.workload)
    G = GpuWorkload(w4, torch, wl, case, device)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()

    # warm-up: W eager steps (also sets the kernels' shared-memory attributes)
    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            G.step(s)
    stream.synchronize()
    for op in (w4.OP_MSD, w4.OP_DEQUANT):
        if w4.w4a16_read_status(G.ws[op], stream) != 0:
            raise RuntimeError("device wait timed out during warm-up")

    # one graph = one full weight rotation (period steps); the timed region
    # replays it until exactly K steps have run
    period = max(1, G.copies // 2)
    per_graph = period * max(1, 400 // period)
    nrep, rem = divmod(args.steps, per_graph)
    def capture(n, body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for s in range(n):
                    body(s)
        return g

    # The timed region's start and stop events are nodes of the captured
    # graphs themselves (the first node of the first graph, the last node of
    # the last), so the window holds exactly the K steps as the device runs
    # them, not the host's submission of the graph; the K steps run as: the
    # first graph, nrep - 1 more full graphs, then the remainder.
    t0 = torch.cuda.Event(enable_timing=True, external=True)
    t1 = torch.cuda.Event(enable_timing=True, external=True)

    def capture_timed(n, start, stop):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                if start:
                    t0.record(stream)
                for s in range(n):
                    G.step(s)
                if stop:
                    t1.record(stream)
        return g

    if nrep == 0:
        timed = [capture_timed(rem, True, True)]
        graph = tail = None
    else:
        first = capture_timed(per_graph, True, rem == 0 and nrep == 1)
        graph = capture(per_graph, G.step) if nrep > 1 else None
        tail = capture_timed(rem, False, True) if (rem or nrep > 1) else None
        timed = [first] + [graph] * (nrep - 1) + ([tail] if tail is not None else [])
    # untimed replay to warm the graphs
    with torch.cuda.stream(stream):
        for gr in {id(gr): gr for gr in timed}.values():
            gr.replay()
    stream.synchronize()

    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    sampler.start()
    time.sleep(0.3)
    barrier(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for gr in timed:
            gr.replay()
    stream.synchronize()
    barrier(device)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_local = t0.elapsed_time(t1)
    ms = max_over_ranks(ms_local, device)

    for op in (w4.OP_MSD, w4.OP_DEQUANT):
        if w4.w4a16_read_status(G.ws[op], stream) != 0:
            raise RuntimeError("device wait timed out during the timed region")

    # per-call durations of each variant in steady state: a graph of
    # consecutive calls of that variant alone (weights still rotating),
    # replayed once untimed and once between two events on the launch stream
    per_call_us = {}
    n_op = 2 * period * max(1, 100 // period)
    for op, name in ((w4.OP_MSD, "msd"), (w4.OP_DEQUANT, "dequant")):
        g_op = capture(n_op, lambda s, op=op: G.call(op, s))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g_op.replay()
            e0.record(stream)
            g_op.replay()
            e1.record(stream)
        stream.synchronize()
        per_call_us[name] = e0.elapsed_time(e1) * 1e3 / n_op
        del g_op

    # end to end through the public API with host buffers: per step, the
    # activations go host->device from pinned memory, both variants run, and
    # both results come back to pinned host memory and are read.
    e2e = run_e2e(args, G, torch, w4, stream, device)

    # the other configurations, timed per call in the same run beside the
    # headline one: decode_m16 (the other M <= 16 case) against the copy
    # bandwidth, prefill and moe_e8 against the tensor-pipe peaks
    side = {}
    main_copies, main_grouped = G.copies, G.grouped
    if wl.name == "decode_m1":
        del graph, tail, timed
        del G
        torch.cuda.empty_cache()
        for other in ("decode_m16", "prefill", "moe_e8"):
            side[other] = per_call_detail(w4, torch, get_workload(other), device, stream, capture)

    b = step_bytes(wl)
    bytes_step = 2 * b["total"]
    flops_step = 2 * step_flops(wl)
    value = whole_job_gbs(bytes_step, args.steps, world, ms)
    hbm, bf16, bf16_sus, peak_kind = load_peaks()

    # dominant kernel: the variant with the longer call
    roof = None
    detail = {}
    for name, us in per_call_us.items():
        gbs = b["total"] / (us * 1e-6) / 1e9
        tfl = step_flops(wl) / (us * 1e-6) / 1e12
        detail[name] = {"us_per_call": round(us, 3), "GB/s": round(gbs, 1), "TFLOP/s": round(tfl, 2),
                        "hbm_frac": round(gbs / hbm, 4)}
    if per_call_us:
        dom = max(per_call_us, key=per_call_us.get)
        us = per_call_us[dom]
        if wl.M <= 16:
            ach = b["total"] / (us * 1e-6) / 1e9
            roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(ach / hbm, 4), "traffic": recorded_traffic(wl.name, dom),
                    "kernel": f"{dom} call", "peak_source": peak_kind}
        else:
            ach = step_flops(wl) / (us * 1e-6) / 1e12
            # MSD counts its 6*M*N*K int8 ops against the int8 peak (2x fp16);
            # dequant its 2*M*N*K fp16 flops against the fp16 peak (= bf16)
            peak = bf16 * (2.0 if dom == "msd" else 1.0)
            ach_eff = ach * (3.0 if dom == "msd" else 1.0)
            roof = {"bound": "tensor", "achieved": round(ach_eff, 1), "peak": peak, "unit": "TFLOP/s",
                    "frac": round(ach_eff / peak, 4), "traffic": recorded_traffic(wl.name, dom),
                    "kernel": f"{dom} call", "peak_source": peak_kind}

    detail.update(side)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16 x, int4 w (MSD: int8 MMA / int32 acc; dequant: fp16 MMA / fp32 acc)",
        "data": "synthetic (seeded; x ~ N(0,1) fp16 with 0.1% x20 outliers, w ~ U{-8..7}, scale ~ U[0.005,0.02])",
        "config": {"workload": f"{wl.name}: M={wl.M} K={wl.K} N={wl.N} g={wl.g}" + (f" E={wl.E}" if wl.E > 1 else "")
                   + "; one step = MSD matmul + dequant matmul",
                   "l2": f"weights rotated over {main_copies} copies (> L2) between calls",
                   "timing": f"{args.steps} steps as CUDA graphs of up to {per_graph} steps, the start and stop "
                             f"events being nodes of the first and last graph; per-call times from graphs of {n_op} "
                             f"calls of one variant",
                   "parallelism": f"{world} independent replica(s), one per GPU" if world > 1 else "single GPU",
                   "tflops_per_s": round(flops_step * args.steps * world / (ms * 1e-3) / 1e12, 3)},
        "roofline": roof, "detail": detail, "e2e": e2e,
        "gpu_launches": launches_per_step(main_grouped) * args.steps,
        "clocks": clocks, "kernel_sha": kernel_sha(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, case, budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        graph = tail = timed = None
        dist.destroy_process_group()


def per_call_detail(w4, torch, wl, device, stream, capture):
    """Per-call device time of each variant on another workload: a CUDA graph
    of consecutive calls of one variant (weights rotating past L2), replayed
    once untimed and once between two events on the launch stream."""
    case = make_workload(wl.name)
    G = GpuWorkload(w4, torch, wl, case, device)
    period = max(1, G.copies // 2)
    n_op = 2 * period * max(1, 50 // period)
    hbm, _, _, _ = load_peaks()
    b = step_bytes(wl)
    out = {}
    _, bf16_peak, _, _ = load_peaks()
    for op, name in ((w4.OP_MSD, "msd"), (w4.OP_DEQUANT, "dequant")):
        with torch.cuda.stream(stream):
            for i in range(3):
                G.call(op, i)
        stream.synchronize()
        g_op = capture(n_op, lambda s, op=op: G.call(op, s))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g_op.replay()
            e0.record(stream)
            g_op.replay()
            e1.record(stream)
        stream.synchronize()
        if w4.w4a16_read_status(G.ws[op], stream) != 0:
            raise RuntimeError("device wait timed out")
        us = e0.elapsed_time(e1) * 1e3 / n_op
        gbs = b["total"] / (us * 1e-6) / 1e9
        tfl = step_flops(wl) / (us * 1e-6) / 1e12
        out[name] = {"us_per_call": round(us, 3), "GB/s": round(gbs, 1), "TFLOP/s": round(tfl, 2),
                     "hbm_frac": round(gbs / hbm, 4)}
        if wl.M > 16:
            # MSD: its 6 M N K int8 ops against the int8 peak (2 x the bf16
            # one); dequant: 2 M N K fp16 flops against the bf16 peak
            out[name]["tensor_frac"] = round(tfl * (3.0 if name == "msd" else 1.0) /
                                             (bf16_peak * (2.0 if name == "msd" else 1.0)), 4)
        del g_op
    out["config"] = f"M={wl.M} K={wl.K} N={wl.N} g={wl.g}; weights rotated over {G.copies} copies"
    del G
    torch.cuda.empty_cache()
    return out


def run_e2e(args, G, torch, w4, stream, device):
    """The step end to end through the public API: every step copies x from
    pinned host memory, runs the MSD and the dequant call back to back and
    copies both results back in one copy, then the host reads them.  The step is submitted as a CUDA
    graph of those API calls (one graph per weight-copy pair, replayed in
    turn, so the weights still come from HBM); the eager per-call
    submission is timed too and reported beside it."""
    wl = G.wl
    x_host = torch.from_numpy(G.c.x).pin_memory()
    y_host = torch.empty((2, wl.M, wl.N), dtype=torch.float16).pin_memory()
    y_np = y_host.numpy()                                  # host view of the pinned results
    x_dev = torch.empty_like(G.x[0])
    steps = max(3, min(args.e2e_steps, args.steps))

    def one_step(s):
        x_dev.copy_(x_host, non_blocking=True)
        for v, op in enumerate((w4.OP_MSD, w4.OP_DEQUANT)):
            G.call(op, 2 * s + v, x=x_dev)
        y_host.copy_(G.y_both, non_blocking=True)          # both results in one D2H copy

    def timed(submit):
        with torch.cuda.stream(stream):
            for s in range(steps + 2):
                if s == 2:
                    stream.synchronize()
                    t0 = time.perf_counter()
                    e0 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                submit(s)
                stream.synchronize()          # the host reads both results every step
                _ = float(y_np[0, 0, 0]) + float(y_np[1, 0, 0])
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
        stream.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), device), time.perf_counter() - t0

    ms_eager, wall_eager = timed(one_step)
    period = max(1, G.copies // 2)
    graphs = []
    with torch.cuda.stream(stream):
        for j in range(period):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                one_step(j)
            graphs.append(gr)
    stream.synchronize()
    ms, wall = timed(lambda s: graphs[s % period].replay())
    del graphs
    b = step_bytes(wl)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    return {"value": round(2 * b["total"] * steps * world / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(b["x"]), "d2h_bytes_per_step": int(2 * b["y"]), "steps": steps,
            "us_per_step": round(ms * 1e3 / steps, 2), "wall_us_per_step": round(wall * 1e6 / steps, 2),
            "eager_us_per_step": round(ms_eager * 1e3 / steps, 2),
            "eager_wall_us_per_step": round(wall_eager * 1e6 / steps, 2),
            "note": "each step: H2D x from pinned memory, MSD + dequant calls through the Python binding of the C "
                    "ABI, one D2H of both y, host read; submitted as a CUDA graph of those calls (eager submission "
                    "timed as well); weights resident"}


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)

def oracle_step_sample(oracle, case, wl, cols):
    """The oracle on a bounded sample of one step: both variants, all rows,
    the first `cols` output columns."""
    rows = np.repeat(np.arange(wl.M), cols)
    cc = np.tile(np.arange(cols), wl.M)
    if wl.E > 1:
        oracle.grouped_at("msd", case.x, case.wp, case.scale, case.offsets, wl.g, rows, cc)
        oracle.grouped_at("dequant", case.x, case.wp, case.scale, case.offsets, wl.g, rows, cc)
    else:
        oracle.msd_at(case.x, case.wp[0], case.scale[0], wl.g, rows, cc)
        oracle.dequant_at(case.x, case.wp[0], case.scale[0], wl.g, rows, cc)


def cpu_baseline(wl, case, budget_s=10.0):
    import oracle
    b = step_bytes(wl)
    # calibrate the per-column cost on a small sample
    cols = max(1, min(wl.N, 8))
    t = time.perf_counter()
    oracle_step_sample(oracle, case, wl, cols)
    per_col = (time.perf_counter() - t) / cols
    cols = int(max(1, min(wl.N, budget_s / 4 / max(per_col, 1e-9))))
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle_step_sample(oracle, case, wl, cols)
        n += 1
        if time.perf_counter() - t0 >= budget_s * 0.5 or n >= 1000:
            break
    dt = time.perf_counter() - t0
    frac = cols / wl.N
    gbs = 2 * b["total"] * frac * n / dt / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} x ({cols} of {wl.N} output columns, all {wl.M} rows, both variants); "
                      f"bytes scaled by the column fraction", "seconds": round(dt, 2)}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    import oracle
    case = make_workload(args.workload)
    b = step_bytes(wl)
    # size each step so that warm-up + K steps take about a minute
    t = time.perf_counter()
    oracle_step_sample(oracle, case, wl, 4)
    per_col = (time.perf_counter() - t) / 4
    cols = int(max(1, min(wl.N, 60.0 / max(args.steps + args.warmup, 1) / max(per_col, 1e-9))))
    for _ in range(args.warmup):
        oracle_step_sample(oracle, case, wl, cols)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step_sample(oracle, case, wl, cols)
    dt = time.perf_counter() - t0
    frac = cols / wl.N
    value = 2 * b["total"] * frac * args.steps / dt / 1e9
    sample = f"each step: {cols} of {wl.N} output columns, all {wl.M} rows, both variants; bytes scaled by the column fraction"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded)",
        "config": {"workload": f"{wl.name}: M={wl.M} K={wl.K} N={wl.N} g={wl.g}" + (f" E={wl.E}" if wl.E > 1 else "")
                   + "; one step = MSD matmul + dequant matmul"},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- profiling modes (--profile)
#
# Not part of the benchmark line: drivers for profilers and per-variant
# timing tables.  Every launch is the library's own.

VARIANT_OPS = {"msd": 0, "dequant": 1, "bf16": 2, "msd2": 3, "msd4": 4}


def _variant_io(torch, w4, name, variant, copies):
    """Device inputs of one workload for one variant (bf16: the same
    distributions encoded as bf16), weights repacked `copies` times."""
    act = "bf16" if variant == "bf16" else "fp16"
    c = make_workload(name, act=act)

    def up(a):
        if act == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(a).cuda()
    x = up(c.x)
    wp = [[w4.repack(torch.from_numpy(p).cuda(), c.K, c.N) for p in c.wp] for _ in range(copies)]
    sc = [up(s) for s in c.scale]
    y = torch.empty((c.M, c.N), dtype=torch.bfloat16 if act == "bf16" else torch.float16, device="cuda")
    op = VARIANT_OPS[variant]
    ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g, E=c.E)
    off = torch.from_numpy(c.offsets).cuda() if c.E > 1 else None

    def call(i):
        wpi = wp[i % copies]
        if c.E > 1:
            w4.w4a16_grouped_matmul(op, x, wpi, sc, off, c.E, c.M, c.K, c.N, c.g, y, ws)
        elif variant in ("msd2", "msd4", "msd"):
            w4.w4a16_msd_matmul_steps({"msd": 3, "msd2": 2, "msd4": 4}[variant], x, wpi[0], sc[0], c.M, c.K, c.N,
                                      c.g, y, ws)
        elif variant == "bf16":
            w4.w4a16_dequant_matmul_bf16(x, wpi[0], sc[0], c.M, c.K, c.N, c.g, y, ws)
        else:
            w4.w4a16_dequant_matmul(x, wpi[0], sc[0], c.M, c.K, c.N, c.g, y, ws)
    return c, call, ws


def _graph_us(torch, fn, reps):
    """Mean device time of `fn` over a CUDA graph of `reps` calls (fn takes
    the call index), between two events on the capture stream."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(reps):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def profile_calls(args):
    """`calls` calls of each variant in turn on the workload, rotating over
    `calls` weight copies; checks the device status word.  For ncu."""
    import torch
    import weight_only_int4_a16w4_b200 as w4
    for v in args.variants.split(","):
        c, call, ws = _variant_io(torch, w4, args.workload, v, args.calls)
        for i in range(args.calls):
            call(i)
        torch.cuda.synchronize()
        if w4.w4a16_read_status(ws) != 0:
            raise SystemExit("device wait timed out")
    print("ok")


def profile_variants(args):
    """A markdown table of us per call for each variant on each workload (a
    CUDA graph of consecutive calls; weights re-read from HBM: copies rotate
    past L2 where one copy would fit)."""
    import torch
    import weight_only_int4_a16w4_b200 as w4
    variants = args.variants.split(",")
    names = args.workloads.split(",")
    print("| workload | " + " | ".join(f"{v} us" for v in variants) + " | " +
          " | ".join(f"{v} TFLOP/s (2MNK)" for v in variants) + " |")
    print("|---|" + "---|" * (2 * len(variants)))
    for name in names:
        wl = get_workload(name)
        b = step_bytes(wl)
        copies = 1 if wl.E > 1 else max(2, int(np.ceil(2.2 * L2_BYTES / (b["w"] + b["scale"]))))
        us = []
        for v in variants:
            c, call, ws = _variant_io(torch, w4, name, v, copies)
            reps = 200 if wl.M * wl.N * wl.K < (1 << 36) else 10
            reps = max(reps, copies)
            us.append(_graph_us(torch, call, reps))
            if w4.w4a16_read_status(ws) != 0:
                raise SystemExit("device status set")
        fl = step_flops(wl)
        print(f"| {name} | " + " | ".join(f"{u:.2f}" for u in us) + " | " +
              " | ".join(f"{fl / u / 1e6:.1f}" for u in us) + " |")


def profile_routing(args):
    """Routing prep of the grouped form at the grouped workload's shape: the
    expert grouping, the row gather, the gate-weighted un-permute, and the
    whole routed matmul next to the grouped matmul on pre-sorted rows (both
    variants), per topk.  Router ids uniform over the experts, gate weights
    uniform in [0, 1), seeded."""
    import torch
    import weight_only_int4_a16w4_b200 as w4
    from inputs import draw_scale, draw_w, draw_x, pack_int4
    wl = get_workload("moe_e8")
    T, E, K, N, g = wl.M, wl.E, wl.K, wl.N, wl.g
    rng = np.random.Generator(np.random.PCG64(20260))
    x = torch.from_numpy(draw_x(rng, T, K)).cuda()
    wp = [w4.repack(torch.from_numpy(pack_int4(draw_w(rng, K, N))).cuda(), K, N) for _ in range(E)]
    sc = [torch.from_numpy(draw_scale(rng, K // g, N)).cuda() for _ in range(E)]
    print(f"routing prep, T={T} E={E} K={K} N={N} g={g} (us per call)")
    print("| topk | align | gather | combine | routed MSD | grouped MSD | routed dequant | grouped dequant |")
    print("|---|---|---|---|---|---|---|---|")
    for topk in [int(t) for t in args.topk.split(",")]:
        rows = T * topk
        ids = torch.from_numpy(rng.integers(0, E, (T, topk)).astype(np.int32)).cuda()
        wts = torch.from_numpy(rng.uniform(0, 1, (T, topk)).astype(np.float32)).cuda()
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        st = torch.empty(rows, dtype=torch.int32, device="cuda")
        inv = torch.empty(rows, dtype=torch.int32, device="cuda")
        hdr = torch.zeros(256, dtype=torch.uint8, device="cuda")
        xs = torch.empty((rows, K), dtype=torch.float16, device="cuda")
        ys = torch.zeros((rows, N), dtype=torch.float16, device="cuda")
        y = torch.empty((T, N), dtype=torch.float16, device="cuda")
        t_align = _graph_us(torch, lambda i: w4.w4a16_moe_align(ids, T, topk, E, offsets, st, inv, hdr), 50)
        t_gather = _graph_us(torch, lambda i: w4.w4a16_moe_gather(x, st, rows, K, xs), 20)
        t_comb = _graph_us(torch, lambda i: w4.w4a16_moe_combine(ys, inv, wts, T, topk, N, y), 20)
        res = []
        for op in (w4.OP_MSD, w4.OP_DEQUANT):
            ws = torch.zeros(w4.w4a16_moe_workspace_size(op, T, topk, K, N, g, E), dtype=torch.uint8, device="cuda")
            gws = w4.alloc_workspace(op, rows, K, N, g, E=E)
            res.append(_graph_us(torch, lambda i: w4.w4a16_moe_matmul(op, x, ids, wts, wp, sc, E, T, topk, K, N, g,
                                                                      y, ws), 5))
            res.append(_graph_us(torch, lambda i: w4.w4a16_grouped_matmul(op, xs, wp, sc, offsets, E, rows, K, N, g,
                                                                          ys, gws), 5))
            if w4.w4a16_read_status(ws) or w4.w4a16_read_status(gws):
                raise SystemExit("device status set")
        print(f"| {topk} | {t_align:.2f} | {t_gather:.2f} | {t_comb:.2f} | {res[0]:.1f} | {res[1]:.1f} | "
              f"{res[2]:.1f} | {res[3]:.1f} |")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_m1", choices=[w.name for w in WORKLOADS])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["calls", "variants", "routing"],
                    help="profiler driver / timing table instead of the benchmark line")
    ap.add_argument("--calls", type=int, default=4, help="--profile calls: calls per variant")
    ap.add_argument("--variants", default="msd,dequant",
                    help="--profile calls|variants: comma list of msd, dequant, bf16, msd2, msd4")
    ap.add_argument("--workloads", default="decode_m1,decode_m16,prefill,moe_e8",
                    help="--profile variants: comma list of workloads")
    ap.add_argument("--topk", default="1,2", help="--profile routing: comma list of topk")
    args = ap.parse_args(argv)
    if args.profile == "calls":
        profile_calls(args)
        return
    if args.profile == "variants":
        profile_variants(args)
        return
    if args.profile == "routing":
        profile_routing(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    wl = get_workload(args.workload)
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    run_gpu(args, wl, rank, world, local)


if __name__ == "__main__":
    main()
