"""Benchmark: SparseConv2D fwd+bwd step on B200 through the svconv C ABI.

One step = the whole hot path on one batch of pruned tokens, the small-channel
adapter convolution workload (T=384 token-frames, 16x16 patch grid, top-77
blob-saliency keep per frame, C_in=C_out=64, bf16 with fp32 accumulation):
    neighbour-index build -> forward -> data gradient -> weight/bias gradient
(and, with --gpus N > 1, an NCCL all-reduce of dW/db: data-parallel weak scaling,
every rank owning its own batch of frames).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

Timing: each step is replayed from a CUDA graph, the 126 MB L2 is flushed by a
256 MiB write between steps (the workload's 8.7 MB would otherwise stay in L2),
and only the step is inside the CUDA-event region.  The roofline object is for
the step's slowest kernel, timed by events around each kernel on the launching
stream in a second pass.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SparseConv2D kept-tokens/sec (fwd, fwd+bwd) and % of roofline on 1 B200"
UNIT = "kept-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_PEAKS["hbm_gbs"], "bf16_tflops": FALLBACK_PEAKS["bf16_tflops"],
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def algorithmic_work(n, T, Cin, Cout):
    """Per-launch algorithmic bytes and flops (unique data touched once)."""
    bf = 2
    nbr = 36 * n
    w_bytes = 9 * Cin * Cout * bf
    return {
        "build_index": {"bytes": 12 * n + 4 * (T + 1) + nbr, "flops": 0},
        "fwd": {"bytes": n * Cin * bf + n * Cout * bf + nbr + w_bytes, "flops": 2 * n * 9 * Cin * Cout},
        "bwd_data": {"bytes": n * Cout * bf + n * Cin * bf + nbr + w_bytes, "flops": 2 * n * 9 * Cin * Cout},
        "bwd_weight": {"bytes": n * Cout * bf + n * Cin * bf + nbr + 4 * (9 * Cin * Cout + Cout),
                       "flops": 2 * n * 9 * Cin * Cout},
    }


def roofline_entry(name, work, ms, peaks):
    sec = ms * 1e-3
    t_hbm = work["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = work["flops"] / (peaks["bf16_tflops"] * 1e12) if work["flops"] else 0.0
    if t_tc > t_hbm:
        achieved = work["flops"] / sec / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"]}
    achieved = work["bytes"] / sec / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"]}


def kernel_traffic(workload_key, kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    ent = d.get(f"{workload_key}/{kernel_key}")
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != ent["source_sha"]:
        return None
    return ent["dram_bytes_per_launch"]


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = [r.split(", ") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        if not rows:
            return None
        try:
            sm = [float(r[1]) for r in rows]
            mx = float(rows[0][2])
        except (ValueError, IndexError):
            return None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, nm in enumerate(names):
                if len(r) > 5 + i and r[5 + i].strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(rows)}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n_gpus > 1 or world > 1:
        if world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch with torch.distributed.run")
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, local, world


WORKLOADS = {
    # name: (generator, base seed)
    "small_c": ("small_c_bf16", 1),
    "large_c_fwd": ("large_c_fwd_bf16", 2),
    "large_c_bwd": ("large_c_bwd_bf16", 3),
    "adapter": ("adapter_bf16", 4),
}
WORKLOAD = "small_c"


def make_inputs(seed_offset=0, workload=None):
    from sparse_convolution_pruned_b200 import workloads as wl
    gen, seed = WORKLOADS[workload or WORKLOAD]
    return getattr(wl, gen)(seed=seed + seed_offset)


# ----------------------------------------------------------------------------- reference arm (CPU oracle)
def cpu_oracle_step(w, frames):
    """One oracle step on the first `frames` frames (frames are independent)."""
    import oracle
    r1 = int(w.frame_off[frames])
    coords = w.coords[:r1]
    off = w.frame_off[: frames + 1]
    t0 = time.perf_counter()
    nbr, _, st = oracle.build_index(coords, off, frames, w.H, w.W, want_map=False)
    oracle.fwd(w.X[:r1], nbr, w.Wt, w.bias)
    oracle.bwd_data(w.dY[:r1], nbr, w.Wt)
    oracle.bwd_weight(w.dY[:r1], w.X[:r1], nbr)
    return time.perf_counter() - t0, r1


def oracle_frames(w, mac_budget):
    """How many leading frames of the workload fit a budget of oracle multiply-adds."""
    per_token = 3 * 9 * w.Cin * w.Cout  # fwd + bwd_data + bwd_weight
    per_frame = per_token * w.n / max(1, w.T)
    return int(max(1, min(w.T, mac_budget // max(1, per_frame))))


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = make_inputs(0)
    if WORKLOAD == "adapter":
        return run_reference_adapter(args, w)
    # each step: the first frames of the workload, about 4e9 multiply-adds (a few seconds)
    frames = oracle_frames(w, 4e9)
    for _ in range(args.warmup):
        cpu_oracle_step(w, frames)
    tot, toks = 0.0, 0
    for _ in range(args.steps):
        dt, r = cpu_oracle_step(w, frames)
        tot += dt
        toks += r
    value = toks / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n_kept": w.n, "sample": f"first {frames} of {w.T} frames per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
                         "sample": f"index+fwd+bwd_data+bwd_weight on the first {frames} frames "
                                   f"({int(w.frame_off[frames])} tokens) per step; 1 core used of "
                                   f"{os.cpu_count()}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def run_reference_adapter(args, w):
    """Oracle index build + adapter forward on the first 8 frames of the long video per step."""
    import oracle
    frames = 8
    r1 = int(w.frame_off[frames])

    def one():
        t0 = time.perf_counter()
        sub_n, _, _ = oracle.build_index(w.coords[:r1], w.frame_off[: frames + 1], frames, w.H, w.W,
                                         want_map=False)
        oracle.adapter_fwd(w.X[:r1], sub_n, 0, r1, w.Wd, w.Wc, w.Wu)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        one()
    tot = sum(one() for _ in range(args.steps))
    value = r1 * args.steps / tot
    sample = (f"index build + adapter forward on the first {frames} of {w.T} frames ({r1} tokens) per step; "
              f"single-threaded C, fp64; 1 core used of {os.cpu_count()}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n_kept": w.n, "sample": f"first {frames} of {w.T} frames per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))
    return 0


# ----------------------------------------------------------------------------- B200 arm
def run_b200(args):
    import torch
    import torch.distributed as dist

    from sparse_convolution_pruned_b200 import svconv as sv
    from sparse_convolution_pruned_b200.data_parallel import allreduce_grads

    rank, local, world = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    w = make_inputs(rank)  # weak scaling: each rank owns its own batch of frames
    n, T, Cin, Cout = w.n, w.T, w.Cin, w.Cout

    # pinned host inputs (the e2e leg copies these every step)
    h_coords = torch.from_numpy(w.coords).pin_memory()
    h_off = torch.from_numpy(w.frame_off).pin_memory()
    h_X = torch.from_numpy(w.X).to(torch.bfloat16).pin_memory()
    h_W = torch.from_numpy(w.Wt).to(torch.bfloat16).pin_memory()
    h_dY = torch.from_numpy(w.dY).to(torch.bfloat16).pin_memory()
    bias = torch.from_numpy(w.bias).to(dev) if w.bias is not None else None

    coords = h_coords.to(dev)
    off = h_off.to(dev)
    X = h_X.to(dev)
    Wt = h_W.to(dev)
    dY = h_dY.to(dev)
    nbr = torch.empty((n, 9), dtype=torch.int32, device=dev)
    Y = torch.empty((n, Cout), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((n, Cin), dtype=torch.bfloat16, device=dev)
    grads = torch.empty((Cout * 9 * Cin + Cout,), dtype=torch.float32, device=dev)
    dW = grads[: Cout * 9 * Cin].view(Cout, 9, Cin)
    db = grads[Cout * 9 * Cin:]
    ws = torch.empty((max(16, sv.svconv_bwd_weight_workspace_size(sv.BF16, n, Cin, Cout),
                          sv.svconv_bwd_workspace_size(sv.BF16, n, Cin, Cout)),), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty((FLUSH_BYTES,), dtype=torch.uint8, device=dev)

    stream = torch.cuda.Stream(device=dev)

    def step_kernels():
        sv.svconv_build_index(coords, off, T, w.H, w.W, nbr=nbr, status=status)
        sv.svconv_fwd(X, nbr, Wt, bias, Y=Y)
        # backward: data and weight gradients in one call (side by side at 64 channels)
        sv.svconv_bwd(dY, X, nbr, Wt, dX=dX, dW=dW, db=db, workspace=ws)

    launches_per_step = 5  # index, fwd, bwd_data, wgrad partials, wgrad reduce

    with torch.cuda.stream(stream):
        step_kernels()  # first call outside capture: caches device info and kernel attributes
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            step_kernels()
        g_fwd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_fwd, stream=stream, capture_error_mode="relaxed"):
            sv.svconv_build_index(coords, off, T, w.H, w.W, nbr=nbr, status=status)
            sv.svconv_fwd(X, nbr, Wt, bias, Y=Y)
    torch.cuda.synchronize()

    def one_step():
        g.replay()
        if world > 1:
            allreduce_grads(grads)

    def timed_loop(fn, steps, warmup, flush_l2=True):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                if flush_l2:
                    flush.zero_()
                fn()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            evs = []
            for _ in range(steps):
                if flush_l2:
                    flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                evs.append((a, b))
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    with ClockSampler(local) as clk:
        total_ms = timed_loop(one_step, args.steps, args.warmup)
    clocks = clk.summary()
    fwd_ms = timed_loop(g_fwd.replay, args.steps, args.warmup)
    # the same step with the workload left in L2 between steps (reported beside the flushed number)
    hot_ms = timed_loop(one_step, args.steps, args.warmup, flush_l2=False)

    t = torch.tensor([total_ms, fwd_ms, hot_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms, fwd_ms, hot_ms = float(t[0]), float(t[1]), float(t[2])

    # per-kernel durations (events between the library calls on the launching stream)
    names = ["build_index", "fwd", "bwd_data", "bwd_weight"]
    calls = [lambda: sv.svconv_build_index(coords, off, T, w.H, w.W, nbr=nbr, status=status),
             lambda: sv.svconv_fwd(X, nbr, Wt, bias, Y=Y),
             lambda: sv.svconv_bwd_data(dY, nbr, Wt, dX=dX),
             lambda: sv.svconv_bwd_weight(dY, X, nbr, dW=dW, db=db, workspace=ws)]
    per = {k: 0.0 for k in names}
    kreps = max(args.steps, 10)
    with torch.cuda.stream(stream):
        for _ in range(3):
            flush.zero_()
            for c in calls:
                c()
        torch.cuda.synchronize()
        recs = []
        for _ in range(kreps):
            # four flush passes (~160 us of GPU work) let the host enqueue every call
            # and event below before the first kernel starts: no launch gaps inside
            for _ in range(4):
                flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
            ev[0].record(stream)
            for i, c in enumerate(calls):
                c()
                ev[i + 1].record(stream)
            recs.append(ev)
        torch.cuda.synchronize()
    for ev in recs:
        for i, k in enumerate(names):
            per[k] += ev[i].elapsed_time(ev[i + 1]) / kreps

    # end-to-end through the public API with host buffers
    h_Y = torch.empty((n, Cout), dtype=torch.bfloat16).pin_memory()
    h_dX = torch.empty((n, Cin), dtype=torch.bfloat16).pin_memory()
    h_grads = torch.empty_like(grads, device="cpu").pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (h_coords, h_off, h_X, h_W, h_dY))
    d2h = sum(x.numel() * x.element_size() for x in (h_Y, h_dX, h_grads))

    def e2e_step():
        coords.copy_(h_coords, non_blocking=True)
        off.copy_(h_off, non_blocking=True)
        X.copy_(h_X, non_blocking=True)
        Wt.copy_(h_W, non_blocking=True)
        dY.copy_(h_dY, non_blocking=True)
        step_kernels()
        if world > 1:
            allreduce_grads(grads)
        h_Y.copy_(Y, non_blocking=True)
        h_dX.copy_(dX, non_blocking=True)
        h_grads.copy_(grads, non_blocking=True)

    e2e_ms = timed_loop(e2e_step, args.steps, args.warmup)
    t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_ms = float(t[0])

    torch.cuda.synchronize()
    st = int(status.item())
    err = sv.svconv_read_error_word()
    if st or err:
        raise SystemExit(f"device status {st} / library error word {err}: results invalid")

    # CPU baseline: the oracle as it stands, rank 0 at N=1 only, on a bounded sample
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        # about 1.6e10 multiply-adds of oracle work (10-15 s on one core)
        frames = oracle_frames(w, 1.6e10)
        macs = 3 * 9 * Cin * Cout * int(w.frame_off[frames])
        reps = int(max(1, round(1.6e10 / macs)))
        dt, toks = 0.0, 0
        for _ in range(reps):
            d, r = cpu_oracle_step(w, frames)
            dt += d
            toks += r
        cpu = {"value": toks / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
               "sample": f"index+fwd+bwd_data+bwd_weight on the first {frames} of {w.T} frames "
                         f"({int(w.frame_off[frames])} tokens), {reps} time(s); single-threaded C, fp64; "
                         f"1 core used of {os.cpu_count()}"}

    if rank == 0:
        peaks = load_peaks()
        work = algorithmic_work(n, T, Cin, Cout)
        if bias is not None:
            work["fwd"]["bytes"] += 4 * Cout
        kern = {k: dict(ms=per[k], **roofline_entry(k, work[k], per[k], peaks)) for k in names}
        top = max(names, key=lambda k: per[k])
        roof = dict(kern[top])
        roof.pop("ms")
        roof["kernel"] = top
        roof["traffic"] = kernel_traffic(args.workload, top)
        roof["peak_source"] = peaks["source"]
        tokens = n * world
        line = {
            "metric": METRIC, "value": tokens * args.steps / (total_ms * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "n_kept_per_gpu": n, "T": T, "H": w.H, "W": w.W, "C_in": Cin,
                       "C_out": Cout, "step": "build_index+fwd+bwd(data, weight: one svconv_bwd call)" +
                                               ("+allreduce(dW,db)" if world > 1 else ""),
                       "l2": f"flushed by a {FLUSH_BYTES >> 20} MiB write between timed steps",
                       "graph": "step replayed from a CUDA graph", "parallelism": f"dp{world}"},
            "fwd": {"value": tokens * args.steps / (fwd_ms * 1e-3), "unit": UNIT,
                    "ms_per_step": fwd_ms / args.steps, "step": "build_index+fwd"},
            "l2_hot": {"value": tokens * args.steps / (hot_ms * 1e-3), "unit": UNIT,
                       "ms_per_step": hot_ms / args.steps, "note": "same step, no L2 flush between steps"},
            "roofline": roof,
            "kernels": kern,
            "e2e": {"value": tokens * args.steps / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        del g, g_fwd
        dist.destroy_process_group()
    return 0


def host_cpu():
    """CPU model and logical core count of this host (for the CPU-baseline record)."""
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


# ----------------------------------------------------------------------------- adapter workload (a5)
def run_adapter(args):
    """Long-video bottleneck adapter: one step = index build + chunked adapter forward.

    X (n x 1024 bf16, 579 MB at the full size) is read and written in place each step,
    far larger than L2, so no flush is needed between steps.
    """
    import torch
    import torch.distributed as dist

    from sparse_convolution_pruned_b200 import svconv as sv

    rank, local, world = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    w = make_inputs(rank)
    n, T, D, R = w.n, w.T, w.D, w.R
    chunk_T = args.adapter_chunk_frames  # frames per chunk (device memory grows with it; cap 1 GB)
    offs = w.frame_off.astype(np.int64)
    max_rows = int(max(offs[min(t + chunk_T, T)] - offs[t] for t in range(0, T, chunk_T)))

    h_coords = torch.from_numpy(w.coords).pin_memory()
    h_off = torch.from_numpy(w.frame_off).pin_memory()
    h_X = torch.from_numpy(w.X).to(torch.bfloat16).pin_memory()
    torch.cuda.reset_peak_memory_stats(dev)
    coords = h_coords.to(dev)
    off = h_off.to(dev)
    X = h_X.to(dev)
    Wd = torch.from_numpy(w.Wd).to(torch.bfloat16).to(dev)
    Wc = torch.from_numpy(w.Wc).to(torch.bfloat16).to(dev)
    Wu = torch.from_numpy(w.Wu).to(torch.bfloat16).to(dev)
    nbr = torch.empty((n, 9), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty((max(16, sv.svconv_adapter_workspace_size(R, max_rows)),), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def index():
        sv.svconv_build_index(coords, off, T, w.H, w.W, nbr=nbr, status=status)

    def adapter():
        sv.svconv_adapter_fwd(X, nbr, off, T, Wd, Wc, Wu, chunk_T=chunk_T, max_chunk_rows=max_rows,
                              workspace=ws, status=status)

    n_chunks = (T + chunk_T - 1) // chunk_T
    launches_per_step = 1 + 3 * n_chunks  # index; per chunk: down GEMM, conv, up GEMM

    def timed(fn, steps, warmup):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            evs = []
            for _ in range(steps):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                evs.append((a, b))
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    def step():
        index()
        adapter()

    with torch.cuda.stream(stream):
        step()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            step()
        g_ad = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_ad, stream=stream, capture_error_mode="relaxed"):
            adapter()
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated(dev)

    with ClockSampler(local) as clk:
        total_ms = timed(g.replay, args.steps, args.warmup)
    clocks = clk.summary()
    ad_ms = timed(g_ad.replay, args.steps, args.warmup) / args.steps
    idx_ms = timed(index, args.steps, args.warmup) / args.steps

    # end to end: the video's coordinates and features in from pinned host memory, the
    # updated features back out
    h_out = torch.empty_like(h_X).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (h_coords, h_off, h_X))
    d2h = h_out.numel() * h_out.element_size()

    def e2e():
        coords.copy_(h_coords, non_blocking=True)
        off.copy_(h_off, non_blocking=True)
        X.copy_(h_X, non_blocking=True)
        step()
        h_out.copy_(X, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    e2e_ms = timed(e2e, e2e_steps, 3)
    t = torch.tensor([total_ms, e2e_ms, ad_ms, idx_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms, e2e_ms, ad_ms, idx_ms = (float(v) for v in t)
    torch.cuda.synchronize()
    st = int(status.item())
    err = sv.svconv_read_error_word()
    if st or err:
        raise SystemExit(f"device status {st} / library error word {err}: results invalid")

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        # whole frames are independent: the oracle runs the first `frames` frames
        frames = 8
        r1 = int(w.frame_off[frames])
        t0 = time.perf_counter()
        sub_n, _, _ = oracle.build_index(w.coords[:r1], w.frame_off[: frames + 1], frames, w.H, w.W,
                                         want_map=False)
        oracle.adapter_fwd(w.X[:r1], sub_n, 0, r1, w.Wd, w.Wc, w.Wu)
        dt = time.perf_counter() - t0
        t1 = time.perf_counter()
        oracle.build_index(w.coords, w.frame_off, T, w.H, w.W, want_map=True)
        idx_cpu_ms = 1e3 * (time.perf_counter() - t1)
        cpu = {"value": r1 / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
               "sample": f"index build + adapter forward on the first {frames} of {T} frames ({r1} tokens); "
                         f"single-threaded C, fp64; 1 core used of {os.cpu_count()}",
               "index_build_full_ms": idx_cpu_ms}

    if rank == 0:
        peaks = load_peaks()
        flops = 2 * n * (D * R + 9 * R * R + R * D)
        ad_work = {"bytes": 2 * n * D * 2 + 36 * n + 2 * (2 * D * R + 9 * R * R), "flops": flops}
        roof = roofline_entry("adapter_fwd", ad_work, ad_ms, peaks)
        roof["kernel"] = f"adapter_fwd ({3 * n_chunks} tcgen05 GEMM launches, timed together)"
        roof["traffic"] = kernel_traffic(args.workload, "adapter_fwd")  # DRAM bytes of the 18 launches
        roof["peak_source"] = peaks["source"]
        idx_work = algorithmic_work(n, T, R, R)["build_index"]
        tokens = n * world
        line = {
            "metric": METRIC, "value": tokens * args.steps / (total_ms * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "n_kept_per_gpu": n, "T": T, "H": w.H, "W": w.W, "D": D, "R": R,
                       "chunk_T": chunk_T, "step": "build_index+adapter_fwd (in place)",
                       "l2": "inputs larger than L2 (X read and written in place each step); no flush",
                       "graph": "step replayed from a CUDA graph", "parallelism": f"dp{world}",
                       "peak_device_bytes": peak},
            "roofline": roof,
            "kernels": {"adapter_fwd": dict(ms=ad_ms, **roofline_entry("adapter_fwd", ad_work, ad_ms, peaks)),
                        "build_index": dict(ms=idx_ms, **roofline_entry("build_index", idx_work, idx_ms, peaks))},
            "e2e": {"value": tokens * e2e_steps / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        del g, g_ad
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--adapter-chunk-frames", type=int, default=1024,
                    help="adapter workload: token frames per chunk of the chunked adapter forward "
                         "(1024: 3 chunks, ~660 MiB peak; 512: 6 chunks, ~610 MiB, 17%% slower)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="small_c",
                    help="small_c (default: the headline configuration), large_c_fwd, large_c_bwd, adapter")
    args = ap.parse_args()
    global WORKLOAD
    WORKLOAD = args.workload
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "adapter":
        return run_adapter(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
