"""Benchmark: SparseConv2D on B200 through the svconv C ABI, every workload in one run.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--no-cpu-baseline] [--sustained-s S]

Workloads (the five SparseConv2D configurations, synthetic seeded inputs):
  tiny_f32     T=4, 8x8 grid, 32 kept per frame, C=16, fp32 (fwd + bwd)
  small_c      T=384, 16x16, top-77 blob-saliency keep, C=64, bf16 (fwd + bwd)
  large_c_fwd  T=384, 16x16, keep 50%, C=256, bf16 + fp32 bias (fwd)
  large_c_bwd  T=384, 16x16, keep U(0.2, 0.8) per frame, C=256, bf16 (fwd + bwd)
  adapter      T=3072 token frames, 16x16, keep 36%, Linear 1024->256, SparseConv 256->256,
               GELU, Linear 256->1024 + residual, chunked over frames (fwd)

One step is one pass of the workload's whole path over its batch: neighbour-index build ->
forward [-> data gradient -> weight / bias gradient] (adapter: index build -> chunked adapter
forward).  The headline (top-level ``value``) is the largest fwd+bwd configuration that fits
one GPU, ``large_c_bwd``; with N = 1 every workload is also reported under ``configs`` with its
own roofline (dominant kernel), per-kernel times, end-to-end leg, CPU-oracle baseline and a
sustained leg (>= 1 s of back-to-back graph replays with its own clock samples).  With N > 1
(torchrun, NCCL) each rank runs its own batch of the headline workload (weak scaling) and the
weight / bias gradients are all-reduced.

Timing: steps are replayed from CUDA graphs and timed with CUDA events on the launching
stream; the 126 MB L2 is flushed by a 256 MiB write between timed steps (outside the events)
for the conv workloads, whose working sets fit in L2; the adapter's in-place X (579 MB) is
larger than L2 and is not flushed.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 flops (FMA) x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FLUSH_BYTES = 256 << 20

# name: (generator in workloads.py, base seed, step kind, compute dtype)
WORKLOADS = {
    "tiny_f32": ("tiny_f32", 0, "fwd+bwd", "f32"),
    "small_c": ("small_c_bf16", 1, "fwd+bwd", "bf16"),
    "large_c_fwd": ("large_c_fwd_bf16", 2, "fwd", "bf16"),
    "large_c_fwd_e4m3": ("large_c_fwd_e4m3", 2, "fwd", "e4m3"),
    "large_c_bwd": ("large_c_bwd_bf16", 3, "fwd+bwd", "bf16"),
    "adapter": ("adapter_bf16", 4, "adapter", "bf16"),
}
ORDER = ["tiny_f32", "small_c", "large_c_fwd", "large_c_fwd_e4m3", "large_c_bwd", "adapter"]
HEADLINE = "large_c_bwd"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def make_inputs(key, seed_offset=0):
    from sparse_convolution_pruned_b200 import workloads as wl
    gen, seed, _, _ = WORKLOADS[key]
    return getattr(wl, gen)(seed=seed + seed_offset)


# ----------------------------------------------------------------------------- algorithmic work
def conv_work(n, T, Cin, Cout, elem, bias, elem_out=None):
    """Per-launch algorithmic bytes and flops: unique data touched once (features, the
    neighbour table at 36 B per token, weights, bias, fp32 weight gradients).  elem: bytes
    per input / weight element; elem_out: bytes per forward output element (default elem)."""
    eo = elem if elem_out is None else elem_out
    nbr = 36 * n
    w_bytes = 9 * Cin * Cout * elem
    fl = 2 * n * 9 * Cin * Cout
    return {
        "build_index": {"bytes": 12 * n + 4 * (T + 1) + nbr, "flops": 0},
        "fwd": {"bytes": n * (Cin * elem + Cout * eo) + nbr + w_bytes + (4 * Cout if bias else 0), "flops": fl},
        "bwd_data": {"bytes": n * (Cin + Cout) * elem + nbr + w_bytes, "flops": fl},
        "bwd_weight": {"bytes": n * (Cin + Cout) * elem + nbr + 4 * (9 * Cin * Cout + Cout), "flops": fl},
    }


def adapter_work(n, D, R):
    return {"bytes": 2 * n * D * 2 + 36 * n + 2 * (2 * D * R + 9 * R * R),
            "flops": 2 * n * (D * R + 9 * R * R + R * D)}


def flop_peak(peaks, alu=False, fp8=False):
    """fp32 CUDA-core peak (alu), e4m3 tensor peak (measured bf16 x the nominal 4.5 / 2.25
    ratio), or the measured bf16 tensor peak."""
    if alu:
        return FP32_ALU_TFLOPS
    return peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)


def floor_seconds(work, peaks, alu=False, fp8=False):
    t_mem = work["bytes"] / (peaks["hbm_gbs"] * 1e9)
    peak_fl = flop_peak(peaks, alu, fp8)
    t_fl = work["flops"] / (peak_fl * 1e12) if work["flops"] else 0.0
    return max(t_mem, t_fl)


def roofline_entry(work, ms, peaks, alu=False, fp8=False):
    """The larger of the byte floor (HBM) and the flop floor (bf16 or e4m3 tensor, or fp32 ALU)."""
    sec = ms * 1e-3
    t_mem = work["bytes"] / (peaks["hbm_gbs"] * 1e9)
    peak_fl = flop_peak(peaks, alu, fp8)
    t_fl = work["flops"] / (peak_fl * 1e12) if work["flops"] else 0.0
    if t_fl > t_mem:
        achieved = work["flops"] / sec / 1e12
        note = ("fp32 CUDA-core peak derived from 148 SMs x 128 lanes x FMA x 1.965 GHz" if alu else
                "e4m3 dense = measured bf16 burst x 2 (nominal 4.5 / 2.25 PFLOP/s)" if fp8 else
                "bf16 dense, burst (kernel timed alone)")
        return {"bound": "alu" if alu else "tensor", "achieved": achieved, "peak": peak_fl, "unit": "TFLOP/s",
                "frac": achieved / peak_fl, "algorithmic": work["flops"], "peak_note": note}
    achieved = work["bytes"] / sec / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "algorithmic": work["bytes"]}


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


# ----------------------------------------------------------------------------- clocks
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
            pw = [float(r[3]) for r in rows]
        except (ValueError, IndexError):
            return None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, nm in enumerate(names):
                if len(r) > 5 + i and r[5 + i].strip().lower() == "active":
                    reasons.add(nm)
        # samples under load: power above the idle level (the first sample is taken before the load)
        loaded = [s for s, p in zip(sm, pw) if p > pw[0] + 30.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(loaded) if loaded is not sm else 0,
                "power_w_max": max(pw)}


# ----------------------------------------------------------------------------- process group
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


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_conv_step(w, frames, with_bwd):
    """One oracle step on the first `frames` frames (frames are independent)."""
    import oracle
    r1 = int(w.frame_off[frames])
    t0 = time.perf_counter()
    nbr, _, _ = oracle.build_index(w.coords[:r1], w.frame_off[: frames + 1], frames, w.H, w.W, want_map=False)
    oracle.fwd(w.X[:r1], nbr, w.Wt, w.bias)
    if with_bwd:
        oracle.bwd_data(w.dY[:r1], nbr, w.Wt)
        oracle.bwd_weight(w.dY[:r1], w.X[:r1], nbr)
    return time.perf_counter() - t0, r1


# the single-threaded oracle does about 1.2e9 multiply-adds per second
ORACLE_MACS_PER_S = 1.2e9


def oracle_conv_frames(w, seconds, with_bwd):
    """Leading frames whose oracle step takes about `seconds` (at least one frame)."""
    per_token = (3 if with_bwd else 1) * 9 * w.Cin * w.Cout
    per_frame = per_token * w.n / max(1, w.T)
    return int(max(1, min(w.T, seconds * ORACLE_MACS_PER_S // max(1, per_frame))))


def cpu_baseline_conv(w, with_bwd, seconds):
    import oracle
    oracle.build()
    frames = oracle_conv_frames(w, seconds, with_bwd)
    r = int(w.frame_off[frames])
    macs = (3 if with_bwd else 1) * 9 * w.Cin * w.Cout * r
    reps = int(max(1, round(seconds * ORACLE_MACS_PER_S / max(1, macs))))
    dt, toks = 0.0, 0
    for _ in range(reps):
        d, rr = oracle_conv_step(w, frames, with_bwd)
        dt += d
        toks += rr
    what = "index+fwd+bwd_data+bwd_weight" if with_bwd else "index+fwd"
    return {"value": toks / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
            "sample": f"{what} on the first {frames} of {w.T} frames ({r} tokens), {reps} time(s); "
                      f"frames are independent, so the rate is the workload's; single-threaded C, fp64; "
                      f"1 core used of {os.cpu_count()}"}


def oracle_adapter_step(w, frames):
    import oracle
    r1 = int(w.frame_off[frames])
    t0 = time.perf_counter()
    sub_n, _, _ = oracle.build_index(w.coords[:r1], w.frame_off[: frames + 1], frames, w.H, w.W, want_map=False)
    oracle.adapter_fwd(w.X[:r1], sub_n, 0, r1, w.Wd, w.Wc, w.Wu)
    return time.perf_counter() - t0, r1


def cpu_baseline_adapter(w, seconds):
    import oracle
    oracle.build()
    per_frame = (w.D * w.R * 2 + 9 * w.R * w.R) * w.n / w.T
    frames = int(max(1, min(w.T, seconds * ORACLE_MACS_PER_S // per_frame)))
    dt, r1 = oracle_adapter_step(w, frames)
    t1 = time.perf_counter()
    oracle.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=True)
    idx_ms = 1e3 * (time.perf_counter() - t1)
    return {"value": r1 / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
            "sample": f"index build + adapter forward on the first {frames} of {w.T} frames ({r1} tokens); "
                      f"frames are independent; single-threaded C, fp64; 1 core used of {os.cpu_count()}",
            "index_build_full_ms": idx_ms}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle on the host cores, on the headline workload, each step a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    key = args.workload or HEADLINE
    w = make_inputs(key)
    kind = WORKLOADS[key][2]
    # whole run (warm-up + timed steps) within about two minutes of CPU time
    per_step_s = max(0.05, min(3.0, 120.0 / (args.steps + args.warmup)))
    if kind == "adapter":
        per_frame = (w.D * w.R * 2 + 9 * w.R * w.R) * w.n / w.T
        frames = int(max(1, min(w.T, per_step_s * ORACLE_MACS_PER_S // per_frame)))

        def one():
            return oracle_adapter_step(w, frames)
    else:
        with_bwd = kind == "fwd+bwd"
        frames = oracle_conv_frames(w, per_step_s, with_bwd)

        def one():
            return oracle_conv_step(w, frames, with_bwd)
    for _ in range(args.warmup):
        one()
    tot, toks = 0.0, 0
    for _ in range(args.steps):
        dt, r = one()
        tot += dt
        toks += r
    value = toks / tot
    sample = f"first {frames} of {w.T} frames ({int(w.frame_off[frames])} tokens) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n_kept": w.n, "step": kind, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_cpu(),
                         "sample": f"{kind} step of the oracle on the {sample}; frames are independent; "
                                   f"single-threaded C, fp64; 1 core used of {os.cpu_count()}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- GPU timing helpers
class Ctx:
    """Per-process GPU state shared by the workload legs."""

    def __init__(self, args, rank, local, world):
        import torch
        self.args, self.rank, self.local, self.world = args, rank, local, world
        self.dev = torch.device("cuda", local)
        self.stream = torch.cuda.Stream(device=self.dev)
        self.flush = torch.empty((FLUSH_BYTES,), dtype=torch.uint8, device=self.dev)
        self.peaks = load_peaks()

    def timed(self, fn, steps, warmup, flush_l2=True):
        """Sum of per-step CUDA-event times on the launching stream (barrier + synchronize on
        both sides; the L2 flush, when asked for, runs before each step outside the events)."""
        import torch
        import torch.distributed as dist
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                if flush_l2:
                    self.flush.zero_()
                fn()
            torch.cuda.synchronize()
            if self.world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            evs = []
            for _ in range(steps):
                if flush_l2:
                    self.flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(self.stream)
                fn()
                b.record(self.stream)
                evs.append((a, b))
            torch.cuda.synchronize()
            if self.world > 1:
                dist.barrier()
            torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    def max_over_ranks(self, *vals):
        import torch
        import torch.distributed as dist
        if self.world == 1:
            return vals
        t = torch.tensor(vals, dtype=torch.float64, device=self.dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return tuple(float(v) for v in t)

    def per_kernel(self, calls, reps):
        """Average event time of each call, queued behind ~160 us of flush work so that the host
        has enqueued every call and event before the first kernel starts (no launch gaps)."""
        import torch
        with torch.cuda.stream(self.stream):
            for _ in range(3):
                self.flush.zero_()
                for _, c in calls:
                    c()
            torch.cuda.synchronize()
            recs = []
            for _ in range(reps):
                for _ in range(4):
                    self.flush.zero_()
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
                ev[0].record(self.stream)
                for i, (_, c) in enumerate(calls):
                    c()
                    ev[i + 1].record(self.stream)
                recs.append(ev)
            torch.cuda.synchronize()
        out = {}
        for i, (name, _) in enumerate(calls):
            out[name] = sum(ev[i].elapsed_time(ev[i + 1]) for ev in recs) / reps
        return out

    def sustained(self, graph, est_ms, seconds):
        """Back-to-back replays of `graph` for about `seconds`, with clock samples."""
        import torch
        reps = int(min(50000, max(10, math.ceil(seconds * 1e3 / max(est_ms, 1e-3)))))
        with torch.cuda.stream(self.stream):
            torch.cuda.synchronize()
            with ClockSampler(self.local) as clk:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(self.stream)
                for _ in range(reps):
                    graph.replay()
                b.record(self.stream)
                torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        return reps, ms, clk.summary()


def capture(stream, fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            fn()
    return g


def check_status(sv, status):
    import torch
    torch.cuda.synchronize()
    st = int(status.item())
    err = sv.svconv_read_error_word()
    if st or err:
        raise SystemExit(f"device status {st} / library error word {err}: results invalid")


# ----------------------------------------------------------------------------- conv workloads
def conv_leg(ctx, key, with_cpu, clock_window=False):
    """One SparseConv2D workload: index build + forward [+ fused backward] per step."""
    import torch

    from sparse_convolution_pruned_b200 import svconv as sv
    from sparse_convolution_pruned_b200.data_parallel import allreduce_grads

    args, dev, stream, world = ctx.args, ctx.dev, ctx.stream, ctx.world
    _, _, kind, dt_name = WORKLOADS[key]
    with_bwd = kind == "fwd+bwd"
    w = make_inputs(key, ctx.rank)  # weak scaling: each rank owns its own batch of frames
    n, T, Cin, Cout = w.n, w.T, w.Cin, w.Cout
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}[dt_name]
    odt = torch.bfloat16 if dt_name == "e4m3" else tdt  # e4m3 inputs give a bf16 output
    code = {"f32": sv.F32, "bf16": sv.BF16, "e4m3": sv.E4M3}[dt_name]
    elem = {"f32": 4, "bf16": 2, "e4m3": 1}[dt_name]
    elem_out = 2 if dt_name == "e4m3" else elem

    # pinned host inputs (the end-to-end leg copies these every step)
    h_coords = torch.from_numpy(w.coords).pin_memory()
    h_off = torch.from_numpy(w.frame_off).pin_memory()
    h_X = torch.from_numpy(w.X).to(tdt).pin_memory()
    h_W = torch.from_numpy(w.Wt).to(tdt).pin_memory()
    h_dY = torch.from_numpy(w.dY).to(odt).pin_memory()
    h_b = torch.from_numpy(w.bias).pin_memory() if w.bias is not None else None
    coords, off, X, Wt, dY = (t.to(dev) for t in (h_coords, h_off, h_X, h_W, h_dY))
    bias = h_b.to(dev) if h_b is not None else None
    nbr = torch.empty((n, 9), dtype=torch.int32, device=dev)
    Y = torch.empty((n, Cout), dtype=odt, device=dev)
    dX = torch.empty((n, Cin), dtype=odt, device=dev)
    grads = torch.empty((Cout * 9 * Cin + Cout,), dtype=torch.float32, device=dev)
    dW = grads[: Cout * 9 * Cin].view(Cout, 9, Cin)
    db = grads[Cout * 9 * Cin:]
    ws_code = code if with_bwd else sv.F32
    ws = torch.empty((max(16, sv.svconv_bwd_weight_workspace_size(ws_code, n, Cin, Cout),
                          sv.svconv_bwd_workspace_size(ws_code, n, Cin, Cout)) if with_bwd else 16,),
                     dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def index():
        sv.svconv_build_index(coords, off, T, w.H, w.W, nbr=nbr, status=status)

    def fwd():
        sv.svconv_fwd(X, nbr, Wt, bias, Y=Y)

    def bwd():
        # data and weight gradients in one call (side by side on disjoint SMs at 64 channels)
        sv.svconv_bwd(dY, X, nbr, Wt, dX=dX, dW=dW, db=db, workspace=ws)

    def step_kernels():
        index()
        fwd()
        if with_bwd:
            bwd()

    wgrad_launches = 2  # tcgen05 / fp32 partials + fixed-order split reduce
    launches = 2 + ((1 + wgrad_launches) if with_bwd else 0)

    with torch.cuda.stream(stream):
        step_kernels()  # first call outside capture: caches device info, kernel attributes, side streams
        stream.synchronize()
    g = capture(stream, step_kernels)
    g_fwd = capture(stream, lambda: (index(), fwd())) if with_bwd else None
    torch.cuda.synchronize()

    def one_step():
        g.replay()
        if world > 1 and with_bwd:
            allreduce_grads(grads)

    clocks = None
    sus = None
    if clock_window:
        # clock samples over the timed steps and the sustained replays right after them
        with ClockSampler(ctx.local) as clk:
            total_ms = ctx.timed(one_step, args.steps, args.warmup)
            if args.sustained_s > 0:
                sus = ctx.sustained(g, total_ms / args.steps, args.sustained_s)
        clocks = clk.summary()
    else:
        total_ms = ctx.timed(one_step, args.steps, args.warmup)
        if args.sustained_s > 0:
            sus = ctx.sustained(g, total_ms / args.steps, args.sustained_s)
    fwd_ms = ctx.timed(g_fwd.replay, args.steps, args.warmup) if with_bwd else total_ms
    hot_ms = ctx.timed(one_step, args.steps, args.warmup, flush_l2=False)
    total_ms, fwd_ms, hot_ms = ctx.max_over_ranks(total_ms, fwd_ms, hot_ms)

    names = [("build_index", index), ("fwd", fwd)]
    if with_bwd:
        names += [("bwd_data", lambda: sv.svconv_bwd_data(dY, nbr, Wt, dX=dX)),
                  ("bwd_weight", lambda: sv.svconv_bwd_weight(dY, X, nbr, dW=dW, db=db, workspace=ws))]
    per = ctx.per_kernel(names, max(args.steps, 10))
    if with_bwd:
        per["bwd (fused call)"] = ctx.per_kernel([("bwd", bwd)], max(args.steps, 10))["bwd"]
    single = with_bwd and dt_name == "bf16" and Cin == 64 and Cout == 64
    if single:
        ws1 = torch.empty((max(16, int(sv.lib().svconv_bwd_single_pass_workspace_size(n))),), dtype=torch.uint8,
                          device=dev)
        per["bwd (single pass)"] = ctx.per_kernel(
            [("bwd1", lambda: sv.svconv_bwd_single_pass(dY, X, nbr, Wt, dX=dX, dW=dW, db=db, workspace=ws1))],
            max(args.steps, 10))["bwd1"]

    # end to end through the Python API with pinned host buffers
    h_Y = torch.empty((n, Cout), dtype=odt).pin_memory()
    h_dX = torch.empty((n, Cin), dtype=odt).pin_memory()
    h_grads = torch.empty_like(grads, device="cpu").pin_memory()
    ins = [h_coords, h_off, h_X, h_W, h_dY] + ([h_b] if h_b is not None else [])
    outs = [h_Y] + ([h_dX, h_grads] if with_bwd else [])
    h2d = sum(x.numel() * x.element_size() for x in ins)
    d2h = sum(x.numel() * x.element_size() for x in outs)

    def e2e_step():
        coords.copy_(h_coords, non_blocking=True)
        off.copy_(h_off, non_blocking=True)
        X.copy_(h_X, non_blocking=True)
        Wt.copy_(h_W, non_blocking=True)
        if bias is not None:
            bias.copy_(h_b, non_blocking=True)
        if with_bwd:
            dY.copy_(h_dY, non_blocking=True)
        step_kernels()
        if world > 1 and with_bwd:
            allreduce_grads(grads)
        h_Y.copy_(Y, non_blocking=True)
        if with_bwd:
            h_dX.copy_(dX, non_blocking=True)
            h_grads.copy_(grads, non_blocking=True)

    if not with_bwd:
        h2d -= h_dY.numel() * h_dY.element_size()
    (e2e_ms,) = ctx.max_over_ranks(ctx.timed(e2e_step, args.steps, args.warmup))
    check_status(sv, status)

    cpu = cpu_baseline_conv(w, with_bwd, args.cpu_seconds) if with_cpu else None

    peaks = ctx.peaks
    alu = dt_name == "f32"
    fp8 = dt_name == "e4m3"
    work = conv_work(n, T, Cin, Cout, elem, bias is not None, elem_out)
    kern = {}
    for k in [nm for nm, _ in names]:
        kern[k] = dict(ms=per[k], **roofline_entry(work[k], per[k], peaks, alu=alu and k != "build_index", fp8=fp8))
    if with_bwd:
        kern["bwd (fused call)"] = {"ms": per["bwd (fused call)"],
                                   "note": "svconv_bwd: both gradients in one call, as the step runs them"}
    if single:
        kern["bwd (single pass)"] = {"ms": per["bwd (single pass)"],
                                    "note": "svconv_bwd_single_pass: both gradients from one pass over dY "
                                            "(one kernel + the split reduce); not the step's schedule"}
    top = max((nm for nm, _ in names), key=lambda k: per[k])
    roof = {k: v for k, v in kern[top].items() if k != "ms"}
    roof["kernel"] = top
    roof["traffic"] = kernel_traffic(key, top)
    roof["peak_source"] = peaks["source"]
    floors = sum(floor_seconds(work[k], peaks, alu=alu and k != "build_index", fp8=fp8) for k, _ in names)
    step_ms = total_ms / args.steps
    tokens = n * world
    res = {
        "workload": w.name, "n_kept_per_gpu": n, "T": T, "H": w.H, "W": w.W, "C_in": Cin, "C_out": Cout,
        "dtype": dt_name, "value": tokens / (step_ms * 1e-3), "unit": UNIT, "ms_per_step": step_ms,
        "step": "build_index+fwd" + ("+bwd(data, weight: one svconv_bwd call)" if with_bwd else "") +
                ("+allreduce(dW,db)" if world > 1 and with_bwd else ""),
        "l2": f"flushed by a {FLUSH_BYTES >> 20} MiB write between timed steps",
        "roofline": roof,
        "step_roofline": {"floor_ms": floors * 1e3, "frac": floors * 1e3 / step_ms,
                          "note": "sum of the step's per-kernel floors / measured step time"},
        "kernels": kern,
        "l2_hot": {"value": tokens * args.steps / (hot_ms * 1e-3), "ms_per_step": hot_ms / args.steps,
                   "note": "same step, no L2 flush between steps"},
        "e2e": {"value": tokens * args.steps / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches_per_step": launches,
        "cpu_baseline": cpu,
    }
    if with_bwd:
        res["fwd"] = {"value": tokens * args.steps / (fwd_ms * 1e-3), "unit": UNIT,
                      "ms_per_step": fwd_ms / args.steps, "step": "build_index+fwd"}
    if sus is not None:
        reps, ms, sclk = sus
        res["sustained"] = {"steps": reps, "seconds": ms * 1e-3, "ms_per_step": ms / reps,
                            "value": n * reps / (ms * 1e-3), "clocks": sclk,
                            "note": "back-to-back graph replays, no L2 flush"}
    if clocks is not None:
        res["clocks"] = clocks
    del g, g_fwd
    return res


# ----------------------------------------------------------------------------- adapter workload
def adapter_leg(ctx, with_cpu, clock_window=False):
    """Long-video bottleneck adapter: one step = index build + chunked adapter forward.

    X (n x 1024 bf16, 579 MB) is read and written in place each step, far larger than L2,
    so no flush is needed between steps.
    """
    import torch

    from sparse_convolution_pruned_b200 import svconv as sv

    args, dev, stream, world = ctx.args, ctx.dev, ctx.stream, ctx.world
    w = make_inputs("adapter", ctx.rank)
    n, T, D, R = w.n, w.T, w.D, w.R
    chunk_T = args.adapter_chunk_frames  # frames per chunk (device memory grows with it; cap 1 GB)
    offs = w.frame_off.astype(np.int64)
    max_rows = int(max(offs[min(t + chunk_T, T)] - offs[t] for t in range(0, T, chunk_T)))

    h_coords = torch.from_numpy(w.coords).pin_memory()
    h_off = torch.from_numpy(w.frame_off).pin_memory()
    h_X = torch.from_numpy(w.X).to(torch.bfloat16).pin_memory()
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated(dev) - ctx.flush.numel()
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

    def index():
        sv.svconv_build_index(coords, off, T, w.H, w.W, nbr=nbr, status=status)

    def adapter():
        sv.svconv_adapter_fwd(X, nbr, off, T, Wd, Wc, Wu, chunk_T=chunk_T, max_chunk_rows=max_rows,
                              workspace=ws, status=status)

    def step():
        index()
        adapter()

    n_chunks = (T + chunk_T - 1) // chunk_T
    launches = 1 + 3 * n_chunks  # index; per chunk: down GEMM, conv, up GEMM
    with torch.cuda.stream(stream):
        step()
        stream.synchronize()
    g = capture(stream, step)
    g_ad = capture(stream, adapter)
    torch.cuda.synchronize()
    # device memory of the workload (the L2-flush buffer and earlier legs' leftovers excluded)
    peak = torch.cuda.max_memory_allocated(dev) - ctx.flush.numel() - max(0, base)

    clocks = None
    sus = None
    if clock_window:
        with ClockSampler(ctx.local) as clk:
            total_ms = ctx.timed(g.replay, args.steps, args.warmup, flush_l2=False)
            if args.sustained_s > 0:
                sus = ctx.sustained(g, total_ms / args.steps, args.sustained_s)
        clocks = clk.summary()
    else:
        total_ms = ctx.timed(g.replay, args.steps, args.warmup, flush_l2=False)
        if args.sustained_s > 0:
            sus = ctx.sustained(g, total_ms / args.steps, args.sustained_s)
    ad_ms = ctx.timed(g_ad.replay, args.steps, args.warmup, flush_l2=False) / args.steps
    idx_ms = ctx.timed(index, args.steps, args.warmup) / args.steps

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
    e2e_ms = ctx.timed(e2e, e2e_steps, 3, flush_l2=False)
    total_ms, e2e_ms, ad_ms, idx_ms = ctx.max_over_ranks(total_ms, e2e_ms, ad_ms, idx_ms)
    check_status(sv, status)

    cpu = cpu_baseline_adapter(w, args.cpu_seconds) if with_cpu else None
    peaks = ctx.peaks
    ad_work = adapter_work(n, D, R)
    roof = {k: v for k, v in roofline_entry(ad_work, ad_ms, peaks).items()}
    roof["kernel"] = f"adapter_fwd ({3 * n_chunks} tcgen05 GEMM launches, timed together)"
    roof["traffic"] = kernel_traffic("adapter", "adapter_fwd")
    roof["peak_source"] = peaks["source"]
    # the adapter forward is a ~0.7 ms sequence of tensor-core launches: also against the sustained peak
    roof["frac_of_sustained_peak"] = ad_work["flops"] / (ad_ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"]
    idx_work = conv_work(n, T, R, R, 2, False)["build_index"]
    step_ms = total_ms / args.steps
    floors = floor_seconds(ad_work, peaks) + floor_seconds(idx_work, peaks)
    tokens = n * world
    res = {
        "workload": w.name, "n_kept_per_gpu": n, "T": T, "H": w.H, "W": w.W, "D": D, "R": R, "dtype": "bf16",
        "chunk_T": chunk_T, "value": tokens / (step_ms * 1e-3), "unit": UNIT, "ms_per_step": step_ms,
        "step": "build_index+adapter_fwd (in place)",
        "l2": "inputs larger than L2 (X read and written in place each step); no flush",
        "peak_device_bytes": peak,
        "roofline": roof,
        "step_roofline": {"floor_ms": floors * 1e3, "frac": floors * 1e3 / step_ms,
                          "note": "sum of the step's per-kernel floors / measured step time"},
        "kernels": {"adapter_fwd": dict(ms=ad_ms, **roofline_entry(ad_work, ad_ms, peaks)),
                    "build_index": dict(ms=idx_ms, **roofline_entry(idx_work, idx_ms, peaks))},
        "e2e": {"value": tokens * e2e_steps / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches_per_step": launches,
        "cpu_baseline": cpu,
    }
    if sus is not None:
        reps, ms, sclk = sus
        res["sustained"] = {"steps": reps, "seconds": ms * 1e-3, "ms_per_step": ms / reps,
                            "value": n * reps / (ms * 1e-3), "clocks": sclk,
                            "note": "back-to-back graph replays (X larger than L2)"}
    if clocks is not None:
        res["clocks"] = clocks
    del g, g_ad
    return res


# ----------------------------------------------------------------------------- keep-rate crossover
CROSSOVER_KEEPS = [0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 0.8, 0.9, 1.0]
CROSSOVER_CHANNELS = [64, 256]


def crossing(keeps, t_sparse, t_dense):
    """Keep rate at which the sparse time meets the dense time (linear between sweep points);
    None when the sparse path is faster at every swept keep rate."""
    d = [a - b for a, b in zip(t_sparse, t_dense)]
    for i in range(len(d)):
        if d[i] >= 0:
            if i == 0:
                return keeps[0]
            return keeps[i - 1] + (keeps[i] - keeps[i - 1]) * (-d[i - 1]) / (d[i] - d[i - 1])
    return None


def crossover_leg(ctx):
    """SparseConv2D against the dense-reconstruction pipeline (scatter -> cuDNN conv2d ->
    gather, PyTorch ops) over keep rates 0.1 .. 1.0 at C = 64 and C = 256 (T = 384 frames,
    16 x 16 grid, blob-saliency top-k keep, bf16), forward and forward + backward."""
    import torch

    from sparse_convolution_pruned_b200 import svconv as sv
    from sparse_convolution_pruned_b200 import workloads as wl
    from sparse_convolution_pruned_b200.dense_recon import DenseRecon, torch_weight

    torch.backends.cudnn.benchmark = True
    args, dev, stream = ctx.args, ctx.dev, ctx.stream
    steps = max(5, min(args.steps, 10))
    out = {"setup": "T=384, 16x16 grid, blob-saliency top-k keep per frame, bf16, no bias; sparse = svconv_fwd "
                    "(+ svconv_bwd) with the neighbour table built once per layout (the page reuses it across "
                    "the layers of a pruning stage; 'with index' adds svconv_build_index); dense = scatter -> "
                    "torch conv2d (cuDNN, channels-last, benchmark mode) -> gather, backward by autograd; "
                    "every step replayed from a CUDA graph, L2 flushed between steps",
           "keeps": CROSSOVER_KEEPS, "curves": {}}
    for C in CROSSOVER_CHANNELS:
        cur = {"sparse_fwd_ms": [], "sparse_fwd_with_index_ms": [], "dense_fwd_ms": [], "dense_conv_only_ms": [],
               "sparse_fwd_bwd_ms": [], "dense_fwd_bwd_ms": [], "n_kept": []}
        for keep in CROSSOVER_KEEPS:
            k = int(round(keep * 256))
            w = wl.small_c_bf16(seed=5, T=384, C=C, k=k)
            coords = torch.from_numpy(w.coords).to(dev)
            off = torch.from_numpy(w.frame_off).to(dev)
            X = torch.from_numpy(w.X).to(torch.bfloat16).to(dev)
            Wt = torch.from_numpy(w.Wt).to(torch.bfloat16).to(dev)
            dY = torch.from_numpy(w.dY).to(torch.bfloat16).to(dev)
            nbr = torch.empty((w.n, 9), dtype=torch.int32, device=dev)
            Y = torch.empty((w.n, C), dtype=torch.bfloat16, device=dev)
            dX = torch.empty_like(Y)
            dW = torch.empty((C, 9, C), dtype=torch.float32, device=dev)
            db = torch.empty((C,), dtype=torch.float32, device=dev)
            ws = torch.empty((max(16, sv.svconv_bwd_workspace_size(sv.BF16, w.n, C, C)),), dtype=torch.uint8,
                             device=dev)
            wtorch = torch_weight(Wt)
            dense = DenseRecon(coords, w.T, w.H, w.W)
            grid_in = dense.scatter(X).contiguous(memory_format=torch.channels_last)

            def index():
                sv.svconv_build_index(coords, off, w.T, w.H, w.W, nbr=nbr)

            def s_fwd():
                sv.svconv_fwd(X, nbr, Wt, None, Y=Y)

            def s_fwd_bwd():
                s_fwd()
                sv.svconv_bwd(dY, X, nbr, Wt, dX=dX, dW=dW, db=db, workspace=ws)

            with torch.cuda.stream(stream):
                index()
                s_fwd_bwd()
                for _ in range(3):  # cuDNN algorithm selection and autograd warm-up outside capture
                    dense.fwd(X, wtorch)
                    dense.fwd_bwd(X, wtorch, dY)
                stream.synchronize()
            graphs = {
                "sparse_fwd_ms": capture(stream, s_fwd),
                "sparse_fwd_with_index_ms": capture(stream, lambda: (index(), s_fwd())),
                "dense_fwd_ms": capture(stream, lambda: dense.fwd(X, wtorch)),
                "dense_conv_only_ms": capture(stream, lambda: torch.nn.functional.conv2d(grid_in, wtorch, padding=1)),
                "sparse_fwd_bwd_ms": capture(stream, s_fwd_bwd),
                "dense_fwd_bwd_ms": capture(stream, lambda: dense.fwd_bwd(X, wtorch, dY)),
            }
            for name, g in graphs.items():
                (ms,) = ctx.max_over_ranks(ctx.timed(g.replay, steps, 3))
                cur[name].append(ms / steps)
            cur["n_kept"].append(w.n)
            del graphs
        cur["crossover_keep_fwd"] = crossing(CROSSOVER_KEEPS, cur["sparse_fwd_ms"], cur["dense_fwd_ms"])
        cur["crossover_keep_fwd_with_index"] = crossing(CROSSOVER_KEEPS, cur["sparse_fwd_with_index_ms"],
                                                        cur["dense_fwd_ms"])
        cur["crossover_keep_fwd_bwd"] = crossing(CROSSOVER_KEEPS, cur["sparse_fwd_bwd_ms"], cur["dense_fwd_bwd_ms"])
        cur["crossover_keep_fwd_vs_conv_only"] = crossing(CROSSOVER_KEEPS, cur["sparse_fwd_ms"],
                                                          cur["dense_conv_only_ms"])
        out["curves"][f"C{C}"] = cur
    out["note"] = ("crossover_keep_* = keep rate where the sparse time meets the dense time (linear between "
                   "sweep points); null = sparse faster at every swept keep rate.  dense_conv_only = the cuDNN "
                   "convolution alone on an already scattered grid (no scatter, no gather).  The page reports 55% "
                   "on its own (unstated) hardware")
    return out


# ----------------------------------------------------------------------------- auxiliary cross-attention
def xattn_leg(ctx, with_cpu):
    """Auxiliary-token cross-attention (Key Design 3) at the long-video adapter's size: one
    CLS token attending over 282,624 down-projected rows of R = 256 (standalone entry point),
    and the chunked adapter forward with the cross-attention inside it."""
    import torch

    from sparse_convolution_pruned_b200 import svconv as sv
    from sparse_convolution_pruned_b200 import workloads as wl

    args, dev, stream = ctx.args, ctx.dev, ctx.stream
    a = make_inputs("adapter", ctx.rank)
    n, R, A = a.n, a.R, 1
    rng = np.random.default_rng(40 + ctx.rank)
    H_np = wl.round_to_bf16(rng.standard_normal((n, R)).astype(np.float32))
    aux_np = wl.round_to_bf16(rng.standard_normal((1, A, R)).astype(np.float32))
    h_H = torch.from_numpy(H_np).to(torch.bfloat16).pin_memory()
    h_aux = torch.from_numpy(aux_np).to(torch.bfloat16).pin_memory()
    goff = torch.tensor([0, n], dtype=torch.int32, device=dev)
    H = h_H.to(dev)
    aux = h_aux.to(dev)
    out = torch.empty((1, A, R), dtype=torch.float32, device=dev)
    h_out = torch.empty_like(out, device="cpu").pin_memory()
    ws = torch.empty((max(16, sv.svconv_xattn_workspace_size(1, n, A)),), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def xa():
        sv.svconv_xattn_aux(H, goff, aux, max_group_rows=n, out=out, workspace=ws, status=status)

    with torch.cuda.stream(stream):
        xa()
        stream.synchronize()
    g = capture(stream, xa)
    ms = ctx.timed(g.replay, args.steps, args.warmup) / args.steps
    per = ctx.per_kernel([("xattn", xa)], max(args.steps, 10))["xattn"]

    def e2e():
        H.copy_(h_H, non_blocking=True)
        aux.copy_(h_aux, non_blocking=True)
        xa()
        h_out.copy_(out, non_blocking=True)

    e2e_ms = ctx.timed(e2e, args.steps, args.warmup) / args.steps
    ms, per, e2e_ms = ctx.max_over_ranks(ms, per, e2e_ms)

    # the adapter with the cross-attention riding on its chunks
    chunk_T = args.adapter_chunk_frames
    offs = a.frame_off.astype(np.int64)
    max_rows = int(max(offs[min(t + chunk_T, a.T)] - offs[t] for t in range(0, a.T, chunk_T)))
    coords = torch.from_numpy(a.coords).to(dev)
    off = torch.from_numpy(a.frame_off).to(dev)
    X = torch.from_numpy(a.X).to(torch.bfloat16).to(dev)
    Wd, Wc, Wu = (torch.from_numpy(v).to(torch.bfloat16).to(dev) for v in (a.Wd, a.Wc, a.Wu))
    nbr = torch.empty((n, 9), dtype=torch.int32, device=dev)
    aux1 = aux[0]
    aux_out = torch.empty((A, R), dtype=torch.float32, device=dev)
    ws2 = torch.empty((max(16, sv.svconv_adapter_xattn_workspace_size(a.T, R, chunk_T, max_rows, A)),),
                      dtype=torch.uint8, device=dev)

    def index():
        sv.svconv_build_index(coords, off, a.T, a.H, a.W, nbr=nbr, status=status)

    def ad_x():
        sv.svconv_adapter_fwd_xattn(X, nbr, off, a.T, Wd, Wc, Wu, aux1, chunk_T=chunk_T, max_chunk_rows=max_rows,
                                    aux_out=aux_out, workspace=ws2, status=status)

    def ad():
        sv.svconv_adapter_fwd(X, nbr, off, a.T, Wd, Wc, Wu, chunk_T=chunk_T, max_chunk_rows=max_rows,
                              workspace=ws2, status=status)

    with torch.cuda.stream(stream):
        index()
        ad_x()
        stream.synchronize()
    g_ax = capture(stream, ad_x)
    g_a = capture(stream, ad)
    ax_ms = ctx.timed(g_ax.replay, args.steps, args.warmup, flush_l2=False) / args.steps
    a_ms = ctx.timed(g_a.replay, args.steps, args.warmup, flush_l2=False) / args.steps
    ax_ms, a_ms = ctx.max_over_ranks(ax_ms, a_ms)
    check_status(sv, status)

    cpu = None
    if with_cpu:
        import oracle
        oracle.build()
        rows = 20000
        t0 = time.perf_counter()
        oracle.xattn_aux(H_np[:rows], np.array([0, rows], np.int32), aux_np)
        dt = time.perf_counter() - t0
        cpu = {"value": rows / dt, "unit": "key rows/s", "cores": 1, "kind": "oracle", "host": host_cpu(),
               "sample": f"one query over the first {rows} of {n} rows (R = {R}); single-threaded C, fp64; "
                         f"1 core used of {os.cpu_count()}"}
    work = {"bytes": n * R * 2 + 2 * A * R + 4 * A * R, "flops": 4 * A * n * R}
    roof = roofline_entry(work, per, ctx.peaks)
    roof["kernel"] = "xattn_partial_kernel + xattn_combine_kernel"
    roof["traffic"] = kernel_traffic("xattn", "xattn")
    roof["peak_source"] = ctx.peaks["source"]
    n_chunks = (a.T + chunk_T - 1) // chunk_T
    del g, g_ax, g_a
    return {
        "workload": f"xattn_aux_n{n}_R{R}_A{A}_heads1 (rows of the long-video adapter's size)",
        "value": n / (ms * 1e-3), "unit": "key rows/s", "ms_per_step": ms,
        "step": "svconv_xattn_aux: one CLS token over one video's down-projected rows",
        "l2": f"flushed by a {FLUSH_BYTES >> 20} MiB write between timed steps",
        "roofline": roof, "kernels": {"xattn (both launches)": dict(ms=per, **roofline_entry(work, per, ctx.peaks))},
        "e2e": {"value": n / (e2e_ms * 1e-3), "unit": "key rows/s", "h2d_bytes_per_step": n * R * 2 + A * R * 2,
                "d2h_bytes_per_step": A * R * 4},
        "gpu_launches_per_step": 2,
        "cpu_baseline": cpu,
        "in_adapter": {"adapter_fwd_xattn_ms": ax_ms, "adapter_fwd_ms": a_ms, "overhead_ms": ax_ms - a_ms,
                       "chunk_T": chunk_T, "gpu_launches_per_step": 3 * n_chunks + n_chunks + 1,
                       "note": "the adapter forward with the cross-attention partials taken after each chunk's "
                               "down-projection (H1 still in L2) and merged after the last chunk"},
    }


def run_leg(ctx, key, with_cpu, clock_window=False):
    if WORKLOADS[key][2] == "adapter":
        return adapter_leg(ctx, with_cpu, clock_window)
    return conv_leg(ctx, key, with_cpu, clock_window)


# ----------------------------------------------------------------------------- B200 arm
def run_b200(args):
    import torch
    import torch.distributed as dist

    rank, local, world = dist_setup(args.gpus)
    ctx = Ctx(args, rank, local, world)
    head_key = args.workload or HEADLINE
    with_cpu = world == 1 and not args.no_cpu_baseline

    # the headline workload first: its timed steps and sustained replays carry the clock record
    if head_key == "xattn":  # the cross-attention leg alone (profiling runs)
        head = xattn_leg(ctx, with_cpu)
        head.update(dtype="bf16", n_kept_per_gpu=None, step_roofline=None)
    else:
        head = run_leg(ctx, head_key, with_cpu, clock_window=True)
    configs = {head_key: head}
    if world == 1 and not args.workload:
        for key in ORDER:
            if key != head_key:
                configs[key] = run_leg(ctx, key, with_cpu)
        configs["xattn"] = xattn_leg(ctx, with_cpu)
        if not args.no_crossover:
            configs["crossover"] = crossover_leg(ctx)

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
            "data": "synthetic",
            "config": {"workload": head["workload"], "n_kept_per_gpu": head["n_kept_per_gpu"],
                       "step": head["step"], "l2": head["l2"], "graph": "step replayed from a CUDA graph",
                       "parallelism": f"dp{world}",
                       "why_headline": ("largest fwd+bwd configuration that fits one GPU" if not args.workload
                                        else "the workload asked for with --workload")},
            "roofline": head["roofline"],
            "step_roofline": head.get("step_roofline"),
            "kernels": head["kernels"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches_per_step"] * args.steps,
            "clocks": dict(head.get("clocks") or {},
                           window="the headline's timed steps and its sustained replays right after them"),
            "cpu_baseline": head["cpu_baseline"],
        }
        if "sustained" in head:
            line["sustained"] = head["sustained"]
        if "fwd" in head:
            line["fwd"] = head["fwd"]
        if len(configs) > 1:
            line["configs"] = {k: {kk: vv for kk, vv in v.items()} for k, v in configs.items() if k != head_key}
        print(json.dumps(line))
    if world > 1:
        torch.cuda.synchronize()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="CPU-oracle work per workload for the cpu_baseline objects (seconds, about)")
    ap.add_argument("--sustained-s", type=float, default=1.0,
                    help="seconds of back-to-back replays per workload for the sustained leg (0: none)")
    ap.add_argument("--adapter-chunk-frames", type=int, default=1024,
                    help="adapter workload: token frames per chunk of the chunked adapter forward "
                         "(1024: 3 chunks, ~660 MiB peak; 512: 6 chunks, ~610 MiB)")
    ap.add_argument("--no-crossover", action="store_true",
                    help="skip the keep-rate sweep against the dense-reconstruction baseline")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["xattn"], default=None,
                    help="time only this workload (as the top-level line); default: the headline "
                         f"({HEADLINE}) plus every other workload under 'configs'")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.steps < 1:
        raise SystemExit("--steps must be >= 1")
    if args.impl == "reference":
        return run_reference(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
