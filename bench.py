#!/usr/bin/env python
"""Throughput of the cone-beam DRR hot path on B200 (one JSON line on stdout).

A step is one pass of the whole path over one batch of synthetic input:
prepare the volume (fp32 -> corner records or xy quads, whichever the
workload's forward runs faster in; bf16 for the bf16 workload), forward
ray-march of every view, zero the gradient volume,
adjoint scatter of an N(0,1) upstream gradient (with a workspace, so that
dense views take the corner-record path).  The default workload is the
256^3 bf16 volume seen by 4 C-arm views of 1024x1024 pixels with 512
samples per ray.  Inputs are resident in HBM when timing
starts.  L2 is flushed (a 256 MiB write) before every step, outside the
step's timing.  Each step is timed with CUDA events on the launching stream;
for N > 1 (torchrun, one process per GPU) every rank runs the same workload
on its own GPU (weak scaling, no collective in the data path) and the time
is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 3]
    python bench.py --impl reference ...   # the fp64 CPU oracle, same metric

`e2e` repeats the step through the public API with pinned HOST buffers:
host->device copies of the volume, poses and upstream gradient, and
device->host reads of the image and the gradient volume, inside the timing,
pipelined over two sets of device buffers (step k+1's uploads and step k's
downloads overlap the kernels on two copy streams).
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Gsamples/s (ray×samples) and DRR FPS at 1 B200; % of L2/HBM gather roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_BYTES = 126 * 1000 * 1000
FLUSH_BYTES = 256 << 20


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=3, choices=[1, 2, 3, 4],
                   help="workload (default 3: 256^3 bf16, 4 views 1024x1024, 512 samples, "
                        "the size the throughput target is quoted at)")
    p.add_argument("--layout", choices=["auto", "padded", "corners", "quads", "linear", "bricks"],
                   default="auto",
                   help="volume layout drr_prepare_volume writes for the forward (auto: the "
                        "faster one measured for the workload, AUTO_LAYOUT)")
    p.add_argument("--texture", action="store_true",
                   help="also time the texture-trilinear comparison forward (libdrr_texture.so)")
    p.add_argument("--pose", action="store_true",
                   help="also time the pose gradient (drr_render_pose_grad) on the same workload")
    p.add_argument("--alpha", action="store_true",
                   help="also time alpha compositing (forward and volume gradient) and the "
                        "Gaussian-Poisson surrogate on the same workload")
    p.add_argument("--siddon", action="store_true",
                   help="also time the cell-constant (Siddon) projector and backprojection on "
                        "the same workload (fp32 linear volume)")
    p.add_argument("--batched", action="store_true",
                   help="also time the batched forward, adjoint and pose gradient: the "
                        "workload's views split one per volume over as many volumes "
                        "(drr_render_batched, drr_render_adjoint_batched_ws, "
                        "drr_render_pose_grad_batched)")
    p.add_argument("--views", type=int, default=0,
                   help="render only the first VIEWS views of the workload (a smaller case of "
                        "the same kernels, for profilers; 0: all)")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the widened rows the default run also times (pose gradient, alpha "
                        "compositing, Siddon pair, batches)")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads' forward / adjoint timings (the configs block)")
    p.add_argument("--partition", choices=["replicas", "views"], default="replicas",
                   help="replicas (default): every rank runs the whole workload (weak scaling, no "
                        "collective); views: one job's detector rows split over the ranks, the "
                        "volume broadcast once, the gradient volume all-reduced every step "
                        "(strong scaling)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks (identity when no
    process group is running).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(world, units_per_rank_step, steps, max_ms):
    """Whole-job rate: the units every rank processed over the slowest rank's
    time (weak scaling: each rank runs its own replica of the workload)."""
    return world * units_per_rank_step * steps / (max_ms * 1e-3)


# ---------------------------------------------------------------------------
# workload description

# The layout each workload's forward runs fastest in on B200: corner records
# (one 16-byte load per sample) where dense bf16 rays reuse them in L1, xy
# quads (two loads, half the footprint) for the fp32 volumes.  Forward times
# measured (ms): 256^3 fp32 seen by 64 views of 200^2: quads 2.00, bricks
# 2.43, padded 2.96, corners 3.01, linear 3.95; 256^3 bf16 seen by 4 views of
# 1024^2: corners 2.86, quads 3.86, bricks 4.78, padded 4.92, linear 6.27;
# 512^3 fp32 seen by 2 views of 2048^2: quads 3.76, corners 3.97, bricks
# 4.53, padded 4.71, linear 6.23.
AUTO_LAYOUT = {1: "corners", 2: "quads", 3: "corners", 4: "quads"}


def workload(cfg, views=0):
    from cone_beam_ct_b200 import workloads as wl
    w = wl.make_config(cfg)
    if views and views < w.B:
        w.Rt = w.Rt[:views]
        if w.grad_out is not None:
            w.grad_out = w.grad_out[:views]
    if w.grad_out is None:
        w.grad_out = np.random.default_rng(2000 + cfg).standard_normal(
            (w.B, w.H, w.W)).astype(np.float32)
    return w


def config_block(w, cfg):
    """The workload, the same for both arms (how each arm stores the volume
    is reported beside it, not in it)."""
    from cone_beam_ct_b200 import workloads as wl
    nx, ny, nz = w.dims
    vol_dtype = "bf16" if w.dtype == wl.DTYPE_BF16 else "fp32"
    mode = "Beer-Lambert" if w.mode == wl.MODE_BEER_LAMBERT else "raw"
    return {
        "workload": f"{nx}^3 {vol_dtype} volume, {w.B} views x {w.H}x{w.W}, "
                    f"{w.n_samples} samples/ray: prepare + forward ({mode}) + adjoint",
        "config_index": cfg,
        "volume": f"{nx}x{ny}x{nz} {vol_dtype}, {float(w.spacing[0])} mm voxels",
        "views": w.B, "detector": [w.H, w.W], "samples_per_ray": w.n_samples,
        "samples_per_step": w.samples,
        "l2": "GPU arm: flushed before every step (256 MiB write, outside the step timing); "
              "CPU arm: not applicable",
        "inputs": "seeded synthetic phantom and poses (cone_beam_ct_b200.workloads)",
    }


# ---------------------------------------------------------------------------
# clocks

def physical_gpu(ordinal):
    """nvidia-smi id of torch device ``ordinal`` (honours CUDA_VISIBLE_DEVICES)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if ordinal < len(ids):
            return ids[ordinal]
    return str(ordinal)


class ClockSampler:
    """nvidia-smi sampled every 100 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# roofline helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def l2_read_peak_gbs(torch, nbytes):
    """L2 read bandwidth over a buffer of ``nbytes`` (the volume's size), best
    of 6 launches of libdrr_probe.so, in GB/s.  Each launch streams the buffer
    enough times to read about 8 GB: shorter launches under-read the peak
    (measured on B200 over 32 MiB: 14.8 TB/s at 0.6 GB per launch, 17.6 at
    2 GB, 18.7 at 8 GB)."""
    import ctypes
    lib = ctypes.CDLL(os.path.join(ROOT, "cone_beam_ct_b200", "libdrr_probe.so"))
    lib.drr_probe_l2_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p]
    lib.drr_probe_l2_read.restype = ctypes.c_int
    n16 = max(1, nbytes // 16)
    buf = torch.ones(n16 * 4, dtype=torch.float32, device="cuda")
    sink = torch.zeros(1, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    reps = max(20, -(-8_000_000_000 // (n16 * 16)))
    best = 0.0
    for _ in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        rc = lib.drr_probe_l2_read(buf.data_ptr(), n16, reps, sink.data_ptr(), stream.cuda_stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if rc != 0:
            return None
        best = max(best, n16 * 16 * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    return best


def l2_red_probe(torch, nbytes):
    """The L2's fp32 reduction throughput over a buffer of ``nbytes`` (the
    gradient volume's size), for each pattern of libdrr_probe.so's
    drr_probe_l2_red: best of 4 launches of ~2 G values each.  Returns
    {pattern: {"gvalues_s", "gsector_ops_s"}} or None."""
    import ctypes
    lib = ctypes.CDLL(os.path.join(ROOT, "cone_beam_ct_b200", "libdrr_probe.so"))
    lib.drr_probe_l2_red.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_void_p]
    lib.drr_probe_l2_red.restype = ctypes.c_int
    n = max(8, (nbytes // 4) // 8 * 8)
    buf = torch.zeros(n, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    res = {}
    # kind: (name, values per pass, sector operations per pass)
    kinds = {0: ("scalar, 8 values per sector op", n, n // 8),
             1: ("16-byte vector, 4 values per sector op", n, n // 4),
             2: ("scalar, 1 value per sector op", n // 8, n // 8)}
    for kind, (name, values, ops) in kinds.items():
        reps = max(1, 2_000_000_000 // values)
        best = 0.0
        for _ in range(4):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            rc = lib.drr_probe_l2_red(buf.data_ptr(), n, reps, kind, stream.cuda_stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if rc != 0:
                return None
            best = max(best, reps / (e0.elapsed_time(e1) * 1e-3))
        res[name] = {"gvalues_s": best * values / 1e9, "gsector_ops_s": best * ops / 1e9}
    return res


def code_digest(paths):
    """First 16 hex digits of the SHA-256 of the sources' code: comments
    removed and whitespace collapsed, so that a comment edit does not count as
    a change of the kernel."""
    digest = hashlib.sha256()
    for src in paths:
        with open(os.path.join(ROOT, src)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        digest.update(" ".join(text.split()).encode())
    return digest.hexdigest()[:16]


def traffic_for(kernel, workload_name, layout_name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current code of the kernel and, for a kernel that reads the volume,
    in the same layout (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    entry = table.get(kernel, {}).get(workload_name)
    if not entry or entry.get("layout", layout_name) != layout_name:
        return None
    if not all(os.path.exists(os.path.join(ROOT, src)) for src in entry["sources"]):
        return None
    if code_digest(entry["sources"]) != entry["code_sha256_16"]:
        return None
    return entry["dram_bytes_per_launch"]


# ---------------------------------------------------------------------------
# the reference arm: the fp64 CPU oracle, timed on the host cores

# the volume adjoint's launches, timed as one group; the record kernel (dense
# views) dominates it
ADJOINT_GROUP = ("volume adjoint: plan_views + zero_records + records_kernel + scatter_records "
                 "+ slab_adjoint_kernel (records_kernel dominant where the views are dense, "
                 "slab_adjoint_kernel where they are sparse)")

REF_SAMPLES_PER_STEP = 4_000_000      # ray-samples per reference-arm step (~0.6 s of fp64 CPU)
BASELINE_SAMPLES = 100_000_000        # ray-samples of the cpu_baseline sample (~15 s)


def oracle_on_rays(w, view, rows, cores):
    """Forward and adjoint of the fp64 oracle over the full-width detector rows
    ``rows`` of view ``view``; returns the ray-samples processed."""
    import oracle
    ids = np.concatenate([np.arange(r * w.W, (r + 1) * w.W) for r in rows]).astype(np.int64)
    Rt = w.Rt[view:view + 1]
    oracle.render_rays(w.vol, w.dims, w.spacing, w.origin, w.K, Rt, w.H, w.W, w.n_samples,
                       w.density_factor, w.mode, ids, nthreads=cores)
    go = np.zeros((1, w.H, w.W), np.float32)
    go[0, rows, :] = w.grad_out[view, rows, :]
    oracle.adjoint(w.dims, w.spacing, w.origin, w.K, Rt, w.H, w.W, w.n_samples,
                   w.density_factor, w.mode, go, vol=w.vol, nthreads=1)
    return len(ids) * w.n_samples


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = workload(args.config, args.views)
    cores = len(os.sched_getaffinity(0))
    rows_per_step = max(1, min(w.H, REF_SAMPLES_PER_STEP // (w.W * w.n_samples)))

    def step(s):
        # step s: view s mod B, the next block of rows_per_step rows (wrapping)
        view = s % w.B
        r0 = (s // w.B) * rows_per_step
        rows = [(r0 + r) % w.H for r in range(rows_per_step)]
        return oracle_on_rays(w, view, rows, cores)

    for s in range(args.warmup):
        step(s)
    done = 0
    t0 = time.perf_counter()
    for s in range(args.steps):
        done += step(args.warmup + s)
    dt = time.perf_counter() - t0
    value = done / dt / 1e9
    sample = (f"{rows_per_step} full detector rows of one view per step ({rows_per_step * w.W} "
              f"rays x {w.n_samples} samples): fp64 forward threaded over rays on {cores} "
              f"cores + fp64 adjoint on one thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Gsamples/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, args.config),
        "layout": "linear fp32 (the oracle's own arrays)",
        "cpu_baseline": {"value": value, "unit": "Gsamples/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "Gsamples/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm

def cpu_baseline(w):
    """The oracle, as it stands, on a bounded sample of the same workload:
    every k-th detector row of every view, k chosen for about
    BASELINE_SAMPLES ray-samples."""
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    k = max(1, -(-w.samples // BASELINE_SAMPLES))
    rows = list(range(0, w.H, k))
    t0 = time.perf_counter()
    done = 0
    for view in range(w.B):
        done += oracle_on_rays(w, view, rows, cores)
    dt = time.perf_counter() - t0
    return {"value": done / dt / 1e9, "unit": "Gsamples/s", "cores": cores, "kind": "oracle",
            "sample": f"every {k}-th detector row of all {w.B} views ({done:.3g} ray-samples), "
                      f"fp64 forward threaded over rays + fp64 adjoint on one thread, "
                      f"{dt:.1f} s"}


def texture_comparison(torch, w, vol32, Rt, exact_out):
    """Forward through the texture units (8-bit interpolation weights) on the
    same workload: kernel time (best of 5) and its difference from the exact
    forward's image (which the parity tests pin to the oracle)."""
    from cone_beam_ct_b200 import texture
    res = {}
    stream = torch.cuda.current_stream()
    for texel, name in ((texture.TEXEL_F32, "fp32 texels"), (texture.TEXEL_F16, "fp16 texels")):
        tv = texture.TextureVolume(vol32, w.dims, texel)
        out = torch.empty_like(exact_out)
        times = []
        for _ in range(6):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            tv.render(w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples, w.density_factor,
                      w.mode, out, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        tv.close()
        ref = exact_out.double()
        scale = ref.abs().max().item()
        diff = (out.double() - ref).abs()
        big = ref.abs() >= 1e-2 * scale
        ms = min(times[1:])
        res[name] = {"ms": ms, "gsamples_s": w.samples / (ms * 1e-3) / 1e9,
                     "normwise_vs_exact": diff.max().item() / scale,
                     "per_pixel_vs_exact": (diff[big] / ref.abs()[big]).max().item()}
    return res


def pose_timing(torch, w, prep, dtype, layout, Rt, grad_out, out, elem, l2_peak, hbm_peak,
                vol_fits_l2):
    """The pose gradient on the same workload (not part of the step): kernel
    time (median of 10, L2 flushed before each) and its gather roofline, the
    forward's 8 voxel reads per sample."""
    from cone_beam_ct_b200 import drr
    from cone_beam_ct_b200 import workloads as wl
    stream = torch.cuda.current_stream()
    g = torch.zeros((w.B, 12), dtype=torch.float32, device=out.device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=out.device)
    fwd = out if w.mode == wl.MODE_BEER_LAMBERT else None
    times = []
    for m in range(13):
        flush.fill_(m & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        drr.drr_render_pose_grad(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, w.B,
                                 w.H, w.W, w.n_samples, w.density_factor, w.mode, grad_out, fwd,
                                 g, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if m >= 3:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    nbytes = 8 * elem * w.samples
    achieved = nbytes / (ms * 1e-3) / 1e9
    bound, peak = ("l2", l2_peak) if vol_fits_l2 and l2_peak else ("hbm", hbm_peak)
    return {"ms": ms, "gsamples_s": w.samples / (ms * 1e-3) / 1e9,
            "roofline": {"kernel": "pose_kernel", "bound": bound, "achieved": achieved,
                         "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "algorithmic_bytes_per_launch": int(nbytes)}}


def _median_ms(torch, fn, reps=10, flush=None):
    stream = torch.cuda.current_stream()
    times = []
    for m in range(reps + 3):
        if flush is not None:
            flush.fill_(m & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        if m >= 3:
            times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def alpha_timing(torch, w, vol32, prep, dtype, layout, Rt, grad_out, elem, l2_peak, hbm_peak,
                 vol_fits_l2):
    """Alpha compositing on the same workload (forward from the prepared
    volume; its pose gradient; its volume gradient, with and without a
    workspace, unless the volume is zero-bordered), and the surrogate on its
    image: median of 10, L2 flushed before each."""
    from cone_beam_ct_b200 import drr
    dev = vol32.device
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, w.H, w.W), dtype=torch.float32, device=dev)
    grad = torch.zeros((w.dims[2], w.dims[1], w.dims[0]), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def fwd():
        drr.drr_render(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                       w.n_samples, w.density_factor, drr.DRR_MODE_ALPHA, out, stream=stream)

    ws = torch.empty(drr.drr_adjoint_workspace_bytes(w.dims, w.B), dtype=torch.uint8, device=dev)

    def adj(workspace):
        if workspace:
            drr.drr_render_alpha_adjoint_ws(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K,
                                            Rt, w.B, w.H, w.W, w.n_samples, w.density_factor,
                                            grad_out, out, grad, ws, stream=stream)
        else:
            drr.drr_render_alpha_adjoint(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K,
                                         Rt, w.B, w.H, w.W, w.n_samples, w.density_factor,
                                         grad_out, out, grad, stream=stream)

    grad_Rt = torch.zeros((w.B, 12), dtype=torch.float32, device=dev)

    def pose():
        drr.drr_render_pose_grad(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, w.B,
                                 w.H, w.W, w.n_samples, w.density_factor, drr.DRR_MODE_ALPHA,
                                 grad_out, out, grad_Rt, stream=stream)

    fwd_ms = _median_ms(torch, fwd, flush=flush)
    pose_ms = _median_ms(torch, pose, flush=flush)
    adj_ms = direct_ms = None
    if layout != drr.DRR_LAYOUT_PADDED:
        adj_ms = _median_ms(torch, lambda: adj(True), flush=flush)
        direct_ms = _median_ms(torch, lambda: adj(False), flush=flush)
    bound, peak = ("l2", l2_peak) if vol_fits_l2 and l2_peak else ("hbm", hbm_peak)

    def roof(kernel, ms, nbytes):
        a = nbytes / (ms * 1e-3) / 1e9
        return {"kernel": kernel, "bound": bound, "achieved": a, "peak": peak, "unit": "GB/s",
                "frac": a / peak, "algorithmic_bytes_per_launch": int(nbytes)}

    z = torch.randn((w.B, w.H, w.W), dtype=torch.float32, device=dev,
                    generator=torch.Generator(device=dev).manual_seed(5))
    noisy = torch.empty_like(out)
    gi = torch.empty_like(out)
    n = out.numel()
    noise_ms = _median_ms(torch, lambda: drr.drr_poisson_noise(out, z, 1e4, noisy, stream=stream))
    noise_bwd_ms = _median_ms(torch, lambda: drr.drr_poisson_noise_backward(
        out, z, 1e4, grad_out, gi, stream=stream))
    res = {"forward": {"ms": fwd_ms, "gsamples_s": w.samples / (fwd_ms * 1e-3) / 1e9,
                       "roofline": roof("forward_kernel<alpha>", fwd_ms, 8 * elem * w.samples)},
           "pose_gradient": {"ms": pose_ms, "gsamples_s": w.samples / (pose_ms * 1e-3) / 1e9,
                             "roofline": roof("pose_kernel<alpha>", pose_ms,
                                              8 * elem * w.samples)},
           "density_factor": w.density_factor,
           "surrogate": {"ms": noise_ms, "backward_ms": noise_bwd_ms,
                         "hbm_gbs": 12 * n / (noise_ms * 1e-3) / 1e9,
                         "backward_hbm_gbs": 16 * n / (noise_bwd_ms * 1e-3) / 1e9}}
    if adj_ms is not None:
        res["adjoint"] = {"ms": adj_ms, "gsamples_s": w.samples / (adj_ms * 1e-3) / 1e9,
                          "roofline": roof("alpha adjoint (with a workspace)", adj_ms,
                                           32 * w.samples),
                          "without_workspace_ms": direct_ms}
    return res


def batched_timing(torch, w, vol32, dtype, layout, Rt, grad_out, elem, l2_peak, hbm_peak,
                   vol_fits_l2):
    """Batches on the same workload: its B views split one per volume over B
    volumes (the phantom scaled by 1 + v/10 for volume v), one channel, in
    the bench's layout and dtype; the batched forward (Beer-Lambert), the
    batched adjoint with a workspace (records per volume) and the batched
    pose gradient: median of 10, L2 flushed before each.  Same ray-samples as the step; B volumes to read and
    B gradient volumes to scatter into instead of one."""
    from cone_beam_ct_b200 import drr
    from cone_beam_ct_b200 import workloads as wl
    dev = vol32.device
    n_vols = w.B
    nx, ny, nz = w.dims
    per = drr.drr_prepared_bytes(w.dims, dtype, layout)
    vols = torch.empty(n_vols * per, dtype=torch.uint8, device=dev)
    for v in range(n_vols):
        drr.drr_prepare_volume((vol32 * (1.0 + 0.1 * v)).contiguous(), w.dims, dtype, layout,
                               vols[v * per:(v + 1) * per], per)
    out = torch.empty((w.B, 1, w.H, w.W), dtype=torch.float32, device=dev)
    grads = torch.zeros((n_vols, 1, nz, ny, nx), dtype=torch.float32, device=dev)
    ws = torch.empty(drr.drr_adjoint_batched_workspace_bytes(w.dims, n_vols, 1, w.B),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    mode = w.mode

    def fwd():
        drr.drr_render_batched(vols, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, n_vols,
                               1, w.B, w.H, w.W, w.n_samples, w.density_factor, mode, out,
                               stream=stream)

    def adj():
        drr.drr_render_adjoint_batched_ws(w.dims, w.spacing, w.origin, w.K, Rt, n_vols, 1, w.B,
                                          w.H, w.W, w.n_samples, w.density_factor, mode,
                                          grad_out, out if mode == wl.MODE_BEER_LAMBERT else None,
                                          grads, ws, stream=stream)

    grad_Rt = torch.zeros((w.B, 12), dtype=torch.float32, device=dev)

    def pose():
        drr.drr_render_pose_grad_batched(vols, dtype, layout, w.dims, w.spacing, w.origin, w.K,
                                         Rt, n_vols, 1, w.B, w.H, w.W, w.n_samples,
                                         w.density_factor, mode, grad_out,
                                         out if mode == wl.MODE_BEER_LAMBERT else None, grad_Rt,
                                         stream=stream)

    fwd_ms = _median_ms(torch, fwd, flush=flush)
    adj_ms = _median_ms(torch, adj, flush=flush)
    pose_ms = _median_ms(torch, pose, flush=flush)
    bound, peak = ("l2", l2_peak) if vol_fits_l2 and l2_peak else ("hbm", hbm_peak)

    def roof(kernel, ms, nbytes):
        a = nbytes / (ms * 1e-3) / 1e9
        return {"kernel": kernel, "bound": bound, "achieved": a, "peak": peak, "unit": "GB/s",
                "frac": a / peak, "algorithmic_bytes_per_launch": int(nbytes)}

    return {"n_vols": n_vols, "channels": 1, "n_views": w.B,
            "pose_gradient": {"ms": pose_ms, "gsamples_s": w.samples / (pose_ms * 1e-3) / 1e9,
                              "roofline": roof("pose_kernel (batched)", pose_ms,
                                               8 * elem * w.samples)},
            "forward": {"ms": fwd_ms, "gsamples_s": w.samples / (fwd_ms * 1e-3) / 1e9,
                        "roofline": roof("forward_kernel (batched)", fwd_ms,
                                         8 * elem * w.samples)},
            "adjoint": {"ms": adj_ms, "gsamples_s": w.samples / (adj_ms * 1e-3) / 1e9,
                        "roofline": roof("adjoint (batched, with a workspace)", adj_ms,
                                         32 * w.samples)}}


def siddon_pieces(w):
    """Cells crossed per ray, summed over the workload (the Siddon walk's unit
    of work): |entry cell - exit cell| summed over the axes, plus one, for every
    ray that hits the cells' box -- geometry only, in numpy fp64."""
    K = np.asarray(w.K, np.float64)
    u, v = np.meshgrid(np.arange(w.W, dtype=np.float64), np.arange(w.H, dtype=np.float64))
    pix = np.stack([u.ravel(), v.ravel(), np.ones(u.size)])
    q = np.linalg.solve(K, pix)
    n = np.asarray(w.dims, np.float64)
    sp = np.asarray(w.spacing, np.float64)
    total = 0
    for b in range(w.B):
        Rt = np.asarray(w.Rt[b], np.float64).reshape(3, 4)
        R, t = Rt[:, :3], Rt[:, 3]
        a = R.T @ q
        d = (a / np.linalg.norm(a, axis=0)) / sp[:, None]
        C = ((-R.T @ t) - np.asarray(w.origin, np.float64)) / sp
        with np.errstate(divide="ignore", invalid="ignore"):
            ta = (-0.5 - C[:, None]) / d
            tb = (n[:, None] - 0.5 - C[:, None]) / d
        tn = np.nanmax(np.where(np.isfinite(ta), np.minimum(ta, tb), -np.inf), axis=0)
        tf = np.nanmin(np.where(np.isfinite(ta), np.maximum(ta, tb), np.inf), axis=0)
        t0 = np.maximum(tn, 0.0)
        hit = tf > t0
        p0 = C[:, None] + t0 * d
        p1 = C[:, None] + tf * d
        c0 = np.clip(np.floor(p0 + 0.5), 0, n[:, None] - 1)
        c1 = np.clip(np.floor(p1 + 0.5), 0, n[:, None] - 1)
        total += int(np.sum((np.abs(c1 - c0).sum(axis=0) + 1)[hit]))
    return total


def siddon_timing(torch, w, vol32, Rt, grad_out, l2_peak, hbm_peak):
    """The cell-constant projector and its backprojection on the same
    workload: median of 10 with L2 flushed before each, per cell crossed."""
    from cone_beam_ct_b200 import drr
    from cone_beam_ct_b200 import workloads as wl
    dev = vol32.device
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, w.H, w.W), dtype=torch.float32, device=dev)
    grad = torch.zeros((w.dims[2], w.dims[1], w.dims[0]), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    mode = w.mode if w.mode != wl.MODE_ALPHA else wl.MODE_RAW
    fwd_ms = _median_ms(torch, lambda: drr.drr_render_siddon(
        vol32, drr.DRR_F32, w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
        w.density_factor, mode, out, stream=stream), flush=flush)
    adj_ms = _median_ms(torch, lambda: drr.drr_render_siddon_adjoint(
        w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.density_factor, mode, grad_out,
        out, grad, stream=stream), flush=flush)
    pieces = siddon_pieces(w)
    fits = w.dims[0] * w.dims[1] * w.dims[2] * 4 < L2_BYTES
    bound, peak = ("l2", l2_peak) if fits and l2_peak else ("hbm", hbm_peak)

    def roof(kernel, ms):
        a = 4 * pieces / (ms * 1e-3) / 1e9      # one fp32 voxel read (or atomic add) per cell
        return {"kernel": kernel, "bound": bound, "achieved": a, "peak": peak, "unit": "GB/s",
                "frac": a / peak, "algorithmic_bytes_per_launch": 4 * pieces}

    return {"cells_crossed": pieces, "volume": "fp32, linear",
            "forward": {"ms": fwd_ms, "gcells_s": pieces / (fwd_ms * 1e-3) / 1e9,
                        "roofline": roof("siddon_forward_kernel", fwd_ms)},
            "adjoint": {"ms": adj_ms, "gcells_s": pieces / (adj_ms * 1e-3) / 1e9,
                        "roofline": roof("siddon_adjoint_kernel", adj_ms)}}


def bricks_timing(torch, w, vol32, Rt, dtype, mode):
    """The bricked layout's forward (drr_render) and the same with each frustum
    layer staged in shared memory by bulk copies (drr_render_staged, the
    measured comparison): median of 5 each, L2 flushed before each."""
    from cone_beam_ct_b200 import drr
    dev = vol32.device
    nbytes = drr.drr_prepared_bytes(w.dims, dtype, drr.DRR_LAYOUT_BRICKS)
    bricks = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    drr.drr_prepare_volume(vol32, w.dims, dtype, drr.DRR_LAYOUT_BRICKS, bricks, nbytes)
    out = torch.empty((w.B, w.H, w.W), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    mode = 0 if mode == 2 else mode
    plain = _median_ms(torch, lambda: drr.drr_render(
        bricks, dtype, drr.DRR_LAYOUT_BRICKS, w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H,
        w.W, w.n_samples, w.density_factor, mode, out), reps=5, flush=flush)
    staged = _median_ms(torch, lambda: drr.drr_render_staged(
        bricks, dtype, w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples,
        w.density_factor, mode, out), reps=5, flush=flush)
    return {"bytes": nbytes, "forward_ms": plain, "staged_forward_ms": staged,
            "gsamples_s": w.samples / (plain * 1e-3) / 1e9,
            "staged_gsamples_s": w.samples / (staged * 1e-3) / 1e9}


# the workloads of the configs block: the other four, config 5 being the
# adjoint of config 2's geometry (RAW, its own seeded N(0, 1) upstream)
OTHER_CONFIGS = {3: (1, 2, 4, 5), 1: (2, 3, 4, 5), 2: (1, 3, 4, 5), 4: (1, 2, 3, 5)}


def config_timing(torch, cfg, hbm_peak, l2_cache):
    """Forward and adjoint (with a workspace) of one more workload, each the
    median of 5 launches with L2 flushed before each, in the layout its
    forward runs fastest in; Gsamples/s, DRR FPS and the gather-roofline
    fraction (L2 read probe for a volume that fits in L2, else HBM)."""
    from cone_beam_ct_b200 import drr
    from cone_beam_ct_b200 import workloads as wl
    w = workload(cfg)
    dev = torch.device("cuda", torch.cuda.current_device())
    geom_cfg = 2 if cfg == 5 else cfg
    lname = AUTO_LAYOUT[geom_cfg]
    layout = {"corners": drr.DRR_LAYOUT_CORNERS, "quads": drr.DRR_LAYOUT_QUADS,
              "bricks": drr.DRR_LAYOUT_BRICKS}[lname]
    dtype = drr.DRR_BF16 if w.dtype == wl.DTYPE_BF16 else drr.DRR_F32
    elem = 2 if dtype == drr.DRR_BF16 else 4
    nx, ny, nz = w.dims
    vol32 = torch.from_numpy(w.vol).to(dev)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).to(dev)
    go = torch.from_numpy(w.grad_out).to(dev)
    pbytes = drr.drr_prepared_bytes(w.dims, dtype, layout)
    prep = torch.empty(pbytes, dtype=torch.uint8, device=dev)
    drr.drr_prepare_volume(vol32, w.dims, dtype, layout, prep, pbytes)
    out = torch.empty((w.B, w.H, w.W), dtype=torch.float32, device=dev)
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device=dev)
    ws = torch.empty(drr.drr_adjoint_workspace_bytes(w.dims, w.B), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    mode = w.mode

    def fwd():
        drr.drr_render(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                       w.n_samples, w.density_factor, mode, out)

    def adj():
        drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                                  w.n_samples, w.density_factor, mode, go,
                                  out if mode == wl.MODE_BEER_LAMBERT else None, grad, ws)

    vol_bytes = nx * ny * nz * elem
    fits = vol_bytes < L2_BYTES
    if fits and vol_bytes not in l2_cache:
        l2_cache[vol_bytes] = l2_read_peak_gbs(torch, vol_bytes)
    bound, peak = ("l2", l2_cache[vol_bytes]) if fits and l2_cache.get(vol_bytes) else (
        "hbm", hbm_peak)

    def entry(name, ms, nbytes):
        a = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "gsamples_s": w.samples / (ms * 1e-3) / 1e9, "fps": w.B / (ms * 1e-3),
                "roofline": {"kernel": name, "bound": bound, "achieved": a, "peak": peak,
                             "unit": "GB/s", "frac": a / peak,
                             "algorithmic_bytes_per_launch": int(nbytes)}}

    res = {"workload": config_block(w, cfg)["workload"], "layout": lname,
           "samples": w.samples}
    fwd()
    if cfg != 5:
        res["forward"] = entry("forward_kernel", _median_ms(torch, fwd, reps=5, flush=flush),
                               8 * elem * w.samples)
    res["adjoint"] = entry(ADJOINT_GROUP, _median_ms(torch, adj, reps=5, flush=flush),
                           32 * w.samples)
    if cfg != 5:
        res["bricks"] = bricks_timing(torch, w, vol32, Rt, dtype, mode)
    if cfg == 5:
        res["workload"] = (f"adjoint of the {nx}^3 / {w.B}-view {w.H}x{w.W} / "
                           f"{w.n_samples}-sample geometry, N(0,1) upstream, RAW")
    else:
        step = res["forward"]["ms"] + res["adjoint"]["ms"]
        res["forward_plus_adjoint"] = {"ms": step, "gsamples_s": w.samples / (step * 1e-3) / 1e9}
    del prep, ws, grad, out, vol32, flush
    torch.cuda.empty_cache()
    return res


def run_e2e(torch, drr, w, args, world, dev, stream, flush, dtype, layout, prep, pbytes, ws,
            ws_bytes, fwd_needed, ref_out, ref_grad):
    """The step through the public API from and to pinned host memory: every
    step uploads its volume, poses and upstream gradient and downloads its
    image and gradient volume, inside the timed region.  Steps are pipelined
    over two sets of device buffers: step k+1's uploads (an upload stream)
    run while step k computes, and step k's downloads (a download stream)
    while step k+1 computes; events keep each buffer's readers and writers
    in order.  Device time of the whole run, max over ranks."""
    nx, ny, nz = w.dims
    h_vol = torch.from_numpy(w.vol).pin_memory()
    h_Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).pin_memory()
    h_go = torch.from_numpy(w.grad_out).pin_memory()
    h_out = [torch.empty((w.B, w.H, w.W), dtype=torch.float32).pin_memory() for _ in range(2)]
    h_grad = [torch.empty((nz, ny, nx), dtype=torch.float32).pin_memory() for _ in range(2)]
    d_vol = [torch.empty_like(h_vol, device=dev) for _ in range(2)]
    d_Rt = [torch.empty_like(h_Rt, device=dev) for _ in range(2)]
    d_go = [torch.empty_like(h_go, device=dev) for _ in range(2)]
    d_out = [torch.empty((w.B, w.H, w.W), dtype=torch.float32, device=dev) for _ in range(2)]
    d_grad = [torch.empty((nz, ny, nx), dtype=torch.float32, device=dev) for _ in range(2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    uploaded, inputs_free, img_ready, img_free, grad_ready, grad_free = (ev() for _ in range(6))
    for j in range(2):                       # every buffer starts free
        for e in (inputs_free[j], img_free[j], grad_free[j]):
            e.record(stream)

    def e2e_step(k):
        j = k & 1
        with torch.cuda.stream(up):          # step k's inputs, once step k-2 is done with them
            up.wait_event(inputs_free[j])
            d_vol[j].copy_(h_vol, non_blocking=True)
            d_Rt[j].copy_(h_Rt, non_blocking=True)
            d_go[j].copy_(h_go, non_blocking=True)
            uploaded[j].record(up)
        flush.fill_(k & 0xFF)
        stream.wait_event(uploaded[j])
        drr.drr_prepare_volume(d_vol[j], w.dims, dtype, layout, prep, pbytes, stream=stream)
        stream.wait_event(img_free[j])
        drr.drr_render(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, d_Rt[j], w.B, w.H,
                       w.W, w.n_samples, w.density_factor, w.mode, d_out[j], stream=stream)
        img_ready[j].record(stream)
        stream.wait_event(grad_free[j])
        d_grad[j].zero_()
        drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, d_Rt[j], w.B, w.H, w.W,
                                  w.n_samples, w.density_factor, w.mode, d_go[j],
                                  d_out[j] if fwd_needed else None, d_grad[j], ws, ws_bytes,
                                  stream=stream)
        inputs_free[j].record(stream)
        grad_ready[j].record(stream)
        with torch.cuda.stream(down):        # step k's results
            down.wait_event(img_ready[j])
            h_out[j].copy_(d_out[j], non_blocking=True)
            img_free[j].record(down)
            down.wait_event(grad_ready[j])
            h_grad[j].copy_(d_grad[j], non_blocking=True)
            grad_free[j].record(down)

    for k in range(2):
        e2e_step(k)
    stream.wait_stream(down)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    for k in range(args.steps):
        e2e_step(k)
    stream.wait_stream(down)
    stream.wait_stream(up)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    h2d = h_vol.numel() * 4 + h_Rt.numel() * 4 + h_go.numel() * 4
    d2h = h_out[0].numel() * 4 + h_grad[0].numel() * 4
    # the last step's downloads against the device-timed step's results (same
    # inputs): the image bit for bit, the gradient up to the atomics' order
    last = (args.steps - 1) & 1
    img_same = bool(torch.equal(h_out[last], ref_out.cpu()))
    g_ref = ref_grad.cpu()
    g_err = float((h_grad[last] - g_ref).abs().max() / g_ref.abs().max().clamp_min(1e-30))
    return {"value": job_throughput(world, w.samples, args.steps, e2e_ms) / 1e9,
            "unit": "Gsamples/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": e2e_ms / args.steps,
            "check": {"image_equal": img_same, "gradient_max_rel_diff": g_err},
            "note": "pipelined over two buffer sets: uploads of step k+1 and downloads of step k "
                    "overlap the kernels; includes the 256 MiB L2 flush write before each step"}


def run_ours(args):
    import torch
    from cone_beam_ct_b200 import drr
    from cone_beam_ct_b200 import workloads as wl

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    drr.lib()

    w = workload(args.config, args.views)
    if args.layout == "auto":
        args.layout = AUTO_LAYOUT[args.config]
    layout = {"padded": drr.DRR_LAYOUT_PADDED, "corners": drr.DRR_LAYOUT_CORNERS,
              "quads": drr.DRR_LAYOUT_QUADS, "linear": drr.DRR_LAYOUT_LINEAR,
              "bricks": drr.DRR_LAYOUT_BRICKS}[args.layout]
    dtype = drr.DRR_BF16 if w.dtype == wl.DTYPE_BF16 else drr.DRR_F32
    elem = 2 if dtype == drr.DRR_BF16 else 4
    nx, ny, nz = w.dims
    vol32 = torch.from_numpy(w.vol).to(dev)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).to(dev)
    grad_out = torch.from_numpy(w.grad_out).to(dev)
    pbytes = drr.drr_prepared_bytes(w.dims, dtype, layout)
    prep = torch.empty(pbytes, dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, w.H, w.W), dtype=torch.float32, device=dev)
    grad = torch.empty((nz, ny, nx), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ws_bytes = drr.drr_adjoint_workspace_bytes(w.dims, w.B)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    fwd_needed = w.mode == wl.MODE_BEER_LAMBERT

    def step(events=None):
        if events:
            events[0].record(stream)
        drr.drr_prepare_volume(vol32, w.dims, dtype, layout, prep, pbytes, stream=stream)
        if events:
            events[1].record(stream)
        drr.drr_render(prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                       w.n_samples, w.density_factor, w.mode, out, stream=stream)
        if events:
            events[2].record(stream)
        grad.zero_()
        if events:
            events[3].record(stream)
        drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                                  w.n_samples, w.density_factor, w.mode, grad_out,
                                  out if fwd_needed else None, grad, ws, ws_bytes, stream=stream)
        if events:
            events[4].record(stream)

    warmup_run = max(args.warmup, 3)          # never time a cold first step
    for _ in range(warmup_run):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    bracket = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu(dev.index)) as clk:
        bracket[0].record(stream)
        for s in range(args.steps):
            flush.fill_(s & 0xFF)
            step(ev[s])
        bracket[1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    per = np.array([[ev[s][i].elapsed_time(ev[s][i + 1]) for i in range(4)]
                    for s in range(args.steps)])          # ms: prepare, forward, zero, adjoint
    step_ms = per.sum(axis=1)
    red = max_over_ranks([float(step_ms.sum())] + list(per.mean(axis=0)), dev)
    total_ms, kern_ms = red[0], np.array(red[1:])
    ms_per_step = total_ms / args.steps
    samples = w.samples
    value = job_throughput(world, samples, args.steps, total_ms) / 1e9
    fps = job_throughput(world, w.B, args.steps, total_ms)

    # e2e through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(torch, drr, w, args, world, dev, stream, flush, dtype, layout, prep, pbytes,
                      ws, ws_bytes, fwd_needed, out, grad)

    # roofline of the dominant kernel
    peaks, peak_src = measured_peaks()
    fwd_ms, adj_ms = float(kern_ms[1]), float(kern_ms[3])
    fwd_bytes = 8 * elem * samples            # 8 voxel reads per sample
    adj_bytes = 8 * 4 * samples               # 8 fp32 atomic adds per sample
    # the bound follows the volume the method reads (n^3 voxels of the storage
    # dtype), not the layout chosen to hold it, so a layout never lowers the bar
    vol_bytes = nx * ny * nz * elem
    vol_fits_l2 = vol_bytes < L2_BYTES
    l2_peak = l2_read_peak_gbs(torch, vol_bytes) if vol_fits_l2 else None
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    def roof(name, ms, nbytes, kernel_key, wname):
        achieved = nbytes / (ms * 1e-3) / 1e9
        if vol_fits_l2 and l2_peak:
            bound, peak, src = "l2", l2_peak, "L2 read probe in this run (libdrr_probe.so)"
        else:
            bound, peak, src = "hbm", hbm_peak, f"MEASURED_PEAKS.json hbm_gbs ({peak_src})"
        return {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": src,
                "frac_of_hbm": achieved / hbm_peak,
                "algorithmic_bytes_per_launch": int(nbytes), "ms_per_launch": ms,
                "traffic": traffic_for(kernel_key, wname, args.layout)}

    wname = config_block(w, args.config)["workload"]
    fwd_roof = roof("forward_kernel", fwd_ms, fwd_bytes, "forward_kernel", wname)
    adj_roof = roof(ADJOINT_GROUP, adj_ms, adj_bytes, "adjoint_kernel", wname)
    # the ceiling of a scatter: the L2's fp32 reduction rate, measured beside
    # the read-bandwidth fraction (8 fp32 values added per ray-sample)
    red = l2_red_probe(torch, nx * ny * nz * 4)
    if red:
        best = max(v["gvalues_s"] for v in red.values())
        adj_roof["red_probe"] = red
        adj_roof["gvalues_s"] = 8 * samples / (adj_ms * 1e-3) / 1e9
        adj_roof["frac_of_best_red_values"] = adj_roof["gvalues_s"] / best
    dominant = adj_roof if adj_ms >= fwd_ms else fwd_roof

    extras = not args.no_extras
    pose = None
    if args.pose or extras:
        pose = pose_timing(torch, w, prep, dtype, layout, Rt, grad_out, out, elem, l2_peak,
                           hbm_peak, vol_fits_l2)

    siddon = None
    if args.siddon or extras:
        siddon = siddon_timing(torch, w, vol32, Rt, grad_out, l2_peak, hbm_peak)

    alpha = None
    if args.alpha or extras:
        alpha = alpha_timing(torch, w, vol32, prep, dtype, layout, Rt, grad_out, elem, l2_peak,
                             hbm_peak, vol_fits_l2)

    batched = None
    if args.batched or extras:
        batched = batched_timing(torch, w, vol32, dtype, layout, Rt, grad_out, elem, l2_peak,
                                 hbm_peak, vol_fits_l2)

    configs = None
    if not args.no_configs:
        l2_cache = {vol_bytes: l2_peak} if vol_fits_l2 else {}
        configs = {str(c): config_timing(torch, c, hbm_peak, l2_cache)
                   for c in OTHER_CONFIGS[args.config]}

    bricks = None
    if extras:
        bricks = bricks_timing(torch, w, vol32, Rt, dtype, w.mode)

    tex = None
    if args.texture:
        tex = texture_comparison(torch, w, vol32, Rt, out)

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(w)

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "Gsamples/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "warmup_run": warmup_run,
        "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": config_block(w, args.config),
        "layout": args.layout,
        "fps": fps,
        "kernels_ms": {"prepare": float(kern_ms[0]), "forward": fwd_ms,
                       "zero_grad (torch)": float(kern_ms[2]), "adjoint": adj_ms},
        "forward": {"gsamples_s": samples / (fwd_ms * 1e-3) / 1e9,
                    "fps": w.B / (fwd_ms * 1e-3), "roofline": fwd_roof},
        "adjoint": {"gsamples_s": samples / (adj_ms * 1e-3) / 1e9, "roofline": adj_roof},
        "roofline": dominant,
        "cpu_baseline": base,
        "e2e": e2e,
        "texture_comparison": tex,
        "pose_gradient": pose,
        "alpha_compositing": alpha,
        "siddon": siddon,
        "batched": batched,
        "configs": configs,
        "bricks": bricks,
        # prepare, forward; adjoint: plan, zero, records, scatter, slab pass
        "gpu_launches": 7 * args.steps,
        "clocks": clocks,
        "bracket_ms": bracket[0].elapsed_time(bracket[1]),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_partitioned(args):
    """One job over all ranks (cone_beam_ct_b200.partition): rank r renders
    and back-projects its share of the detector rows; the volume is broadcast
    from rank 0 once, before timing; every step ends with one NCCL all-reduce
    of the fp32 gradient volume.  value = the whole job's ray-samples per
    second, timed as the max over ranks (strong scaling)."""
    import datetime
    import torch
    import torch.distributed as dist
    from cone_beam_ct_b200 import drr
    from cone_beam_ct_b200 import partition as P
    from cone_beam_ct_b200 import workloads as wl

    world, rank, local = dist_env()
    torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    drr.lib()
    w = workload(args.config, args.views)
    if args.layout == "auto":
        args.layout = AUTO_LAYOUT[args.config]
    layout = {"padded": drr.DRR_LAYOUT_PADDED, "corners": drr.DRR_LAYOUT_CORNERS,
              "quads": drr.DRR_LAYOUT_QUADS, "linear": drr.DRR_LAYOUT_LINEAR,
              "bricks": drr.DRR_LAYOUT_BRICKS}[args.layout]
    dtype = drr.DRR_BF16 if w.dtype == wl.DTYPE_BF16 else drr.DRR_F32
    nx, ny, nz = w.dims
    part = P.Partition(w.B, w.H, w.W, world, rank)
    # the volume lives on rank 0 and reaches the others by one broadcast
    vol32 = (torch.from_numpy(w.vol).to(dev) if rank == 0 else
             torch.empty((nz, ny, nx), dtype=torch.float32, device=dev))
    P.broadcast_volume(vol32)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).to(dev)
    go = torch.from_numpy(np.ascontiguousarray(
        w.grad_out.reshape(-1)[part.local_slice()])).to(dev)
    pbytes = drr.drr_prepared_bytes(w.dims, dtype, layout)
    prep = torch.empty(pbytes, dtype=torch.uint8, device=dev)
    out = torch.empty(max(1, part.rays), dtype=torch.float32, device=dev)
    grad = torch.empty((nz, ny, nx), dtype=torch.float32, device=dev)
    ws = torch.empty(drr.drr_adjoint_workspace_bytes(w.dims, w.B), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    fwd_needed = w.mode == wl.MODE_BEER_LAMBERT

    def step():
        drr.drr_prepare_volume(vol32, w.dims, dtype, layout, prep, pbytes, stream=stream)
        P.render_partitioned(part, prep, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt,
                             w.n_samples, w.density_factor, w.mode, out, stream=stream)
        grad.zero_()
        P.adjoint_partitioned(part, w.dims, w.spacing, w.origin, w.K, Rt, w.n_samples,
                              w.density_factor, w.mode, go, out if fwd_needed else None, grad,
                              workspace=ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total = 0.0
    with ClockSampler(physical_gpu(dev.index)) as clk:
        for s in range(args.steps):
            flush.fill_(s & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks([total], dev)[0]
    # prepare; per call: forward, then plan, zero, records, scatter, slab pass
    launches = 1 + 6 * len(part.segments)
    line = {
        "metric": METRIC, "value": w.samples * args.steps / (total_ms * 1e-3) / 1e9,
        "unit": "Gsamples/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "layout": args.layout,
        "config": dict(config_block(w, args.config),
                       parallelism=f"detector rows split over {world} ranks, volume replicated, "
                                   "gradient all-reduced (NCCL) every step"),
        "fps": w.B * args.steps / (total_ms * 1e-3),
        "rows_per_rank": [P.Partition(w.B, w.H, w.W, world, r).rows for r in range(world)],
        "e2e": None, "cpu_baseline": None, "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.steps < 1 or args.warmup < 0:
        raise SystemExit("--steps must be >= 1 and --warmup >= 0")
    if args.impl == "reference":
        return run_reference(args)
    if args.partition == "views":
        return run_partitioned(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
