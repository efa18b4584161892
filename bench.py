#!/usr/bin/env python
"""Throughput benchmark of the fused MiMo-V2 preprocessing path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c5] [--dtype f32|bf16]

A step is one call of the C-ABI entry point mimo_preprocess_batch over the
whole batch of the workload (default: 256 images 1080x1920, half RGB / half
RGBA -> 1088x1920, fp32 rows + column-order permutation), with the packed
uint8 inputs already resident in HBM. Timing: W untimed warm-up steps, then K
steps bracketed by barrier + synchronize, CUDA events on the launching stream,
max over ranks. Inputs (1.86 GB) and outputs (12.8 GB fp32) are far larger
than the 126 MB L2, so no flush is needed between steps. Smaller workloads
(c2, c4) are not flushed either; the line's config.l2 says so.

Under torchrun each rank processes its own batch (different seed), with no
collective on the data path: weak scaling.

Also reported on the same JSON line:
  roofline     algorithmic bytes of the kernel (uint8 read + rows written +
               permutation written) / its average event-timed duration,
               against the measured HBM copy bandwidth;
  e2e          the same metric through mimo_preprocess_batch_host: pinned
               host images in, pinned host rows out, copies inside the timing;
  cpu_baseline the CPU oracle timed on a bounded sample of the same workload
               on this host's cores (rank 0, N=1 only);
  clocks       SM clock and throttle reasons sampled through NVML during the
               timed region;
  also         (default c5 fp32 line, one GPU) the two other configurations held
               to the bandwidth target, c5 with bf16 rows and c3 with fp32 rows,
               each timed the same way in this process with its own roofline;
               and the patch embedding on the c5 bf16 rows (tensor roofline,
               cuBLAS on the same operands beside it).

--impl reference times the CPU oracle alone (rank 0; other ranks exit).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "images/s and output HBM GB/s (% of B200 peak) for fused MiMo preprocess"
UNIT = "images/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c5", choices=["c2", "c3", "c4", "c5", "v1", "pe"],
                    help="pe: the patch embedding GEMM on the bf16 rows of c5 (--images sets the image count)")
    ap.add_argument("--embed-dim", type=int, default=1280, help="pe: output width of the patch embedding")
    ap.add_argument("--gemm-only", action="store_true", help="pe: time the GEMM alone (no cuBLAS, no pixel chain)")
    ap.add_argument("--chain-only", action="store_true",
                    help="pe: time only mimo_preprocess_embed (uint8 pixels -> embeddings through a scratch)")
    ap.add_argument("--scratch-mb", type=int, default=192, help="pe: scratch of the chained pixels-to-embeddings call")
    ap.add_argument("--dtype", default=None, choices=["f32", "bf16"])
    ap.add_argument("--images", type=int, default=None, help="override the workload's image count")
    ap.add_argument("--order", default="merge", choices=["merge", "column"], help="row order of the output")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", action="store_true",
                    help="every rank takes the same batch and runs its own merge-unit window of it "
                         "(mimo_preprocess_units): strong scaling of one batch, images split across ranks")
    ap.add_argument("--no-also", action="store_true",
                    help="c5 default line: skip the c3 fp32, c5 bf16 and patch-embedding measurements added "
                         "under 'also'")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step from a CUDA graph (the launch without the host-side call overhead)")
    return ap.parse_args()


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {
    "preprocess": ("vision_lm_image_b200/csrc/mimo_preprocess.cu", "vision_lm_image_b200/csrc/mimo_internal.h"),
    "patch_embed": ("vision_lm_image_b200/csrc/mimo_patch_embed.cu", "vision_lm_image_b200/csrc/mimo_internal.h"),
}


def kernel_source_digest(kernel: str = "preprocess") -> str:
    """Digest of a kernel's source code, comments and blank lines left out (a comment edit does not
    make a capture of the same code stale)."""
    import re

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, dtype: str, kernel: str = "preprocess", rows: int | None = None,
                images: int | None = None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel source.

    An entry with a per-image slope and a fixed offset (two captures of different
    sizes) is evaluated at ``images``; an entry captured on a smaller case than
    the launch timed here (``full_rows`` differs from ``rows``) is scaled by rows;
    an entry captured on the whole workload applies only to that workload."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    entry = d.get(f"{workload}_{dtype}")
    if not entry or entry.get("kernel_digest") != kernel_source_digest(kernel):
        return None
    traffic = entry.get("dram_bytes_per_launch")
    if "per_image" in entry:
        if images is not None:
            traffic = int(round(entry["per_image"] * images + entry["offset"]))
        return traffic
    if "full_rows" not in entry and images is not None and entry.get("full_images", images) != images:
        return None
    if rows is not None and entry.get("full_rows") and entry["full_rows"] != rows:
        traffic = int(round(traffic * rows / entry["full_rows"]))
    return traffic


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
            bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            for b, name in self.REASONS.items():
                if bits & b:
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.nv is not None:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(s)}


L2_BYTES = 126 * 1000 * 1000  # B200 L2 cache (nominal)


def l2_note(input_bytes: int, output_bytes: int) -> str:
    """How a workload's timed steps stand to the L2 cache; no timing loop here flushes it."""
    if input_bytes > L2_BYTES:
        return "inputs (%.2f GB) and outputs (%.2f GB) larger than L2 (no flush)" % (input_bytes / 1e9,
                                                                                   output_bytes / 1e9)
    return ("inputs (%.1f MB) smaller than the 126 MB L2 and not flushed between steps: they may stay partly "
            "L2-resident; outputs %.1f MB" % (input_bytes / 1e6, output_bytes / 1e6))


def workload_config(args, w, world: int, n_img: int, out_dtype: str, column_perm: bool, total_rows: int,
                    input_bytes: int) -> dict:
    """The line's config: the same keys and values on both arms (the reference arm computes the rows
    with the oracle's geometry, this arm with the library's; the tests hold the two equal)."""
    out_bytes = int(total_rows) * 1536 * (2 if out_dtype == "bf16" else 4) + (4 * int(total_rows) if column_perm else 0)
    return {"workload": args.workload, "description": w["description"], "images_per_gpu": n_img,
            "out_dtype": out_dtype, "column_perm": column_perm, "rows_per_gpu": int(total_rows),
            "row_order": args.order, "launch": "cuda_graph" if args.graph else "api_call",
            "l2": l2_note(input_bytes, out_bytes),
            "parallelism": f"dp{world}" + (" merge-unit windows of one batch" if getattr(args, "shard", False) else "")}


def algorithmic_bytes(packed, total_rows, dtype_bytes, perm: bool) -> dict:
    read = int(sum(int(h) * int(w) * int(c) for h, w, c in zip(packed.heights, packed.widths, packed.channels)))
    write_rows = int(total_rows) * 1536 * dtype_bytes
    write_perm = int(total_rows) * 4 if perm else 0
    return {"read": read, "write_rows": write_rows, "write_perm": write_perm,
            "total": read + write_rows + write_perm}


def cpu_baseline(w, sample_images: int, threads: int, min_seconds: float = 0.0):
    """Images/s of the oracle on the first `sample_images` images, repeating passes until at least
    `min_seconds` of work (one pass when 0)."""
    import oracle

    imgs = w["images"][:sample_images]
    oracle.build()
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.preprocess(imgs, w["mean"], w["std"], column_perm=w["column_perm"], threads=threads)
        done += len(imgs)
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            return done / dt, dt


def dominant_kernel(grid, heights, widths, out_dtype: str, video: bool = False) -> str:
    """The pixel kernel a launch runs, by the library's dispatch rule: for images, the warp-staged
    warp_kernel when every height shrinks by 1.25 or more and no axis gathers its taps (a shrink of
    about 1.94 or more gathers); else the unstaged direct_kernel when every width is kept and either
    the rows are bf16, or every height is kept too, or the launch is a video; else the staged
    preprocess_kernel."""
    import numpy as np

    grid = np.asarray(grid)
    h, w = np.asarray(heights, dtype=np.int64), np.asarray(widths, dtype=np.int64)
    hr, wr = grid[:, 1].astype(np.int64) * 16, grid[:, 2].astype(np.int64) * 16
    shrunk = bool(np.all(4 * h >= 5 * hr))
    gather = bool(np.any(32 * h > 62 * hr) or np.any(32 * w > 62 * wr))
    if shrunk and not gather and not video:
        return "warp_kernel"
    widths_kept = bool(np.all(wr == w))
    heights_kept = bool(np.all(hr == h))
    return ("direct_kernel" if widths_kept and (out_dtype == "bf16" or heights_kept or video)
            else "preprocess_kernel")


def image_cpu_baseline(w, n_img: int, cores: int, min_seconds: float = 10.0, single_seconds: float = 5.0) -> dict:
    """The oracle on `cores` host threads over the first 64 images (the reported baseline), plus a
    single-threaded figure over the first 8."""
    sample_n = max(1, min(n_img, 64))
    v, dt = cpu_baseline(w, sample_n, cores, min_seconds=min_seconds)
    single_n = max(1, min(n_img, 8))
    v1, dt1 = cpu_baseline(w, single_n, 1, min_seconds=single_seconds)
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {sample_n} of the {n_img} workload images, passes repeated for {dt:.1f} s",
            "single_thread": {"value": v1, "unit": UNIT, "cores": 1,
                              "sample": f"first {single_n} images, passes repeated for {dt1:.1f} s"}}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference_other(args, world):
    """The oracle on the video clip (frames/s) or on the patch embedding (tokens/s)."""
    import numpy as np

    import oracle
    import workloads

    oracle.build()
    cores = host_cores()
    if args.workload == "v1":
        # a bounded sample: the first 4 frames of the clip (two temporal patches) per step
        w = workloads.video_workload("v1", n_frames=4)
        run = lambda: oracle.preprocess_video(w["frames"], w["mean"], w["std"], total_max_pixels=w["total_max_pixels"])
        units, unit, sample = 4, "frames/s", "first 4 frames of the 64-frame clip per step, oracle on 1 thread"
        metric = METRIC + " (video frames)"
    else:
        # a bounded sample: 256 rows of the embedding per step, fp64 on one thread
        rng = np.random.Generator(np.random.PCG64(17))
        a = rng.standard_normal((256, 1536)).astype(np.float32)
        wt = (rng.standard_normal((args.embed_dim, 1536)) * 0.02).astype(np.float32)
        run = lambda: oracle.patch_embed(a, wt)
        units, unit, sample = 256, "tokens/s", "256 rows x 1536 -> embed_dim per step, fp64 on 1 thread"
        metric = "patch-embedding tokens/s (Conv3d 3x2x16x16 -> embed_dim as a bf16 GEMM)"
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    t = time.perf_counter() - t0
    value = units * args.steps / t
    print(json.dumps({
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload},
        "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference(args, rank, world):
    import workloads

    if rank != 0:
        return
    if args.workload in ("v1", "pe"):
        run_reference_other(args, world)
        return
    w = workloads.workload(args.workload, n_images=args.images)
    if args.dtype:
        w["dtype"] = args.dtype
    import oracle

    oracle.build()
    total_rows = sum(oracle.get_number_of_image_patches(im.shape[0], im.shape[1]) for im in w["images"])
    input_bytes = sum(int(im.size) for im in w["images"])
    config = workload_config(args, w, world, len(w["images"]), w["dtype"], bool(w["column_perm"]), total_rows,
                             input_bytes)
    cores = host_cores()
    per_step = max(1, min(len(w["images"]), 2 * cores, 16))
    sample = f"{per_step} of the workload's {len(w['images'])} images per step, oracle on {cores} threads"
    for _ in range(args.warmup):
        cpu_baseline(w, per_step, cores)
    t = 0.0
    for _ in range(args.steps):
        _, dt = cpu_baseline(w, per_step, cores)
        t += dt
    value = per_step * args.steps / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_video(args, rank, world, local_rank):
    """Frames/s of the video path (one clip per rank, frames resident in HBM)."""
    import numpy as np
    import torch

    import workloads
    from vision_lm_image_b200 import mimo

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.video_workload(args.workload, seed_offset=7919 * rank, n_frames=args.images)
    frames = w["frames"]
    n, H, W, C = frames.shape
    out_dtype = args.dtype or w["dtype"]
    tdtype = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    params = mimo.make_params(w["mean"], w["std"])
    stride = (H * W * C + 15) // 16 * 16
    d_frames = torch.zeros(n * stride, dtype=torch.uint8, device=dev)
    d_frames.view(n, stride)[:, :H * W * C].copy_(torch.from_numpy(frames.reshape(n, -1)))
    grid, rows = mimo.plan_video(n, H, W, w["total_max_pixels"], params)
    out = torch.empty((rows, 1536), dtype=tdtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mimo.preprocess_video_raw(params, d_frames, n, stride, H, W, C, out, w["total_max_pixels"],
                                  order=args.order, stream=stream)

    for _ in range(max(args.warmup, 0)):
        step()
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    read = n * H * W * C
    written = rows * 1536 * (2 if out_dtype == "bf16" else 4)
    peak, peak_kind = measured_hbm_peak()
    achieved = (read + written) / (ms / K * 1e-3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": METRIC + " (video frames)", "value": world * n * K / (ms * 1e-3), "unit": "frames/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": out_dtype, "data": "synthetic",
            "config": {"workload": args.workload, "description": w["description"], "frames": int(n),
                       "grid_thw": [int(v) for v in grid], "out_dtype": out_dtype, "row_order": args.order,
                       "l2": l2_note(read, written)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind, "traffic": None, "algorithmic_bytes_per_launch": read + written,
                         "kernel": dominant_kernel([grid], [H], [W], out_dtype, video=True), "avg_launch_ms": ms / K},
            "gpu_launches": K, "clocks": clocks.summary(), "e2e": None, "cpu_baseline": None,
        }), flush=True)


def compare_patch_embed(args, mimo, w, dev, rows, weight, bias, out, err, stream, timed):
    """cuBLAS on the same operands, and pixels -> embeddings as two calls vs the chunked entry point."""
    import torch

    out_ref = torch.empty_like(out)
    lib_step = lambda: torch.addmm(bias.to(torch.bfloat16), rows, weight.t(), out=out_ref)
    for _ in range(max(args.warmup, 0)):
        lib_step()
    lib_ms = timed(lib_step, args.steps)
    # the whole chain from uint8 pixels: two calls over the batch vs the chunked entry point
    params = mimo.make_params(w["mean"], w["std"])
    packed = mimo.pack_images(w["images"], device=dev)
    scratch = torch.empty(args.scratch_mb << 20, dtype=torch.uint8, device=dev)
    two = lambda: (mimo.preprocess_batch_ex(params, packed, rows, None, stream=stream),
                   mimo.patch_embed(rows, weight, bias, out=out, error=err, stream=stream, check=False))
    chain = lambda: mimo.preprocess_embed(packed, weight, bias, w["mean"], w["std"], scratch=scratch, stream=stream,
                                          check=False)
    for _ in range(max(args.warmup, 0)):
        two()
        chain()
    two_ms = timed(two, args.steps)
    chain_ms = timed(chain, args.steps)
    return lib_ms, two_ms, chain_ms


def run_chain_only(args, mimo, w, dev, rank, world):
    """Images/s of mimo_preprocess_embed alone: uint8 pixels resident in HBM to bf16 embeddings, the bf16
    rows passing through a scratch of --scratch-mb (what an ncu capture of this command sees is exactly
    the chained call's kernels)."""
    import torch

    params = mimo.make_params(w["mean"], w["std"])
    packed = mimo.pack_images(w["images"], device=dev)
    N = args.embed_dim
    g = torch.Generator(device="cpu").manual_seed(17 + rank)
    weight = (torch.randn((N, 1536), generator=g) * 0.02).to(torch.bfloat16).to(dev)
    bias = torch.randn(N, generator=g).to(dev)
    scratch = torch.empty(args.scratch_mb << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    _, offs = mimo.plan_batch(packed.heights, packed.widths, params)
    M = int(offs[-1])
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    chain = lambda: mimo.preprocess_embed(packed, weight, bias, w["mean"], w["std"], scratch=scratch, stream=stream,
                                          out=out, error=err, check=False)
    for _ in range(max(args.warmup, 0)):
        chain()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            chain()
        e1.record(stream)
        torch.cuda.synchronize()
    if int(err.item()):
        raise SystemExit(f"patch_embed reported pipeline error {int(err.item())}")
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    n_img = len(w["images"])
    flops = 2.0 * M * N * 1536
    if rank == 0:
        print(json.dumps({
            "metric": "pixels-to-embeddings images/s (mimo_preprocess_embed)", "value": world * n_img / (ms * 1e-3),
            "unit": "images/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "pe_chain", "images": n_img, "rows": M, "embed_dim": N,
                       "scratch_mb": args.scratch_mb},
            "tflops": flops / (ms * 1e-3) / 1e12, "clocks": clocks.summary(), "e2e": None, "cpu_baseline": None,
        }), flush=True)


def run_patch_embed(args, rank, world, local_rank):
    """Tokens/s of the tensor-core patch embedding on the bf16 rows of the c5 batch (rows resident in HBM)."""
    import numpy as np
    import torch

    import workloads
    from vision_lm_image_b200 import mimo

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.workload("c5", seed_offset=7919 * rank, n_images=args.images)
    if args.chain_only:
        run_chain_only(args, mimo, w, dev, rank, world)
        return
    rows, _, _ = mimo.preprocess(w["images"], w["mean"], w["std"], dtype=torch.bfloat16, device=dev)
    M, K, N = rows.shape[0], rows.shape[1], args.embed_dim
    g = torch.Generator(device="cpu").manual_seed(17 + rank)
    weight = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16).to(dev)
    bias = torch.randn(N, generator=g).to(dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for _ in range(steps):
            fn()
        ev[1].record(stream)
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1]) / steps

    step = lambda: mimo.patch_embed(rows, weight, bias, out=out, error=err, stream=stream, check=False)
    for _ in range(max(args.warmup, 0)):
        step()
    with ClockSampler(local_rank) as clocks:
        ms = timed(step, args.steps)
    code = int(err.item())
    if code:
        raise SystemExit(f"patch_embed reported pipeline error {code}")
    lib_ms = two_ms = chain_ms = float("nan")
    n_img = len(w["images"])
    if not args.gemm_only:
        lib_ms, two_ms, chain_ms = compare_patch_embed(args, mimo, w, dev, rows, weight, bias, out, err, stream, timed)
    flops = 2.0 * M * N * K
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        peak, peak_sus, kind = float(pk["bf16_tflops"]), float(pk["bf16_tflops_sustained"]), "measured"
    except Exception:
        peak, peak_sus, kind = 1590.0, 1400.0, "fallback"
    achieved = flops / (ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        oracle.build()
        sample = 256
        a = rows[:sample].float().cpu().numpy()
        wt = weight.float().cpu().numpy()
        bb = bias.cpu().numpy()
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 10.0:
            oracle.patch_embed(a, wt, bb)
            done += sample
        dt = time.perf_counter() - t0
        cpu = {"value": done / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"first {sample} of {M} rows, passes repeated for {dt:.1f} s, single thread"}
    if rank == 0:
        print(json.dumps({
            "metric": "patch-embedding tokens/s (Conv3d 3x2x16x16 -> embed_dim as a bf16 GEMM)",
            "value": world * M / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "pe", "description": f"bf16 rows of c5 ({M} x {K}) x weight [{N}, {K}] + bias "
                       f"-> bf16 [{M}, {N}]", "rows": M, "embed_dim": N, "K": K,
                       "l2": "rows (%.1f GB) and output larger than L2 (no flush)" % (M * K * 2 / 1e9)},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "frac_of_sustained": achieved / peak_sus, "peak_kind": kind,
                         "traffic": ncu_traffic("pe", "bf16", "patch_embed", M),
                         "algorithmic_flops_per_launch": flops, "kernel": "patch_embed_kernel",
                         "algorithmic_bytes_per_launch": M * K * 2 + N * K * 2 + N * 4 + M * N * 2,
                         "avg_launch_ms": ms},
            "library_gemm": None if args.gemm_only else {
                "impl": "torch.addmm (cuBLAS)", "ms": lib_ms, "tflops": flops / (lib_ms * 1e-3) / 1e12},
            "pixels_to_embeddings": None if args.gemm_only else {"images": n_img, "two_calls_ms": two_ms, "chained_ms": chain_ms,
                                     "two_calls_images_per_s": n_img / (two_ms * 1e-3),
                                     "chained_images_per_s": n_img / (chain_ms * 1e-3), "scratch_mb": args.scratch_mb},
            "gpu_launches": args.steps, "clocks": clocks.summary(), "e2e": None, "cpu_baseline": cpu,
        }), flush=True)


def also_config(args, mimo, workloads, name: str, out_dtype: str, dev, stream, scratch) -> dict:
    """One more configuration timed like the main line (W warm-up launches, then K launches between CUDA
    events on the launching stream), its rows written into `scratch` (the main line's output buffer,
    reinterpreted), with its own roofline."""
    import torch

    w = workloads.workload(name)
    tdtype = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    dbytes = 2 if out_dtype == "bf16" else 4
    params = mimo.make_params(w["mean"], w["std"])
    host = mimo.pack_images(w["images"], device="cpu", pin_memory=True)
    packed = host.to(dev)
    grid, offs = mimo.plan_batch(host.heights, host.widths, params)
    total = int(offs[-1])
    flat = scratch.view(torch.uint8).view(-1)
    need = total * 1536 * dbytes + (4 * total if w["column_perm"] else 0)
    assert need <= flat.numel(), "scratch too small"
    out = flat[:total * 1536 * dbytes].view(tdtype).view(total, 1536)
    perm = flat[total * 1536 * dbytes:need].view(torch.int32) if w["column_perm"] else None
    launches = (host.n + 511) // 512
    for _ in range(max(args.warmup, 0)):
        mimo.preprocess_batch_ex(params, packed, out, perm, order=args.order, stream=stream)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with ClockSampler(dev.index) as clocks:
        ev[0].record(stream)
        for _ in range(args.steps):
            mimo.preprocess_batch_ex(params, packed, out, perm, order=args.order, stream=stream)
        ev[1].record(stream)
        torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / args.steps
    nbytes = algorithmic_bytes(host, total, dbytes, perm is not None)
    peak, peak_kind = measured_hbm_peak()
    achieved = nbytes["total"] / (ms / launches * 1e-3) / 1e9
    del packed
    return {"workload": name, "description": w["description"], "images": host.n, "out_dtype": out_dtype,
            "column_perm": perm is not None, "rows": total, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "value": host.n / (ms * 1e-3), "unit": UNIT,
            "l2": l2_note(nbytes["read"], nbytes["write_rows"] + nbytes["write_perm"]),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "traffic": ncu_traffic(name, out_dtype, images=host.n),
                         "algorithmic_bytes_per_launch": nbytes["total"] // launches,
                         "kernel": dominant_kernel(grid, host.heights, host.widths, out_dtype),
                         "avg_launch_ms": ms / launches},
            "gpu_launches": args.steps * launches, "clocks": clocks.summary()}


def also_patch_embed(args, mimo, w, dev, stream, scratch) -> dict:
    """The patch embedding on the bf16 rows of the same c5 batch `w` (W warm-up launches, then K launches
    timed with CUDA events), with cuBLAS on the same operands in the same process for context: the K
    launches of each run in four alternating parts, so that both see the same clock. The rows and the
    embeddings live in `scratch` (the main line's output buffer)."""
    import torch

    params = mimo.make_params(w["mean"], w["std"])
    host = mimo.pack_images(w["images"], device="cpu", pin_memory=True)
    packed = host.to(dev)
    _, offs = mimo.plan_batch(host.heights, host.widths, params)
    M, K, N = int(offs[-1]), 1536, args.embed_dim
    flat = scratch.view(torch.uint8).view(-1)
    assert (M * K + M * N) * 2 <= flat.numel(), "scratch too small"
    rows = flat[:M * K * 2].view(torch.bfloat16).view(M, K)
    out = flat[M * K * 2:(M * K + M * N) * 2].view(torch.bfloat16).view(M, N)
    mimo.preprocess_batch_ex(params, packed, rows, None, stream=stream)
    del packed
    g = torch.Generator(device="cpu").manual_seed(17)
    weight = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16).to(dev)
    bias = torch.randn(N, generator=g).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def interleaved(fns, rounds=4):
        # W warm-up launches of each, then K launches of each in `rounds` alternating runs between CUDA
        # events: a clock that drifts under the power cap during the measurement weighs on both alike
        for fn in fns:
            for _ in range(max(args.warmup, 0)):
                fn()
        torch.cuda.synchronize()
        runs = [args.steps // rounds + (1 if r < args.steps % rounds else 0) for r in range(rounds)]
        total = [0.0] * len(fns)
        for n in runs:
            for i, fn in enumerate(fns):
                if n == 0:
                    continue
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                ev[0].record(stream)
                for _ in range(n):
                    fn()
                ev[1].record(stream)
                torch.cuda.synchronize()
                total[i] += ev[0].elapsed_time(ev[1])
        return [t / args.steps for t in total]

    bias16 = bias.to(torch.bfloat16)
    with ClockSampler(dev.index) as clocks:
        ms, lib_ms = interleaved([
            lambda: mimo.patch_embed(rows, weight, bias, out=out, error=err, stream=stream, check=False),
            lambda: torch.addmm(bias16, rows, weight.t(), out=out)])
    if int(err.item()):
        raise SystemExit(f"patch_embed reported pipeline error {int(err.item())}")
    flops = 2.0 * M * N * K
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        peak, kind = float(pk["bf16_tflops"]), "measured"
    except Exception:
        peak, kind = 1590.0, "fallback"
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": "pe", "description": f"bf16 rows of c5 ({M} x {K}) x weight [{N}, {K}] + bias -> bf16 "
            f"[{M}, {N}]", "rows": M, "embed_dim": N, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "value": M / (ms * 1e-3), "unit": "tokens/s",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_kind": kind,
                         "traffic": ncu_traffic("pe", "bf16", "patch_embed", M),
                         "algorithmic_flops_per_launch": flops, "kernel": "patch_embed_kernel",
                         "avg_launch_ms": ms},
            "library_gemm": {"impl": "torch.addmm (cuBLAS)", "ms": lib_ms,
                             "tflops": flops / (lib_ms * 1e-3) / 1e12},
            "timing": "K launches of each in 4 alternating runs", "gpu_launches": args.steps,
            "clocks": clocks.summary()}


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import workloads
    from vision_lm_image_b200 import build as _build
    from vision_lm_image_b200 import mimo

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    if not os.path.exists(_build.LIB_PATH):
        _build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # weak scaling: each rank its own batch; --shard: one batch, a merge-unit window per rank
    w = workloads.workload(args.workload, seed_offset=0 if args.shard else 7919 * rank, n_images=args.images)
    out_dtype = args.dtype or w["dtype"]
    tdtype = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    dbytes = 2 if out_dtype == "bf16" else 4
    params = mimo.make_params(w["mean"], w["std"])
    host = mimo.pack_images(w["images"], device="cpu", pin_memory=True)
    packed = host.to(dev)
    grid, offs = mimo.plan_batch(host.heights, host.widths, params)
    total = int(offs[-1])
    window = None
    if args.shard:
        from vision_lm_image_b200 import shard

        if args.order != "merge":
            raise SystemExit("--shard runs merge order only")
        window = shard.unit_windows(total // 4, world)[rank]
    out_rows = 4 * window[1] if window else total
    out = torch.empty((out_rows, 1536), dtype=tdtype, device=dev)
    perm = torch.empty(total, dtype=torch.int32, device=dev) if w["column_perm"] else None
    n_img = host.n
    launches_per_step = (n_img + 511) // 512
    stream = torch.cuda.current_stream(dev)

    def launch(on=None):
        if window:
            mimo.preprocess_units(params, packed, window[0], window[1], out, perm, stream=on)
        else:
            mimo.preprocess_batch_ex(params, packed, out, perm, order=args.order, stream=on)

    def step():
        launch(stream)

    graph = None
    if args.graph:
        # capture one step (planning and validation run once, at capture); replays launch the same kernels
        step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            launch()
        step = graph.replay

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        ev[0].record(stream)
        for k in range(K):
            step()
            ev[k + 1].record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    per_launch_ms = [ev[k].elapsed_time(ev[k + 1]) for k in range(K)]
    elapsed_ms = ev[0].elapsed_time(ev[K])
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())

    nbytes = algorithmic_bytes(host, total, dbytes, perm is not None)
    if window:
        # this rank's share: its window's rows and permutation entries, and each touched image's bytes
        # in proportion to the image's units inside the window
        lo, hi = 4 * window[0], 4 * (window[0] + window[1])
        read = 0.0
        for i in range(n_img):
            inside = max(0, min(hi, int(offs[i + 1])) - max(lo, int(offs[i])))
            read += int(host.heights[i]) * int(host.widths[i]) * int(host.channels[i]) * inside / max(
                int(offs[i + 1] - offs[i]), 1)
        rows_w = 4 * window[1]
        nbytes = {"read": int(read), "write_rows": rows_w * 1536 * dbytes,
                  "write_perm": 4 * rows_w if perm is not None else 0}
        nbytes["total"] = nbytes["read"] + nbytes["write_rows"] + nbytes["write_perm"]
    avg_launch_ms = sum(per_launch_ms) / K / launches_per_step
    peak, peak_kind = measured_hbm_peak()
    achieved = nbytes["total"] / (avg_launch_ms * 1e-3) / 1e9
    # whole-job images/s: every rank's own batch (weak), or the one shared batch (--shard)
    value = (1 if window else world) * n_img * K / (max_ms * 1e-3)
    out_gbs = nbytes["write_rows"] / (max_ms / K * 1e-3) / 1e9

    # e2e: host images in, host rows out, through the host-buffer entry point
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0 and not window:
        # with several ranks on one host each rank pins a 64-image prefix of its batch (the full batch
        # would pin ~15 GB of host memory per rank); images/s is per image either way
        e2e_n = n_img if world == 1 else min(n_img, 64)
        host_e = host if e2e_n == n_img else mimo.pack_images(w["images"][:e2e_n], device="cpu", pin_memory=True)
        rows_e = total if e2e_n == n_img else int(mimo.plan_batch(host_e.heights, host_e.widths, params)[1][-1])
        out_h = torch.empty((rows_e, 1536), dtype=tdtype, pin_memory=True)
        perm_h = torch.empty(rows_e, dtype=torch.int32, pin_memory=True) if perm is not None else None
        mimo.preprocess_batch_host(params, host_e, out_h, perm_h, packed.buffer, out, perm, stream)  # warm-up
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            mimo.preprocess_batch_host(params, host_e, out_h, perm_h, packed.buffer, out, perm, stream)
        torch.cuda.synchronize()
        e2e_s = time.perf_counter() - t0
        te = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.barrier()
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": world * e2e_n * args.e2e_steps / float(te.item()), "unit": UNIT,
               "images_per_rank": e2e_n,
               "h2d_bytes_per_step": int(host_e.buffer.numel()),
               "d2h_bytes_per_step": int(out_h.numel() * out_h.element_size()
                                         + (perm_h.numel() * 4 if perm_h is not None else 0)),
               "timing": "host wall clock around the synchronous host-to-host call"}
        del out_h, perm_h, host_e

    # the other configurations held to the bandwidth target, timed in this process on one GPU
    also = None
    if (world == 1 and args.workload == "c5" and args.dtype is None and args.images is None and not args.no_also
            and not args.shard):
        del packed
        also = {"c5_bf16": also_config(args, mimo, workloads, "c5", "bf16", dev, stream, out),
                "c3_f32": also_config(args, mimo, workloads, "c3", "f32", dev, stream, out),
                "pe_bf16": also_patch_embed(args, mimo, w, dev, stream, out)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = image_cpu_baseline(w, n_img, host_cores())

    if dist is not None:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "strong" if window else "weak",
            "vs_baseline": None, "dtype": out_dtype, "data": "synthetic",
            "config": workload_config(args, w, world, n_img, out_dtype, perm is not None, total,
                                      algorithmic_bytes(host, total, dbytes, False)["read"]),
            "output_gbs": out_gbs,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "traffic": ncu_traffic(args.workload, out_dtype, images=n_img) if window is None else None,
                         "algorithmic_bytes_per_launch": nbytes["total"] // launches_per_step,
                         "kernel": dominant_kernel(grid, host.heights, host.widths, out_dtype),
                         "avg_launch_ms": avg_launch_ms},
            "gpu_launches": K * launches_per_step,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        if also:
            line["also"] = also
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.impl == "reference" else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload == "pe":
        run_patch_embed(args, rank, world, local_rank)
    elif args.workload.startswith("v"):
        run_video(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
