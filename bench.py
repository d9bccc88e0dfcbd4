"""Benchmark: SubMConv3d Mvox/s and fraction of roofline at 128^3 / 128 ch / 10 %
occupancy, plus map-build ms (the workload of the lato.2_mrp_mlx README's
"Fleet benchmark": 209,715 voxels, 128 -> 128 channels, warm neighbour map).

One step = ten chained 128 -> 128 bf16 layers over one cached map (ping-pong
buffers), inputs resident in HBM; value = active voxels x layers / step seconds
/ 1e6 (Mvox/s per layer, the pages' unit).  L2 is flushed (a 512 MB write)
between timed steps; each step is timed with CUDA events on the launching stream.
The map build is timed separately (map_build_ms).  e2e repeats the step through
the public API from pinned host buffers: coordinates, features and weights
copied in, map built, ten layers, output copied back.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same workload on its own GPU (replicas; the
layer has no exchange step), times are the max over ranks, value is the sum.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "SubMConv3d Mvox/s and % of roofline at 128^3/128ch/10% occ; map-build ms"
# The pages' own figure for this metric and workload (lato.2_mrp_mlx README, "Fleet
# benchmark": 13.8 ms per layer on an Apple M3 Ultra, 80 GPU cores).  Another
# machine's number: context for vs_baseline, not a target.
PAGES_MVOX = 15.25
PAGES_REF = "Apple M3 Ultra (80 GPU cores), 15.25 Mvox/s, lato.2_mrp_mlx README 'Fleet benchmark'; context only"
UNIT = "Mvox/s"
LAYERS = 10
WORKLOAD = "uniform"
CONFIG = {
    "workload": "SubMConv3d k=3, 128^3 grid, 209,715 active voxels (~10%) uniform without replacement, "
                "batch 1, 128->128 channels, bf16 in / fp32 accumulate, map built once and reused for 10 layers",
    "grid": 128, "voxels": 209715, "cin": 128, "cout": 128, "kernel_size": 3, "layers_per_step": LAYERS,
    "l2": "flushed between timed steps (512 MB write)",
}


# DRAM traffic of one forward launch from the committed ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel
# sources it was taken on: reported as null once their hash changes.
PROFILED_TRAFFIC = {
    "kernel": "k_subm_win<128,128>",
    "bytes": None,
    "sources_sha256": None,
}
KERNEL_SOURCES = ("forward_win.cu", "sm100.cuh", "common.cuh")


def kernel_sources_sha256() -> str:
    """sha256 of the kernel sources' code: comments and whitespace are dropped, so
    an edit of a comment does not retire the measured traffic, a code change does."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "submanifold_sparse_convolution_submconv3d_b200", "csrc", name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def tc_kernel_name(cin: int, cout: int) -> str:
    """The forward kernel instantiation the library dispatches for these channels."""
    bm = 128 if cout % 128 == 0 else 64
    kc = 128 if cin % 128 == 0 else 64 if cin % 64 == 0 else 32 if cin % 32 == 0 else 16
    return f"k_subm_win<{bm},{kc}>"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's x (the slowest rank sets a multi-GPU time);
    every rank must call it, in the same order."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_mvox(world: int, steps: int, layers: int, n: int, total_ms: float) -> float:
    """Whole-job throughput in Mvox/s per layer: every rank processes its own copy
    of the n-voxel workload (replicas), so the units add up over ranks."""
    return world * steps * layers * n / (total_ms / 1e3) / 1e6


def mma_column_efficiency(nbr: np.ndarray, tile_rows: int, bm: int = 128, job_rows: int = 48,
                          n_align: int = 16) -> float:
    """Fraction of the MMA columns the forward issues that carry a real pair.

    Per tile it issues centre jobs of bm rows and, per other offset, jobs of up to
    job_rows compacted hits; each job's MMA N is rounded up to n_align."""
    n = nbr.shape[0]
    t = -(-n // tile_rows)
    hits = np.zeros((t * tile_rows, nbr.shape[1]), dtype=bool)
    hits[:n] = nbr >= 0
    counts = hits.reshape(t, tile_rows, -1).sum(axis=1)  # [tiles, 27]

    def issued(c: np.ndarray, chunk: int) -> int:
        rem = c % chunk
        return int((c // chunk).sum() * chunk + ((rem + n_align - 1) // n_align * n_align).sum())

    centre = nbr.shape[1] // 2
    cols = issued(counts[:, centre], bm)
    for k in range(nbr.shape[1]):
        if k != centre:
            cols += issued(counts[:, k], job_rows)
    return float(hits.sum()) / cols


def roofline_bytes_flops(n: int, pairs: int, cin: int, cout: int) -> tuple[float, float]:
    """Compulsory bytes and useful FLOPs of one k=3 layer: x read once, W once, bias,
    out written once, 4 bytes per non-centre neighbour pair; 2*Cin*Cout per pair."""
    byts = n * cin * 2 + 27 * cin * cout * 2 + cout * 2 + n * cout * 2 + 4 * (pairs - n)
    flops = 2.0 * cin * cout * pairs
    return float(byts), flops


def cpu_baseline(wl, target_s: float = 10.0) -> dict:
    """The CPU oracle (plain C, fp64, one thread), as it stands, on a bounded sample:
    the full neighbour map, then the first layer's forward on a row sample sized for
    about target_s seconds.  Returns Mvox/s per layer = sampled rows / forward seconds."""
    import oracle
    t0 = time.perf_counter()
    nbr = oracle.neighbor_map(wl.coords, wl.grid)
    build_s = time.perf_counter() - t0
    layer = wl.layers[0]
    probe = np.arange(0, min(wl.n, 2000))
    t0 = time.perf_counter()
    oracle.forward(nbr, wl.x, layer.w, layer.bias, rows=probe)
    per_row = max((time.perf_counter() - t0) / len(probe), 1e-9)
    rows = np.arange(0, int(min(wl.n, max(2000, target_s / per_row))))
    t0 = time.perf_counter()
    oracle.forward(nbr, wl.x, layer.w, layer.bias, rows=rows)
    fwd_s = time.perf_counter() - t0
    return {"value": len(rows) / fwd_s / 1e6, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"C oracle (fp64, 1 thread): neighbour map of all {wl.n} voxels in {build_s * 1e3:.0f} ms, "
                      f"then layer 1 forward on the first {len(rows)} of {wl.n} rows in {fwd_s:.2f} s"}


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    wl = workloads.make_workload(WORKLOAD, 0, n_layers=1)
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        b = cpu_baseline(wl, target_s=max(2.0, min(10.0, 60.0 / max(1, args.steps + args.warmup))))
        if i >= args.warmup:
            per_step.append(b["value"])
            base = b
    value = statistics.median(per_step)
    base["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": LAYERS * wl.n / (value * 1e6) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": value / PAGES_MVOX, "vs_baseline_ref": PAGES_REF,
            "dtype": "f64", "data": "synthetic",
            "config": CONFIG, "cpu_baseline": base,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    import submanifold_sparse_convolution_submconv3d_b200 as sp

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    wl = workloads.make_workload(WORKLOAD, 0, n_layers=LAYERS)
    n, cin, cout = wl.n, 128, 128

    coords_h = torch.from_numpy(wl.coords).pin_memory()
    x_h = torch.from_numpy(wl.x).to(torch.bfloat16).pin_memory()
    w_h = [torch.from_numpy(l.w).to(torch.bfloat16).pin_memory() for l in wl.layers]
    b_h = [torch.from_numpy(l.bias).to(torch.bfloat16).pin_memory() for l in wl.layers]
    out_h = torch.empty((n, cout), dtype=torch.bfloat16).pin_memory()

    coords_d = coords_h.to(dev)
    ws = [w.to(dev) for w in w_h]
    bs = [b.to(dev) for b in b_h]
    bufs = [x_h.to(dev), torch.empty((n, cout), dtype=torch.bfloat16, device=dev)]
    x0 = bufs[0].clone()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    m = sp.spconv_build_map(coords_d, wl.grid, 3)
    pairs = m.pairs
    col_eff = mma_column_efficiency(m.neighbor_map().cpu().numpy(), m.tile_rows)

    def step(events=None):
        for i in range(LAYERS):
            src, dst = bufs[i % 2], bufs[(i + 1) % 2]
            if events is not None:
                events[i][0].record(stream)
            sp.spconv_subm_forward(m, src, ws[i], bs[i], out=dst)
            if events is not None:
                events[i][1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        bufs[0].copy_(x0)
        step()
    m.check()

    # ---- timed region: K steps, L2 flushed between them
    visible = [s for s in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if s]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank))
    sampler.start()
    layer_ms, step_ms = [], []
    barrier()
    for _ in range(args.steps):
        bufs[0].copy_(x0)
        flush.fill_(1.0)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(LAYERS)]
        step(ev)
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in ev]
        layer_ms.extend(ms)
        step_ms.append(ev[0][0].elapsed_time(ev[-1][1]))
    barrier()
    clocks = sampler.stop()
    m.check()
    total_ms = sum(step_ms)
    total_ms = max_over_ranks(total_ms, world, dev)
    value = whole_job_mvox(world, args.steps, LAYERS, n, total_ms)

    # ---- map build, timed separately (pack + insert + probe, one host sync inside)
    build_ms = []
    for i in range(max(3, args.steps)):
        flush.fill_(1.0)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        mm = sp.spconv_build_map(coords_d, wl.grid, 3)
        build_ms.append((time.perf_counter() - t0) * 1e3)
        mm.free()

    # ---- e2e through the public API from pinned host memory
    h2d = coords_h.numel() * 4 + x_h.numel() * 2 + sum(w.numel() * 2 for w in w_h) + sum(b.numel() * 2 for b in b_h)
    d2h = out_h.numel() * 2
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush.fill_(1.0)
        barrier()
        t0 = time.perf_counter()
        c_d = coords_h.to(dev, non_blocking=True)
        xa = x_h.to(dev, non_blocking=True)
        wd = [w.to(dev, non_blocking=True) for w in w_h]
        bd = [b.to(dev, non_blocking=True) for b in b_h]
        me = sp.spconv_build_map(c_d, wl.grid, 3)
        xb = torch.empty_like(xa)
        pp = [xa, xb]
        for li in range(LAYERS):
            sp.spconv_subm_forward(me, pp[li % 2], wd[li], bd[li], out=pp[(li + 1) % 2])
        out_h.copy_(pp[LAYERS % 2], non_blocking=True)
        torch.cuda.synchronize()
        dt = (time.perf_counter() - t0) * 1e3
        me.free()
        if i >= args.warmup:
            e2e_ms.append(dt)
    e2e_total = sum(e2e_ms)
    e2e_total = max_over_ranks(e2e_total, world, dev)
    e2e_value = whole_job_mvox(world, args.steps, LAYERS, n, e2e_total)

    if rank != 0:
        return
    hbm, tf_burst, tf_sust, peak_kind = _peaks()
    byts, flops = roofline_bytes_flops(n, pairs, cin, cout)
    avg_launch_s = statistics.mean(layer_ms) / 1e3
    achieved_gbs = byts / avg_launch_s / 1e9
    t_hbm, t_tensor = byts / (hbm * 1e9), flops / (tf_burst * 1e12)
    kname = tc_kernel_name(cin, cout)
    traffic = None
    if kname == PROFILED_TRAFFIC["kernel"] and kernel_sources_sha256() == PROFILED_TRAFFIC["sources_sha256"]:
        traffic = PROFILED_TRAFFIC["bytes"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": value / PAGES_MVOX, "vs_baseline_ref": PAGES_REF, "dtype": "bf16", "data": "synthetic", "config": CONFIG,
        "impl": "ours",
        "layer_ms_mean": statistics.mean(layer_ms), "layer_ms_min": min(layer_ms),
        "layer_ms_median": statistics.median(layer_ms),
        # first layer of every step: L2 was flushed just before it
        "layer_ms_cold_l2_median": statistics.median(layer_ms[0::LAYERS]),
        "map_build_ms": statistics.median(build_ms), "pairs": pairs,
        # build floor: coords read once + one 4-byte index per non-centre pair
        "map_build_floor_gbs": (16 * n + 4 * (pairs - n)) / (statistics.median(build_ms) / 1e3) / 1e9,
        "tile_rows": m.tile_rows, "mma_columns_useful_frac": col_eff,
        "roofline": {"bound": "hbm" if t_hbm >= t_tensor else "tensor", "achieved": achieved_gbs,
                     "peak": hbm, "unit": "GB/s", "frac": achieved_gbs / hbm, "traffic": traffic,
                     "kernel": kname, "algorithmic_bytes_per_launch": byts,
                     "useful_flops_per_launch": flops, "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tensor * 1e6,
                     "frac_of_roofline_time": max(t_hbm, t_tensor) / avg_launch_s,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback"},
        "clocks": clocks,
        "gpu_launches": args.steps * LAYERS,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_total / args.steps,
                "includes": "H2D coords+features+weights, map build, 10 layers, D2H output"},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(workloads.make_workload(WORKLOAD, 0, n_layers=1))
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
