"""Throughput bench of the NVFP4 quantizer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...)

One step is one pass of the whole hot path over one tensor resident in HBM:
    nvfp4_amax -> nvfp4_quantize (Four Over Six, MSE rule: codes, scales, tensor scale,
    choice bits) -> nvfp4_dequantize,
on the 1 GiB workload: BF16 65536 x 8192, N(0,1), 1% zero blocks, 1% blocks x1e-6.
Each rank quantizes its own tensor (weak scaling, no collective on the data path).
`value` is input GB/s over all ranks: ranks * 2 * numel / (max over ranks of step time).

Rank 0 prints one JSON line with the roofline of the dominant kernel (quantize), measured
live with CUDA events; the end-to-end number through the public API with host buffers;
the Four Over Six overhead against scale-6 on the same GPU; and the CPU oracle timed on a
bounded sample of the same workload. `--impl reference` times the CPU oracle alone.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "c5"
MODE, RULE = 1, 2                      # Four Over Six, MSE
GB = 1e9


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle leg")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--rows", type=int, default=None,
                    help="rows of the 65536 x 8192 workload to use (default: all; smaller slices for tests)")
    return ap.parse_args()


# ---- distributed plumbing -------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- clocks during the timed region ---------------------------------------------------------

class ClockSampler:
    """Polls NVML (SM clock, max clock, throttle reasons) every few ms in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _poll(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
            bits = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for k, name in self.REASONS.items():
                if bits & k:
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.nvml:
            self._sample()
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nvml:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---- the workload ---------------------------------------------------------------------------

def algorithmic_bytes(n: int, groups: int):
    nb = n // 16
    q = 2 * n + n // 2 + nb + (nb + 7) // 8 + 8 * groups     # read x + amax; write codes, scales, choice, tscale
    return {"amax": 2 * n + 4 * groups, "quantize": q, "dequantize": n // 2 + nb + 4 * groups + 2 * n}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def ncu_traffic(kernel: str):
    """Per-launch DRAM traffic of `kernel` from the committed ncu summary, or None when the
    kernel's source changed after the capture (the summary stores the source hash)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = b""
    for f in ("kernels.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "nvfp4_block_scaled_13_b200", "csrc", f), "rb") as fh:
            src += fh.read()
    h = hashlib.sha256(src).hexdigest()[:16]
    vals = {}
    with open(path) as f:
        for ln in f:
            if ":" in ln and not ln.startswith("#"):
                k, v = ln.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != h:
        return None
    v = vals.get(f"{kernel}_bytes_per_launch")
    return float(v) if v else None


def make_input(rank: int, rows=None):
    from nvfp4_block_scaled_13_b200 import synth

    cfg = synth.CONFIGS[WORKLOAD]
    seed = cfg.seed + 1000 * rank
    x, shape = synth.make(WORKLOAD, rows=rows, seed=seed)
    return x, shape


# ---- CPU oracle legs -----------------------------------------------------------------------

def oracle_step(x_rows: np.ndarray, rows: int, cols: int):
    import oracle as O

    a = O.amax(x_rows, 1, rows, cols)
    q = O.quantize(x_rows, 1, rows, cols, a, MODE, RULE)
    O.dequantize(q["codes"], q["scales"], q["tscale"], 1, rows, cols)


def cpu_baseline(x: np.ndarray, cols: int, rows: int = 12288):
    """The oracle as it stands (C, one thread) on the first `rows` rows of the workload."""
    xs = np.ascontiguousarray(x[: rows * cols])
    t0 = time.perf_counter()
    oracle_step(xs, rows, cols)
    dt = time.perf_counter() - t0
    return {"value": round(2 * rows * cols / dt / GB, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of the 65536x8192 tensor ({rows * cols / 1e6:.1f} M elements): "
                      f"amax + 4/6-MSE quantize + dequantize, single thread, {dt:.1f} s",
            "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on the machine's host cores (rank 0 only)."""
    if rank != 0:
        return
    x, (g, r, c) = make_input(0, args.rows)
    # calibrate, then size each step's sample so that the whole run takes about two minutes
    cal_rows = 64
    t0 = time.perf_counter()
    oracle_step(np.ascontiguousarray(x[: cal_rows * c]), cal_rows, c)
    per_row = (time.perf_counter() - t0) / cal_rows
    rows = int(max(1, min(4096, r // 2, 120.0 / max(1, args.steps + args.warmup) / per_row)))
    for i in range(args.warmup):
        s = (i * rows) % (r - rows)
        oracle_step(np.ascontiguousarray(x[s * c:(s + rows) * c]), rows, c)
    t0 = time.perf_counter()
    for i in range(args.steps):
        s = ((args.warmup + i) * rows) % (r - rows)
        oracle_step(np.ascontiguousarray(x[s * c:(s + rows) * c]), rows, c)
    dt = time.perf_counter() - t0
    value = 2 * rows * c * args.steps / dt / GB
    sample = f"{rows} rows x 8192 per step ({rows * c / 1e6:.2f} M elements): amax + 4/6-MSE quantize + dequantize"
    print(json.dumps({
        "impl": "reference", "metric": "NVFP4 quantize input GB/s & % of B200 HBM peak; 4/6 overhead vs scale-6",
        "value": round(value, 6), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"c5: BF16 {r}x{c} N(0,1), 1% zero blocks, 1% blocks x1e-6; "
                               "Four Over Six, MSE rule", "shape": [1, r, c], "step": "amax + quantize + dequantize"},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---- GPU legs ------------------------------------------------------------------------------

def run_ours(args, rank, world, local):
    import torch

    import nvfp4_block_scaled_13_b200 as nv

    nv.load()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    x_np, (g, r, c) = make_input(rank, args.rows)
    n, nb = g * r * c, g * r * c // 16
    xd = torch.from_numpy(x_np.view(np.int16)).to(dev)
    amax = torch.empty(g, dtype=torch.float32, device=dev)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(nb, dtype=torch.uint8, device=dev)
    tscale = torch.empty(g, dtype=torch.float32, device=dev)
    choice = torch.empty((nb + 7) // 8, dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=torch.int16, device=dev)
    s = stream.cuda_stream

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        nv.nvfp4_amax(xd, g, r, c, amax, s)
        if ev is not None:
            ev[1].record(stream)
        nv.nvfp4_quantize(xd, g, r, c, amax, MODE, RULE, codes, scales, tscale, choice, s)
        if ev is not None:
            ev[2].record(stream)
        nv.nvfp4_dequantize(codes, scales, tscale, g, r, c, y, s)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)

    # ---- timed region: exactly K steps ----
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    elapsed_ms = start.elapsed_time(stop)
    t_amax = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_quant = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    t_deq = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    step_ms = max_over_ranks(elapsed_ms / args.steps, world)
    value = world * 2 * n / (step_ms * 1e-3) / GB
    launches = 3 * args.steps

    # ---- Four Over Six overhead vs scale-6 on the same GPU (quantize kernel, amax given) ----
    variants = [("scale6", 0, 2), ("46_maxerr", 1, 0), ("46_mae", 1, 1), ("46_mse", 1, 2)]
    times = {v[0]: [] for v in variants}
    for rep in range(12):
        for name, mode, rule in (variants if rep % 2 == 0 else variants[::-1]):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            nv.nvfp4_quantize(xd, g, r, c, amax, mode, rule, codes, scales, tscale, choice, s)
            b.record(stream)
            b.synchronize()
            if rep >= 2:
                times[name].append(a.elapsed_time(b))
    med = {k: statistics.median(v) for k, v in times.items()}
    overhead = {k: round(med[k] / med["scale6"] - 1.0, 4) for k in med if k != "scale6"}

    # ---- end to end through the public API with host buffers ----
    x_pin = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    out_pin = {k: torch.empty(v.numel(), dtype=v.dtype).pin_memory()
               for k, v in (("codes", codes), ("scales", scales), ("tscale", tscale), ("choice", choice))}
    h2d = x_pin.numel() * 2
    d2h = sum(v.numel() * v.element_size() for v in out_pin.values())

    def e2e_step():
        xd.copy_(x_pin, non_blocking=True)
        nv.nvfp4_amax(xd, g, r, c, amax, s)
        nv.nvfp4_quantize(xd, g, r, c, amax, MODE, RULE, codes, scales, tscale, choice, s)
        nv.nvfp4_dequantize(codes, scales, tscale, g, r, c, y, s)
        for k, buf in (("codes", codes), ("scales", scales), ("tscale", tscale), ("choice", choice)):
            out_pin[k].copy_(buf, non_blocking=True)

    e2e_k = max(1, args.e2e_steps)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record(stream)
    for _ in range(e2e_k):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t0
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_k, world)
    e2e_value = world * 2 * n / (e2e_ms * 1e-3) / GB
    torch.cuda.synchronize(dev)

    # ---- CPU oracle on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x_np, c, rows=min(12288, r))

    if rank == 0:
        peak, peak_kind = measured_peak()
        ab = algorithmic_bytes(n, g)
        ach = {k: ab[k] / (t * 1e-3) / GB for k, t in (("amax", t_amax), ("quantize", t_quant), ("dequantize", t_deq))}
        traffic = ncu_traffic("quantize")
        line = {
            "metric": "NVFP4 quantize input GB/s & % of B200 HBM peak; 4/6 overhead vs scale-6",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {
                "workload": f"c5: BF16 {r}x{c} ({2 * n / 2**30:.3g} GiB) N(0,1), 1% zero blocks, 1% blocks x1e-6; "
                            "Four Over Six, MSE rule; one tensor per rank",
                "shape": [g, r, c], "step": "amax + quantize (codes, scales, tscale, choice) + dequantize",
                "l2": "no flush: every step streams 1 GiB of input, 8x the 126 MB L2",
                "parallelism": f"dp{world} (independent tensors, no collective on the data path)",
            },
            "roofline": {
                "kernel": "quantize_kernel<four_over_six, mse, codes>", "bound": "hbm",
                "achieved": round(ach["quantize"], 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach["quantize"] / peak, 4), "peak_kind": peak_kind,
                "bytes_per_launch": ab["quantize"], "traffic": traffic,
            },
            "kernels": {
                k: {"ms": round(t, 4), "GBps": round(ach[k], 1), "frac_of_peak": round(ach[k] / peak, 4),
                    "bytes_per_launch": ab[k]}
                for k, t in (("amax", t_amax), ("quantize", t_quant), ("dequantize", t_deq))
            },
            "quantize_input_GBps": round(2 * n / (t_quant * 1e-3) / GB, 1),
            "overhead_46_vs_scale6": {"ms": {k: round(v, 4) for k, v in med.items()}, "overhead": overhead},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_k, "wall_s": round(wall, 3),
                    "path": "pinned host x -> H2D -> nvfp4_amax -> nvfp4_quantize -> nvfp4_dequantize -> "
                            "D2H of codes, scales, tscale, choice"},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")}
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
