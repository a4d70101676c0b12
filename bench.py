"""Throughput bench of the NVFP4 quantizer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...)

One step is one pass of the whole hot path over one tensor resident in HBM:
    nvfp4_amax -> nvfp4_quantize (Four Over Six, MSE rule: codes, scales, tensor scale,
    choice bits) -> nvfp4_dequantize,
on the 1 GiB workload: BF16 65536 x 8192, N(0,1), 1% zero blocks, 1% blocks x1e-6.
Each rank quantizes its own tensor (weak scaling, no collective on the data path).
`value` is the metric's quantize-kernel input GB/s with the amax given: ranks * 2 * numel /
(max over ranks of the quantize launch's mean CUDA-event time inside the timed steps);
`step_input_GBps` is the same over the whole step (amax + quantize + dequantize).

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
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-workload leg")
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


def fp4_peak():
    """Dense FP4 tensor-core peak: the measured BF16 GEMM peak (burst) times 4, the ratio of the
    nominal dense FP4 and BF16 peaks (9 and 2.25 PFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            v = json.load(f).get("bf16_tflops")
        if v:
            return round(4.0 * float(v), 1), "measured bf16 x 4"
    return 4.0 * 1590.0, "fallback bf16 x 4"


def ncu_traffic(kernel: str):
    """Per-launch DRAM traffic of `kernel` from the committed ncu summary, or None when the
    kernel's source changed after the capture (the summary stores the source hash)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = b""
    for f in ("kernels.cuh", "block.cuh", "ptx.cuh"):
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

def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_step(x_rows: np.ndarray, rows: int, cols: int, threads: int = 1, amax=None):
    """The oracle's quantize (Four Over Six, MSE) of `rows` rows with the tensor amax given,
    the metric's operation; with amax=None, amax + quantize + dequantize (the whole path). Its
    C functions are called on `threads` row ranges at once (the oracle's calls release the
    interpreter lock and blocks are independent, so the ranges give the same bytes as one call
    over all rows)."""
    import oracle as O

    O.lib()
    whole = amax is None
    if threads <= 1:
        a = O.amax(x_rows, 1, rows, cols) if whole else amax
        q = O.quantize(x_rows, 1, rows, cols, a, MODE, RULE)
        if whole:
            O.dequantize(q["codes"], q["scales"], q["tscale"], 1, rows, cols)
        return
    from concurrent.futures import ThreadPoolExecutor

    bounds = [(rows * i // threads, rows * (i + 1) // threads) for i in range(threads)]
    bounds = [(lo, hi) for lo, hi in bounds if hi > lo]
    part = lambda lo, hi: x_rows[lo * cols:hi * cols]
    with ThreadPoolExecutor(len(bounds)) as ex:
        a = np.max(list(ex.map(lambda b: O.amax(part(*b), 1, b[1] - b[0], cols), bounds)), axis=0) if whole else amax

        def rest(b):
            q = O.quantize(part(*b), 1, b[1] - b[0], cols, a, MODE, RULE)
            if whole:
                O.dequantize(q["codes"], q["scales"], q["tscale"], 1, b[1] - b[0], cols)

        list(ex.map(rest, bounds))


def tensor_amax(x: np.ndarray) -> np.ndarray:
    """max |x| of a BF16 tensor (uint16 bits) as binary32: BF16 magnitudes order like their bits."""
    m = int(np.max(x & np.uint16(0x7FFF))) if x.size else 0
    return np.array([m << 16], np.uint32).view(np.float32)


def cpu_baseline(x: np.ndarray, cols: int, amax: np.ndarray, rows: int = 12288):
    """The oracle as it stands (C) on the first `rows` rows of the workload, quantizing with
    the whole tensor's amax given (the metric's operation): on all host cores (the reported
    value), and on one thread."""
    xs = np.ascontiguousarray(x[: rows * cols])
    threads = host_threads()
    t0 = time.perf_counter()
    oracle_step(xs, rows, cols, threads, amax=amax)
    dt_all = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle_step(xs, rows, cols, 1, amax=amax)
    dt_one = time.perf_counter() - t0
    return {"value": round(2 * rows * cols / dt_all / GB, 5), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of the 65536x8192 tensor ({rows * cols / 1e6:.1f} M elements): "
                      f"4/6-MSE quantize with the tensor amax given, on {threads} threads ({dt_all:.2f} s); "
                      f"one thread: {dt_one:.1f} s",
            "single_thread": {"value": round(2 * rows * cols / dt_one / GB, 5), "unit": "GB/s"}}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on the machine's host cores (rank 0 only)."""
    if rank != 0:
        return
    x, (g, r, c) = make_input(0, args.rows)
    threads = host_threads()
    amax = tensor_amax(x)          # the metric quantizes with the amax given
    # calibrate, then size each step's sample so that the whole run takes about two minutes
    cal_rows = 16 * threads
    t0 = time.perf_counter()
    oracle_step(np.ascontiguousarray(x[: cal_rows * c]), cal_rows, c, threads, amax=amax)
    per_row = (time.perf_counter() - t0) / cal_rows
    rows = int(max(threads, min(8192, r // 2, 120.0 / max(1, args.steps + args.warmup) / per_row)))
    for i in range(args.warmup):
        s = (i * rows) % (r - rows)
        oracle_step(np.ascontiguousarray(x[s * c:(s + rows) * c]), rows, c, threads, amax=amax)
    t0 = time.perf_counter()
    for i in range(args.steps):
        s = ((args.warmup + i) * rows) % (r - rows)
        oracle_step(np.ascontiguousarray(x[s * c:(s + rows) * c]), rows, c, threads, amax=amax)
    dt = time.perf_counter() - t0
    value = 2 * rows * c * args.steps / dt / GB
    sample = (f"{rows} rows x 8192 per step ({rows * c / 1e6:.2f} M elements): 4/6-MSE quantize with the tensor "
              f"amax given, on {threads} threads")
    print(json.dumps({
        "impl": "reference", "metric": "NVFP4 quantize input GB/s & % of B200 HBM peak; 4/6 overhead vs scale-6",
        "value": round(value, 6), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"c5: BF16 {r}x{c} N(0,1), 1% zero blocks, 1% blocks x1e-6; "
                               "Four Over Six, MSE rule", "shape": [1, r, c],
                   "step": "quantize (codes, scales, tscale, choice) of a row sample with the tensor amax given"},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---- GPU legs ------------------------------------------------------------------------------

def gemm_leg(nv, torch, dev, peak_tflops, m=8192, n=4096, k=4096, reps=20):
    """The block-scaled FP4 GEMM on a transformer-layer shape (m tokens x k -> n): activations
    quantized once (Four Over Six, MSE) then nvfp4_gemm, the BF16-output variant whose epilogue
    also finds the result's amax (nvfp4_gemm_bf16), and the variant that quantizes the
    activations in its prologue. TFLOP/s = 2 m n k / t against the FP4 dense peak."""
    gen = torch.Generator(device=dev).manual_seed(7)
    x = (torch.randn(m, k, device=dev, generator=gen) * torch.exp(torch.randn(k, device=dev, generator=gen))
         ).to(torch.bfloat16)
    w = (torch.randn(n, k, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
    wq = nv.quantize_for_gemm(w)
    ax = nv.amax(x, 1)
    xq = nv.quantize_for_gemm(x, amax_values=ax)
    y = torch.empty(m, n, dtype=torch.float32, device=dev)
    y16 = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    y_amax = torch.empty(1, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev).cuda_stream
    legs = {
        "quantize_x": lambda: nv.nvfp4_quantize_gemm(x, m, k, ax, 1, 2, xq[0], xq[1], xq[2], None, s),
        "gemm": lambda: nv.nvfp4_gemm(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], m, n, k, y, status, s),
        "gemm_bf16_amax": lambda: nv.nvfp4_gemm_bf16(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], m, n, k, y16, y_amax,
                                                     status, s),
        "prologue": lambda: nv.nvfp4_gemm_quantize_x(x, ax, 1, 2, wq[0], wq[1], wq[2], m, n, k, y, status, s),
    }
    ms = {}
    for name, fn in legs.items():
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        b.synchronize()
        ms[name] = a.elapsed_time(b) / reps
    flops = 2.0 * m * n * k
    tf = flops / (ms["gemm"] * 1e-3) / 1e12
    out = {"shape": [m, n, k], "kernel": "gemm_fp4_kernel (tcgen05.mma.kind::mxf4nvf4.block_scale.block16)",
           "ms": {k2: round(v, 4) for k2, v in ms.items()}, "tflops": round(tf, 1),
           "peak_tflops": peak_tflops, "frac": round(tf / peak_tflops, 4),
           "quantize_then_gemm_tflops": round(flops / ((ms["gemm"] + ms["quantize_x"]) * 1e-3) / 1e12, 1),
           "prologue_tflops": round(flops / (ms["prologue"] * 1e-3) / 1e12, 1),
           "bf16_amax_tflops": round(flops / (ms["gemm_bf16_amax"] * 1e-3) / 1e12, 1),
           "status": int(status.item())}
    del x, w, wq, xq, y, y16
    return out


L2_BYTES = 126 * 2**20
OVERHEAD_BATCH = 8


def batch_ms(torch, stream, fn, count):
    """Mean time of `count` launches of fn enqueued back to back between two events."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(count):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / count


def per_config_leg(nv, torch, dev, stream, peak, resident=None):
    """The quantize kernel on each workload with its amax given (the fixed-scale path): time,
    input GB/s (2N / t), algorithmic bytes / t against the HBM peak, amax + quantize, and the
    Four Over Six overhead against scale-6 timed in interleaved repetitions on the same tensor.
    Inputs that fit in L2 are timed cold (a 512 MiB write flushes L2 before each launch) and
    warm (back to back); the 512 KiB workload is timed by CUDA-graph replay of 50 launches.
    Cold has two figures. "cold" comes from CUDA graphs of 10 (flush, launch) pairs against
    graphs of the 10 flushes alone: the difference over 10 is the launch's device time after a
    flush, free of the host's launch latency. "cold_single" brackets one launch after a flush
    with two events, and so also holds the gap between the flush's end and the kernel's start
    (about 6 us for a one-element kernel, measured the same way)."""
    from nvfp4_block_scaled_13_b200 import synth

    s = stream.cuda_stream
    flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
    modes = {"scale6": 0, "four_over_six": 1}
    rules = {"maxerr": 0, "mae": 1, "mse": 2}
    out = {}
    for name, cfg in synth.CONFIGS.items():
        x, (g, r, c) = resident[name] if resident and name in resident else synth.make(name)
        n, nb = g * r * c, g * r * c // 16
        xd = torch.from_numpy(x.view(np.int16)).to(dev)
        del x
        amax = torch.empty(g, dtype=torch.float32, device=dev)
        tscale = torch.empty(g, dtype=torch.float32, device=dev)
        choice = torch.empty((nb + 7) // 8, dtype=torch.uint8, device=dev)
        fq = cfg.output == "fakequant"
        if fq:
            y = torch.empty(n, dtype=torch.int16, device=dev)
            nbytes = 4 * n + (nb + 7) // 8 + 4 * g
        else:
            codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
            scales = torch.empty(nb, dtype=torch.uint8, device=dev)
            nbytes = algorithmic_bytes(n, g)["quantize"]

        def launch(mode, rule):   # on the current stream (a graph's capture stream while capturing)
            cs = torch.cuda.current_stream(dev).cuda_stream
            if fq:
                nv.nvfp4_fakequant(xd, g, r, c, amax, mode, rule, y, choice, cs)
            else:
                nv.nvfp4_quantize(xd, g, r, c, amax, mode, rule, codes, scales, tscale, choice, cs)

        nv.nvfp4_amax(xd, g, r, c, amax, s)
        variants = [("scale6", 0, 2)]
        if cfg.mode == "four_over_six":
            names = ["maxerr", "mae", "mse"] if name == WORKLOAD else [cfg.rule]
            variants += [(f"46_{k}", 1, rules[k]) for k in names]
        for v in variants:
            launch(v[1], v[2])
        torch.cuda.synchronize(dev)
        small = 2 * n <= 4 * 2**20
        fits_l2 = 2 * n <= L2_BYTES
        res = {"shape": [g, r, c], "output": cfg.output, "bytes_per_launch": nbytes}

        def timed(fn, cold):
            if not cold:   # a batch back to back (see the overhead leg)
                return batch_ms(torch, stream, fn, OVERHEAD_BATCH)
            flush.zero_()   # still running when the launch is enqueued, so no idle gap is timed
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            return a.elapsed_time(b)

        def graph_cold_ms(fn, pairs=10, rounds=8):
            ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(ga):
                for _ in range(pairs):
                    flush.zero_()
                    fn()
            with torch.cuda.graph(gb):
                for _ in range(pairs):
                    flush.zero_()
            ga.replay()
            gb.replay()
            torch.cuda.synchronize(dev)
            ta, tb = [], []
            for i in range(rounds):
                for gr, tl in ((ga, ta), (gb, tb)) if i % 2 == 0 else ((gb, tb), (ga, ta)):
                    tl.append(batch_ms(torch, stream, gr.replay, 1))
            del ga, gb
            return (statistics.median(ta) - statistics.median(tb)) / pairs

        if small:
            per = {}
            for vname, mode, rule in variants:
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    for _ in range(50):
                        launch(mode, rule)
                graph.replay()
                torch.cuda.synchronize(dev)
                reps = []
                for _ in range(10):
                    reps.append(timed(graph.replay, False) / 50)
                per[vname] = statistics.median(reps)
                del graph
            res["timing"] = "warm, CUDA-graph replay of 50 launches"
        else:
            kinds = [("cold_single", True), ("warm", False)] if fits_l2 else [("", False)]
            per = {}
            if fits_l2:
                for rep_i in range(2):
                    for vname, mode, rule in (variants if rep_i % 2 == 0 else variants[::-1]):
                        per.setdefault(vname + "_cold", []).append(
                            graph_cold_ms(lambda mode=mode, rule=rule: launch(mode, rule)))
                for k in list(per):
                    per[k] = statistics.median(per[k])
            for kind, cold in kinds:
                t = {v[0]: [] for v in variants}
                for rep_i in range(14):
                    for vname, mode, rule in (variants if rep_i % 2 == 0 else variants[::-1]):
                        dt = timed(lambda: launch(mode, rule), cold)
                        if rep_i >= 2:
                            t[vname].append(dt)
                for vname in t:
                    per[vname + (f"_{kind}" if kind else "")] = statistics.median(t[vname])
            res["timing"] = ("L2 flushed before each launch: cold = graphs of (flush, launch) pairs minus graphs "
                             "of the flushes, per launch; cold_single = one launch between two events after a "
                             "flush; warm = back to back" if fits_l2
                             else "back to back; the input is larger than L2")
        main_v = variants[-1][0]
        suffix = "_cold" if (fits_l2 and not small) else ""
        tq = per[main_v + suffix]
        res["ms"] = {k: round(v, 5) for k, v in per.items()}
        res["kernel"] = f"{'fakequant' if fq else 'quantize'} {main_v}"
        res["input_GBps"] = round(2 * n / (tq * 1e-3) / GB, 1)
        res["GBps"] = round(nbytes / (tq * 1e-3) / GB, 1)
        res["frac_of_peak"] = round(nbytes / (tq * 1e-3) / GB / peak, 4)
        if len(variants) > 1:
            res["overhead_46_vs_scale6"] = {
                k[3:]: round(per[k + suffix] / per["scale6" + suffix] - 1.0, 4) for k, _, _ in variants[1:]}
        def both():
            nv.nvfp4_amax(xd, g, r, c, amax, torch.cuda.current_stream(dev).cuda_stream)
            launch(variants[-1][1], variants[-1][2])

        t_aq = []
        if small:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(50):
                    both()
            graph.replay()
            torch.cuda.synchronize(dev)
            t_aq = [timed(graph.replay, False) / 50 for _ in range(10)]
            del graph
        else:
            for rep_i in range(8):
                dt = timed(both, fits_l2)
                if rep_i >= 2:
                    t_aq.append(dt)
        res["amax_plus_quantize_ms"] = round(statistics.median(t_aq), 5)

        # the same two steps in one launch (grid-wide barrier), flushed or in batches as above
        work = torch.zeros(2, dtype=torch.int32, device=dev)

        def one_launch():
            cs = torch.cuda.current_stream(dev).cuda_stream
            m, rl = variants[-1][1], variants[-1][2]
            if fq:
                nv.nvfp4_amax_fakequant(xd, g, r, c, m, rl, amax, y, choice, work[0:1], work[1:2], cs)
            else:
                nv.nvfp4_amax_quantize(xd, g, r, c, m, rl, amax, codes, scales, tscale, choice, work[0:1], work[1:2],
                                       cs)

        one_launch()
        t_one = []
        for rep_i in range(8):
            dt = timed(one_launch, fits_l2)
            if rep_i >= 2:
                t_one.append(dt)
        res["amax_quantize_one_launch_ms"] = round(statistics.median(t_one), 5)
        res["one_launch_status"] = int(work[1].item())
        out[name] = res
        del xd
        if fq:
            del y
        else:
            del codes, scales
    del flush
    torch.cuda.empty_cache()
    return out

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
    # the metric: quantize-kernel input GB/s with the amax given, 2N / t_q over all ranks, t_q the
    # mean CUDA-event time of the quantize launch inside the K timed steps (max over ranks)
    tq_ms = max_over_ranks(t_quant, world)
    value = world * 2 * n / (tq_ms * 1e-3) / GB
    step_value = world * 2 * n / (step_ms * 1e-3) / GB
    launches = 3 * args.steps

    # ---- Four Over Six overhead vs scale-6 on the same GPU (quantize kernel, amax given) ----
    # Each sample is a batch of launches of one variant back to back between two events, so the
    # host's submission of a launch never leaves the GPU idle inside the timed interval (with a
    # synchronize after every single launch, that idle time would be counted as kernel time);
    # the variants alternate batch by batch.
    variants = [("scale6", 0, 2), ("46_maxerr", 1, 0), ("46_mae", 1, 1), ("46_mse", 1, 2)]
    times = {v[0]: [] for v in variants}
    with ClockSampler(local) as clocks_overhead:   # the issue-bound 4/6 kernels follow the SM clock
        for rep in range(10):
            for name, mode, rule in (variants if rep % 2 == 0 else variants[::-1]):
                dt = batch_ms(torch, stream, lambda: nv.nvfp4_quantize(xd, g, r, c, amax, mode, rule, codes, scales,
                                                                       tscale, choice, s), OVERHEAD_BATCH)
                if rep >= 2:
                    times[name].append(dt)
    med = {k: statistics.median(v) for k, v in times.items()}
    overhead = {k: round(med[k] / med["scale6"] - 1.0, 4) for k in med if k != "scale6"}

    # ---- end to end through the public API with host buffers ----
    # Each step copies its input from pinned host memory, runs amax -> quantize -> dequantize and
    # copies its quantized result back. Steps alternate between two device buffer sets on three
    # streams, so that step i + 1's host-to-device copy overlaps step i's compute and its
    # device-to-host copy (the two directions use separate copy engines).
    x_pin = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    sets = [dict(x=xd, amax=amax, codes=codes, scales=scales, tscale=tscale, choice=choice, y=y)]
    sets.append({k: torch.empty_like(v) for k, v in sets[0].items()})
    keys = ("codes", "scales", "tscale", "choice")
    out_pin = [{k: torch.empty(st[k].numel(), dtype=st[k].dtype).pin_memory() for k in keys} for st in sets]
    h2d = x_pin.numel() * 2
    d2h = sum(v.numel() * v.element_size() for v in out_pin[0].values())
    s_h, s_c, s_d = (torch.cuda.Stream(dev) for _ in range(3))
    ev_h, ev_c, ev_d = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_step(i):
        b = i % 2
        st = sets[b]
        s_h.wait_event(ev_c[b])                  # step i - 2's compute has read this buffer
        with torch.cuda.stream(s_h):
            st["x"].copy_(x_pin, non_blocking=True)
        ev_h[b].record(s_h)
        s_c.wait_event(ev_h[b])
        s_c.wait_event(ev_d[b])                  # step i - 2's results have been copied out
        cs = s_c.cuda_stream
        nv.nvfp4_amax(st["x"], g, r, c, st["amax"], cs)
        nv.nvfp4_quantize(st["x"], g, r, c, st["amax"], MODE, RULE, st["codes"], st["scales"], st["tscale"],
                          st["choice"], cs)
        nv.nvfp4_dequantize(st["codes"], st["scales"], st["tscale"], g, r, c, st["y"], cs)
        ev_c[b].record(s_c)
        s_d.wait_event(ev_c[b])
        with torch.cuda.stream(s_d):
            for k in keys:
                out_pin[b][k].copy_(st[k], non_blocking=True)
        ev_d[b].record(s_d)

    e2e_k = max(1, args.e2e_steps)
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record(s_h)
    for i in range(e2e_k):
        e2e_step(i)
    b.record(s_d)                                # the last device-to-host copy is the last work
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t0
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_k, world)
    e2e_value = world * 2 * n / (e2e_ms * 1e-3) / GB
    del sets[1]
    torch.cuda.synchronize(dev)

    # ---- every workload's quantize kernel (N = 1 only) ----
    per_cfg = None
    if world == 1 and not args.no_per_config:
        with ClockSampler(local) as clocks_per_config:
            per_cfg = per_config_leg(nv, torch, dev, stream, measured_peak()[0],
                                     resident={WORKLOAD: (x_np, (g, r, c))} if args.rows is None else None)
        per_cfg["clocks"] = clocks_per_config.summary()

    # ---- the FP4 tensor-core GEMM (N = 1 only) ----
    gemm = None
    if world == 1 and not args.no_per_config:
        gemm = gemm_leg(nv, torch, dev, fp4_peak()[0])

    # ---- CPU oracle on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x_np, c, tensor_amax(x_np), rows=min(12288, r))

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
            "value_definition": "quantize-kernel input GB/s with the amax given: ranks * 2N / t_q, t_q the mean "
                                "CUDA-event time of the nvfp4_quantize launch inside the K timed steps (max over "
                                "ranks)",
            "quantize_ms": round(tq_ms, 5),
            "step_input_GBps": round(step_value, 2),
            "config": {
                "workload": f"c5: BF16 {r}x{c} ({2 * n / 2**30:.3g} GiB) N(0,1), 1% zero blocks, 1% blocks x1e-6; "
                            "Four Over Six, MSE rule; one tensor per rank",
                "shape": [g, r, c], "step": "amax + quantize (codes, scales, tscale, choice) + dequantize",
                "l2": "no flush: every step streams 1 GiB of input, 8x the 126 MB L2",
                "parallelism": f"dp{world} (independent tensors, no collective on the data path)",
            },
            "roofline": {
                "kernel": "quantize_grouped_kernel<four_over_six, mse, codes>", "bound": "hbm",
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
            "overhead_46_vs_scale6": {"ms": {k: round(v, 4) for k, v in med.items()}, "overhead": overhead,
                                      "clocks": clocks_overhead.summary()},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_k, "wall_s": round(wall, 3),
                    "path": "pinned host x -> H2D -> nvfp4_amax -> nvfp4_quantize -> nvfp4_dequantize -> "
                            "D2H of codes, scales, tscale, choice; two buffer sets on three streams, so step "
                            "i+1's H2D overlaps step i's compute and D2H"},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
        }
        if per_cfg is not None:
            line["per_config"] = per_cfg
        if gemm is not None:
            gemm["peak_kind"] = fp4_peak()[1]
            line["gemm_fp4"] = gemm
        if cpu is not None:
            line["cpu_baseline"] = {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample", "single_thread")}
        print(json.dumps(line), flush=True)


# ---- profiling tools: one small, self-terminating run of one kernel family -------------------
# python bench.py --tool case --workload c5 --rows 16384 --mode four_over_six --rule mse --reps 3
#     amax, quantize (or fakequant / tiled-scale quantize) and dequantize on one workload slice
# python bench.py --tool gemm --m 8192 --n 4096 --k 4096 --reps 20
#     the block-scaled FP4 GEMM (pre-quantized, BF16 result, activation quantize, prologue)
# python bench.py --tool kl --rows 4096 --vocab 131072 --reps 20 [--no-grad]
#     the QAD distillation loss kernel
# They print CUDA-event times; ncu captures in profiles/ name these commands.

def tool_case(argv):
    import torch

    import nvfp4_block_scaled_13_b200 as nv
    from nvfp4_block_scaled_13_b200 import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="c5", choices=sorted(synth.CONFIGS))
    ap.add_argument("--rows", type=int, default=None)
    ap.add_argument("--groups", type=int, default=None)
    ap.add_argument("--mode", default="four_over_six")
    ap.add_argument("--rule", default="mse")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--fakequant", action="store_true")
    ap.add_argument("--gemm-layout", action="store_true", help="nvfp4_quantize_gemm (tiled scales; one group)")
    a = ap.parse_args(argv)

    nv.load()
    x, (g, r, c) = synth.make(a.workload, rows=a.rows, groups=a.groups)
    n, nb = g * r * c, g * r * c // 16
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    amax = torch.empty(g, dtype=torch.float32, device="cuda")
    codes = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(nv.gemm_scale_bytes(g * r, c) if a.gemm_layout else nb, dtype=torch.uint8, device="cuda")
    tscale = torch.empty(g, dtype=torch.float32, device="cuda")
    choice = torch.empty((nb + 7) // 8, dtype=torch.uint8, device="cuda")
    y = torch.empty(n, dtype=torch.int16, device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(a.reps):
        ev[0].record()
        nv.nvfp4_amax(xd, g, r, c, amax)
        ev[1].record()
        if a.fakequant:
            nv.nvfp4_fakequant(xd, g, r, c, amax, a.mode, a.rule, y, choice)
        elif a.gemm_layout:
            nv.nvfp4_quantize_gemm(xd, g * r, c, amax, a.mode, a.rule, codes, scales, tscale, choice)
        else:
            nv.nvfp4_quantize(xd, g, r, c, amax, a.mode, a.rule, codes, scales, tscale, choice)
        ev[2].record()
        if not a.gemm_layout:
            nv.nvfp4_dequantize(codes, scales, tscale, g, r, c, y)
        ev[3].record()
    torch.cuda.synchronize()
    print(f"{a.workload} [{g},{r},{c}] {a.mode}/{a.rule}: amax {ev[0].elapsed_time(ev[1]):.4f} ms, "
          f"{'fakequant' if a.fakequant else ('quantize_gemm' if a.gemm_layout else 'quantize')} "
          f"{ev[1].elapsed_time(ev[2]):.4f} ms, "
          f"dequantize {ev[2].elapsed_time(ev[3]):.4f} ms (last rep)")



def tool_gemm(argv):
    import torch

    import nvfp4_block_scaled_13_b200 as nv

    ap = argparse.ArgumentParser()
    ap.add_argument("--m", type=int, default=8192)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--mode", default="four_over_six")
    ap.add_argument("--rule", default="mse")
    a = ap.parse_args(argv)

    nv.load()
    gen = torch.Generator(device="cuda").manual_seed(7)
    t = torch.randn(a.m, a.k, device="cuda", generator=gen)
    t = t / torch.sqrt(torch.rand(a.m, a.k, device="cuda", generator=gen).clamp_min(1e-3))   # heavy tails
    chan = torch.exp(torch.randn(a.k, device="cuda", generator=gen))
    x = (t * chan).to(torch.bfloat16).contiguous()
    w = (torch.randn(a.n, a.k, device="cuda", generator=gen) * 0.02).to(torch.bfloat16).contiguous()
    del t
    wq = nv.quantize_for_gemm(w, "four_over_six", "mse")
    ax = nv.amax(x, 1)
    xq = nv.quantize_for_gemm(x, a.mode, a.rule, amax_values=ax)
    y = torch.empty(a.m, a.n, dtype=torch.float32, device="cuda")
    y16 = torch.empty(a.m, a.n, dtype=torch.bfloat16, device="cuda")
    y_amax = torch.empty(1, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def run_gemm():
        nv.nvfp4_gemm(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], a.m, a.n, a.k, y, status, s)

    def run_gemm_bf16():
        nv.nvfp4_gemm_bf16(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], a.m, a.n, a.k, y16, y_amax, status, s)

    def run_quant():
        nv.nvfp4_quantize_gemm(x, a.m, a.k, ax, a.mode, a.rule, xq[0], xq[1], xq[2], None, s)

    def run_prologue():
        nv.nvfp4_gemm_quantize_x(x, ax, a.mode, a.rule, wq[0], wq[1], wq[2], a.m, a.n, a.k, y, status, s)

    flops = 2.0 * a.m * a.n * a.k
    out = {"m": a.m, "n": a.n, "k": a.k, "mode": a.mode, "rule": a.rule}
    for name, fn in (("gemm", run_gemm), ("gemm_bf16", run_gemm_bf16), ("quantize_x", run_quant),
                     ("prologue", run_prologue)):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(a.reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / a.reps
        out[name + "_ms"] = round(ms, 4)
        if name != "quantize_x":
            out[name + "_tflops"] = round(flops / ms / 1e9, 1)
    out["status"] = int(status.item())
    print(json.dumps(out))



def tool_kl(argv):
    import torch

    import nvfp4_block_scaled_13_b200 as nv

    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=4096)
    ap.add_argument("--vocab", type=int, default=131072)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--tau", type=float, default=1.0)
    ap.add_argument("--no-grad", action="store_true")
    a = ap.parse_args(argv)

    nv.load()
    gen = torch.Generator(device="cuda").manual_seed(5)
    t = (torch.randn(a.rows, a.vocab, device="cuda", generator=gen) * 3.0).to(torch.bfloat16)
    s = (t.float() + torch.randn(a.rows, a.vocab, device="cuda", generator=gen) * 0.3).to(torch.bfloat16)
    kl = torch.empty(a.rows, dtype=torch.float32, device="cuda")
    g = None if a.no_grad else torch.empty_like(s)
    gs = 1.0 / (a.tau * a.rows)
    for _ in range(3):
        nv.nvfp4_qad_kl(t, s, a.rows, a.vocab, a.tau, gs, kl, g)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        nv.nvfp4_qad_kl(t, s, a.rows, a.vocab, a.tau, gs, kl, g)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.reps
    n = a.rows * a.vocab
    algo = 4 * n + (0 if a.no_grad else 2 * n)
    moved = 4 * n + (0 if a.no_grad else 6 * n)
    print(json.dumps({"rows": a.rows, "vocab": a.vocab, "grad": not a.no_grad, "ms": round(ms, 4),
                      "algorithmic_GBps": round(algo / ms / 1e6, 1), "moved_GBps": round(moved / ms / 1e6, 1),
                      "mean_kl": float(kl.mean())}))



TOOLS = {"case": tool_case, "gemm": tool_gemm, "kl": tool_kl}


def main():
    if len(sys.argv) > 2 and sys.argv[1] == "--tool":
        TOOLS[sys.argv[2]](sys.argv[3:])
        return
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
