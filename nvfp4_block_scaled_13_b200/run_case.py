"""Run the hot path once on one workload, for profilers.

    python -m nvfp4_block_scaled_13_b200.run_case --workload c5 --rows 16384 \
        --mode four_over_six --rule mse --reps 3 [--fakequant]

Generates the workload's synthetic input with the given number of rows (same distribution
as the full-size workload), then launches nvfp4_amax, nvfp4_quantize (or nvfp4_fakequant)
and nvfp4_dequantize `reps` times on the current CUDA device. Prints the kernel times it
measured with CUDA events. Used to capture small, self-terminating ncu profiles.
"""
from __future__ import annotations

import argparse

import numpy as np


def main():
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
    a = ap.parse_args()

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


if __name__ == "__main__":
    main()
