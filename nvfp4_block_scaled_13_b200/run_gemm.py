"""Time the block-scaled FP4 GEMM on the tensor cores.

    python -m nvfp4_block_scaled_13_b200.run_gemm --m 8192 --n 4096 --k 4096 --reps 20

Synthetic operands drawn on the GPU from a seeded generator: activations x [m, k] BF16 with
Student-t(3)-like tails times a lognormal per-channel scale, weights w [n, k] BF16 N(0, 0.02).
The weights are quantized once (Four Over Six, MSE). Reported, as mean CUDA-event times over
`reps` launches after warm-up, with TFLOP/s = 2 m n k / t:
  gemm         nvfp4_gemm on pre-quantized activations,
  gemm_bf16    nvfp4_gemm_bf16 (BF16 result and its amax from the epilogue),
  quantize_x   nvfp4_quantize_gemm of the activations (amax given),
  prologue     nvfp4_gemm_quantize_x (activations quantized inside the GEMM).
"""
from __future__ import annotations

import argparse
import json


def main():
    import torch

    import nvfp4_block_scaled_13_b200 as nv

    ap = argparse.ArgumentParser()
    ap.add_argument("--m", type=int, default=8192)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--mode", default="four_over_six")
    ap.add_argument("--rule", default="mse")
    a = ap.parse_args()

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


if __name__ == "__main__":
    main()
