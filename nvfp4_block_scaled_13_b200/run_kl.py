"""Time the QAD distillation loss kernel (nvfp4_qad_kl) on synthetic logits.

    python -m nvfp4_block_scaled_13_b200.run_kl --rows 4096 --vocab 131072 --reps 20 [--no-grad]

Teacher logits N(0, 9) and a student equal to the teacher plus N(0, 0.09), drawn on the GPU
from a seeded generator (BF16). Prints the mean CUDA-event time of the kernel over `reps`
launches after warm-up, and the bandwidth against the algorithmic bytes (each logit read
once; BF16 gradient written once) and against the bytes the two-pass kernel moves.
"""
from __future__ import annotations

import argparse
import json


def main():
    import torch

    import nvfp4_block_scaled_13_b200 as nv

    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=4096)
    ap.add_argument("--vocab", type=int, default=131072)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--tau", type=float, default=1.0)
    ap.add_argument("--no-grad", action="store_true")
    a = ap.parse_args()

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


if __name__ == "__main__":
    main()
