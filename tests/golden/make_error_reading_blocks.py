"""Writes tests/golden/error_reading_blocks.txt: single 16-element blocks, with a tensor scale,
on which the two readings of the Four Over Six error term choose different candidates.

The page ("Four Over Six", technical summary > Method > Adaptive block scaling algorithm)
says each candidate's error is measured against the original high-precision values; it does
not fix the rounding. Reading kept: e_i = RN(x_i - v_i d), the exact difference between the
original value and the dequantized value v_i d, rounded once. The other reading rounds the
dequantized value first: e_i = RN(x_i - RN(v_i d)). On most blocks both give the same choice;
this script searches random blocks for those where they do not, so that a pin can tell the
two readings apart.

Only INPUTS are written (block values as BF16 bits, the tensor scale as binary32 bits, the
rule). The search itself uses the oracle for the block scales and codes and numpy binary32
arithmetic for the two error readings; the pin (tests/test_oracle_pins.py) recomputes both
readings in exact rational arithmetic and checks the oracle against the kept one.

    python tests/golden/make_error_reading_blocks.py
"""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "error_reading_blocks.txt")
GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)


def f32(a):
    return np.asarray(a, np.float64).astype(np.float32)


def candidate_errors(x, alpha, K, rule):
    """x (B, 16) binary32 holding BF16 values, alpha (B,) binary32: the candidate's error under
    both readings, (err_once, err_twice), binary32 (B,)."""
    m = np.max(np.abs(x), axis=1)
    beta = f32(np.float64(K) * alpha)
    t = np.where(beta > 0, f32(m.astype(np.float64) / np.where(beta > 0, beta, 1)), np.float32(0))
    s = O.f32_to_e4m3_array(t)
    sv = O.e4m3_to_f32(np.arange(256))[s]
    d = f32(sv.astype(np.float64) * alpha)
    r = np.where(d > 0, np.minimum(f32(1.0 / np.where(d > 0, d, 1).astype(np.float64)), np.finfo(np.float32).max),
                 np.float32(0))
    y = f32(x.astype(np.float64) * r[:, None])
    code = O.f32_to_e2m1_array(y.ravel()).reshape(y.shape)
    v = GRID[code & 7] * np.where(code & 8, -1.0, 1.0)
    vd = v * d[:, None].astype(np.float64)                       # exact in binary64
    e_once = f32(x.astype(np.float64) - vd)                       # the exact difference, rounded once
    e_twice = f32(x.astype(np.float64) - f32(vd).astype(np.float64))
    out = []
    for e in (e_once, e_twice):
        e64 = e.astype(np.float64)
        if rule == 0:
            err = np.max(np.abs(e), axis=1)
        else:
            acc = np.zeros((x.shape[0], 2), np.float32)
            for i in range(16):
                term = np.abs(e64[:, i]) if rule == 1 else e64[:, i] * e64[:, i]
                acc[:, i & 1] = f32(acc[:, i & 1].astype(np.float64) + term)
            err = f32(acc[:, 0].astype(np.float64) + acc[:, 1])
        out.append(err)
    return out


def main(per_rule=12, seed=11):
    rng = np.random.default_rng(seed)
    lines = []
    for rule in (2, 1, 0):
        found = 0
        while found < per_rule:
            B = 200000
            scale = rng.lognormal(0.0, 1.0, (B, 1))
            xb = O.f32_to_bf16_array((rng.standard_normal((B, 16)) * scale).astype(np.float32).ravel())
            x = (xb.astype(np.uint32) << 16).view(np.float32).reshape(B, 16)
            amax = np.max(np.abs(x), axis=1) * f32(rng.uniform(1.0, 3.0, B))
            alpha = f32(amax.astype(np.float64) / 1536.0)
            e6 = candidate_errors(x, alpha, 6, rule)
            e4 = candidate_errors(x, alpha, 4, rule)
            differ = np.flatnonzero((e4[0] < e6[0]) != (e4[1] < e6[1]))
            for b in differ[: per_rule - found]:
                bits = " ".join(f"{int(v):04x}" for v in xb.reshape(B, 16)[b])
                lines.append(f"{rule} {int(alpha[b:b + 1].view(np.uint32)[0]):08x} {bits}")
                found += 1
    with open(OUT, "w") as f:
        f.write("# Blocks on which the two readings of the error term choose differently (inputs only).\n")
        f.write("# Written by tests/golden/make_error_reading_blocks.py; the reading kept is the exact\n")
        f.write("# difference x - v d rounded once (\"Four Over Six\", Method > Adaptive block scaling\n")
        f.write("# algorithm: error against the original values; the rounding is this build's reading).\n")
        f.write("# rule (0 max, 1 MAE, 2 MSE)  alpha (binary32 bits)  16 BF16 values (bits)\n")
        f.write("\n".join(lines) + "\n")
    print(f"wrote {len(lines)} blocks to {OUT}")


if __name__ == "__main__":
    main()
