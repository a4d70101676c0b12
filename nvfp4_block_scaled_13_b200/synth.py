"""Seeded synthetic BF16 inputs shaped like the pages' LLM weights and activations.

This module holds no quantization arithmetic: it only draws numbers (numpy PCG64 in
binary32) and rounds them to BF16 with torch's CPU cast, so that the CUDA path and the
oracle receive the same bits. The trained weights, activations and datasets the pages
measure on are not available; these recipes stand in for them:

  c1  256 x 1024, i.i.d. N(0, 1)                                   (seed 0)
  c2  4096 x 4096 weight, N(0, 0.02); 0.1% of entries, chosen uniformly without
      replacement, multiplied by 20 (outliers)                    (seed 1)
  c3  8192 tokens x 4096 hidden activations: Student-t(nu=3) times a per-channel
      (last dimension) scale drawn lognormal(0, 1)               (seed 2)
  c4  64 experts x 4096 x 1024 weight stack, each N(0, 0.02), one tensor scale per
      expert (groups = 64)                                        (seed 3)
  c5  65536 x 8192 (1 GiB), N(0, 1); 1% of the 16-element blocks (uniform, without
      replacement) set to zero and a disjoint 1% multiplied by 1e-6 (tiny block scales)
                                                                  (seed 4)

Every generator accepts smaller shapes so the same distributions can be checked against
the oracle at sizes it finishes in seconds.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BLOCK = 16


@dataclass(frozen=True)
class Config:
    name: str
    groups: int
    rows: int
    cols: int
    seed: int
    mode: str          # "scale6" or "four_over_six"
    rule: str          # "maxerr", "mae" or "mse"
    output: str        # "codes" or "fakequant"
    description: str

    @property
    def numel(self) -> int:
        return self.groups * self.rows * self.cols


CONFIGS = {
    "c1": Config("c1", 1, 256, 1024, 0, "four_over_six", "mse", "codes",
                 "BF16 256x1024 i.i.d. N(0,1); scale-6 and 4/6-MSE; codes, scales, tensor scale, choice bits"),
    "c2": Config("c2", 1, 4096, 4096, 1, "four_over_six", "mse", "codes",
                 "BF16 weight 4096x4096 N(0,0.02), 0.1% entries x20; 4/6-MSE; codes + row-major scales"),
    "c3": Config("c3", 1, 8192, 4096, 2, "four_over_six", "mae", "fakequant",
                 "BF16 activations 8192x4096 Student-t(3) x lognormal(0,1) per channel; 4/6-MAE fake-quant"),
    "c4": Config("c4", 64, 4096, 1024, 3, "four_over_six", "mse", "codes",
                 "MoE stack 64x4096x1024 N(0,0.02), one tensor scale per expert; 4/6-MSE"),
    "c5": Config("c5", 1, 65536, 8192, 4, "four_over_six", "mse", "codes",
                 "BF16 65536x8192 (1 GiB) N(0,1), 1% zero blocks, 1% blocks x1e-6; scale-6 and 4/6 max/MAE/MSE"),
}


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """binary32 array -> BF16 bit patterns (uint16), rounded by torch's CPU cast."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _normal(rng, n, std):
    x = rng.standard_normal(n, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def gen_c1(rows=256, cols=1024, seed=0, groups=1):
    rng = np.random.default_rng(seed)
    return _normal(rng, groups * rows * cols, 1.0)


def gen_c2(rows=4096, cols=4096, seed=1, groups=1):
    rng = np.random.default_rng(seed)
    n = groups * rows * cols
    x = _normal(rng, n, 0.02)
    k = max(1, int(n * 0.001))
    pos = rng.choice(n, size=k, replace=False)
    x[pos] *= np.float32(20.0)
    return x


def gen_c3(rows=8192, cols=4096, seed=2, groups=1):
    rng = np.random.default_rng(seed)
    t = rng.standard_t(3.0, size=(groups * rows, cols)).astype(np.float32)
    chan = rng.lognormal(0.0, 1.0, size=cols).astype(np.float32)
    return (t * chan[None, :]).ravel()


def gen_c4(rows=4096, cols=1024, seed=3, groups=64):
    rng = np.random.default_rng(seed)
    return _normal(rng, groups * rows * cols, 0.02)


def gen_c5(rows=65536, cols=8192, seed=4, groups=1):
    rng = np.random.default_rng(seed)
    n = groups * rows * cols
    x = _normal(rng, n, 1.0)
    nblocks = n // BLOCK
    k = max(1, nblocks // 100)
    picked = rng.choice(nblocks, size=min(2 * k, nblocks), replace=False)
    xb = x.reshape(nblocks, BLOCK)
    xb[picked[:k]] = 0.0
    xb[picked[k:]] *= np.float32(1e-6)
    return x


_GEN = {"c1": gen_c1, "c2": gen_c2, "c3": gen_c3, "c4": gen_c4, "c5": gen_c5}


def make(name: str, rows: int | None = None, cols: int | None = None, groups: int | None = None,
         seed: int | None = None):
    """BF16 bits (uint16, flat, row-major [groups, rows, cols]) and (groups, rows, cols)."""
    cfg = CONFIGS[name]
    rows = cfg.rows if rows is None else rows
    cols = cfg.cols if cols is None else cols
    groups = cfg.groups if groups is None else groups
    seed = cfg.seed if seed is None else seed
    assert cols % BLOCK == 0 and rows >= 0 and groups >= 1
    x = _GEN[name](rows=rows, cols=cols, seed=seed, groups=groups)
    return to_bf16_bits(x), (groups, rows, cols)


def random_case(seed: int):
    """A random small shape (groups 1-5, rows 1-33, cols 16-1024 in steps of 16) drawn from a
    random mix of the distributions above plus a few scaled copies."""
    rng = np.random.default_rng(10_000 + seed)
    groups = int(rng.integers(1, 6))
    rows = int(rng.integers(1, 34))
    cols = int(16 * rng.integers(1, 65))
    name = ["c1", "c2", "c3", "c4", "c5"][int(rng.integers(0, 5))]
    x = _GEN[name](rows=rows, cols=cols, seed=int(rng.integers(0, 2**31)), groups=groups)
    # per-group magnitude spread so groups get different tensor scales
    spread = np.exp2(rng.integers(-20, 21, size=groups)).astype(np.float32)
    x = (x.reshape(groups, -1) * spread[:, None]).ravel()
    return to_bf16_bits(x), (groups, rows, cols)


def qad_logits(rows: int, vocab: int, seed: int = 5, noise: float = 0.3, scale: float = 3.0, peaked: float = 0.25):
    """Teacher and student logits for the QAD loss, as BF16 bits [rows, vocab].

    Stand-in for a frozen teacher and an NVFP4 student on the same tokens (no model or data
    is available): teacher logits N(0, scale^2) with a fraction `peaked` of rows made
    confident (one logit raised by 4 * scale); the student is the teacher plus N(0, noise^2),
    the small disagreement that quantization noise leaves."""
    rng = np.random.default_rng(seed)
    t = rng.standard_normal((rows, vocab), dtype=np.float32) * np.float32(scale)
    npk = int(rows * peaked)
    if npk and vocab > 1:
        idx = rng.integers(0, vocab, npk)
        t[np.arange(npk), idx] += np.float32(4 * scale)
    s = t + rng.standard_normal((rows, vocab), dtype=np.float32) * np.float32(noise)
    return to_bf16_bits(t).reshape(rows, vocab), to_bf16_bits(s).reshape(rows, vocab)
