"""Pins of the oracle's block-scaled FP4 GEMM reference (oracle.gemm_nvfp4).

"Four Over Six" (Implementation details) runs NVFP4 operands on Blackwell's FP4 tensor
cores; a stored value is v(code) * E4M3 block scale * FP32 tensor scale (Problem
definition). The reference must therefore equal alpha_a * alpha_b * sum_k (v s)_a (v s)_b.
These tests check it against exact rational arithmetic built only from the format tables in
tests/exact.py (a one-hot closed form, and brute force on tiny random operands), and show
that a plausible slip (nibble order, a transposed operand, a missing tensor scale, scales
applied per 32 elements) fails them."""
from fractions import Fraction as F

import numpy as np
import pytest

import oracle as O
from tests import exact as X


def pack(codes4: np.ndarray) -> np.ndarray:
    """[rows, k] 4-bit codes -> [rows, k/2] bytes, element 2j in the low nibble."""
    c = codes4.astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def e2m1(c: int) -> F:
    mag = X.E2M1_GRID[c & 7]
    return -mag if c & 8 else mag


def exact_gemm(a4, sa, alpha_a, b4, sb, alpha_b):
    m, k = a4.shape
    n = b4.shape[0]
    aa, ab = X.f32_value(float(np.float32(alpha_a))), X.f32_value(float(np.float32(alpha_b)))
    y = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            acc = F(0)
            for kk in range(k):
                acc += e2m1(int(a4[i, kk])) * X.E4M3[int(sa[i, kk // 16])] * e2m1(int(b4[j, kk])) * X.E4M3[int(sb[j, kk // 16])]
            y[i, j] = float(acc * aa * ab)
    return y


def random_operands(rng, m, n, k):
    a4 = rng.integers(0, 16, size=(m, k))
    b4 = rng.integers(0, 16, size=(n, k))
    sa = rng.integers(0, 0x7F, size=(m, k // 16))          # every finite non-negative E4M3 code
    sb = rng.integers(0, 0x7F, size=(n, k // 16))
    return a4, sa, b4, sb


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(500 + seed)
    m, n, k = 3, 2, 48
    a4, sa, b4, sb = random_operands(rng, m, n, k)
    alpha_a, alpha_b = np.float32(rng.uniform(1e-3, 3.0)), np.float32(rng.uniform(1e-3, 3.0))
    got = O.gemm_nvfp4(pack(a4), sa, alpha_a, pack(b4), sb, alpha_b, m, n, k)
    want = exact_gemm(a4, sa, alpha_a, b4, sb, alpha_b)
    assert np.array_equal(got, want)


def test_one_hot_weights_reproduce_the_activations():
    """B row j has a single 1.0 at k = j (code 2, scale 0x38 = 1.0, alpha 1): Y[:, j] is the
    exact value of A[:, j] times alpha_a."""
    rng = np.random.default_rng(7)
    m, n, k = 5, 32, 32
    a4 = rng.integers(0, 16, size=(m, k))
    sa = rng.integers(0x08, 0x7F, size=(m, k // 16))
    b4 = np.zeros((n, k), np.int64)
    b4[np.arange(n), np.arange(n)] = 2
    sb = np.full((n, k // 16), 0x38)
    alpha_a = np.float32(0.3)
    got = O.gemm_nvfp4(pack(a4), sa, alpha_a, pack(b4), sb, 1.0, m, n, k)
    aa = X.f32_value(float(alpha_a))
    want = np.array([[float(e2m1(int(a4[i, j])) * X.E4M3[int(sa[i, j // 16])] * aa) for j in range(n)] for i in range(m)])
    assert np.array_equal(got, want)


def mutated(kind):
    """A copy of the reference with one plausible slip."""
    def f(a_codes, a_scales, a_alpha, b_codes, b_scales, b_alpha, m, n, k):
        if kind == "nibbles":
            a_codes = ((np.asarray(a_codes) >> 4) | (np.asarray(a_codes) << 4)).astype(np.uint8)
        if kind == "no_alpha":
            b_alpha = 1.0
        if kind == "scale_per_32":
            s = np.asarray(a_scales).reshape(m, k // 16)
            a_scales = np.repeat(s[:, 0::2], 2, axis=1)[:, : k // 16]
        y = O.gemm_nvfp4(a_codes, a_scales, a_alpha, b_codes, b_scales, b_alpha, m, n, k)
        if kind == "transposed":
            y = (O.gemm_nvfp4(b_codes, b_scales, b_alpha, a_codes, a_scales, a_alpha, n, m, k).T)[::-1]
        return y
    return f


@pytest.mark.parametrize("kind", ["nibbles", "no_alpha", "scale_per_32", "transposed"])
def test_pins_reject_mutants(kind):
    rng = np.random.default_rng(501)
    m, n, k = 3, 2, 64
    a4, sa, b4, sb = random_operands(rng, m, n, k)
    alpha_a, alpha_b = np.float32(0.7), np.float32(1.9)
    got = mutated(kind)(pack(a4), sa, alpha_a, pack(b4), sb, alpha_b, m, n, k)
    assert not np.array_equal(got, exact_gemm(a4, sa, alpha_a, b4, sb, alpha_b))
