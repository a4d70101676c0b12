"""Pins of the oracle's QAD distillation loss (CPU): KL(p || q) with p = softmax(teacher),
q = softmax(student), and its gradient with respect to the student logits.
Source: "Quantization-Aware Distillation for NVFP4 Inference Accuracy Recovery", technical
summary §2 (L_QAD = D_KL(p_teacher || p_student))."""
import math

import numpy as np
import pytest

import oracle as O
from nvfp4_block_scaled_13_b200 import synth


def bf16(a):
    return synth.to_bf16_bits(np.asarray(a, np.float32))


def bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_kl_of_identical_distributions_is_zero():
    rng = np.random.default_rng(0)
    t = bf16(rng.normal(0, 3, (4, 257)))
    kl, g = O.qad_kl(t, t, 4, 257)
    assert np.all(np.abs(kl) < 1e-14) and np.all(np.abs(g) < 1e-15)


def test_two_outcome_closed_form():
    # teacher logits (a, 0), student logits (b, 0): p = sigmoid(a), q = sigmoid(b)
    for a, b in [(1.0, -1.0), (2.5, 0.5), (-3.0, 4.0), (0.0, 0.0)]:
        t, s = bf16([[a, 0.0]]), bf16([[b, 0.0]])
        kl, g = O.qad_kl(t, s, 1, 2)
        p, q = 1 / (1 + math.exp(-a)), 1 / (1 + math.exp(-b))
        want = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
        assert abs(kl[0] - want) < 1e-13
        assert abs(g[0] - (q - p)) < 1e-15 and abs(g[1] - ((1 - q) - (1 - p))) < 1e-15


def test_invariant_to_shifting_each_row():
    # logits on a 1/8 grid in [-8, 8): adding 3.5 keeps every value exact in BF16
    rng = np.random.default_rng(1)
    t = (rng.integers(-64, 64, (3, 100)) / 8.0).astype(np.float32)
    s = (rng.integers(-64, 64, (3, 100)) / 8.0).astype(np.float32)
    base, gb = O.qad_kl(bf16(t), bf16(s), 3, 100)
    shifted, gs = O.qad_kl(bf16(t + 3.5), bf16(s - 3.5), 3, 100)
    assert np.allclose(base, shifted, rtol=0, atol=1e-13)
    assert np.allclose(gb, gs, rtol=0, atol=1e-15)


def test_gradient_sums_to_zero_and_matches_finite_differences():
    rng = np.random.default_rng(2)
    vocab = 7
    t = bf16(rng.normal(0, 1, (1, vocab)))
    s = bf16(rng.normal(0, 1, (1, vocab)))
    kl, g = O.qad_kl(t, s, 1, vocab)
    assert abs(g.sum()) < 1e-15
    # finite differences in binary64 of the same definition, perturbing the student logits
    tv, sv = bf16_value(t), bf16_value(s)

    def kl64(svec):
        lp = tv - (tv.max() + np.log(np.exp(tv - tv.max()).sum()))
        lq = svec - (svec.max() + np.log(np.exp(svec - svec.max()).sum()))
        return float((np.exp(lp) * (lp - lq)).sum())

    assert abs(kl64(sv) - kl[0]) < 1e-14
    for v in range(vocab):
        e = np.zeros(vocab)
        e[v] = 1e-6
        fd = (kl64(sv + e) - kl64(sv - e)) / 2e-6
        assert abs(fd - g[v]) < 1e-7


def test_temperature_and_grad_scale():
    rng = np.random.default_rng(3)
    t = bf16(rng.normal(0, 4, (2, 50)))
    s = bf16(rng.normal(0, 4, (2, 50)))
    k2, g2 = O.qad_kl(t, s, 2, 50, tau=2.0, grad_scale=0.25)
    tv, sv = bf16_value(t).reshape(2, 50) / 2.0, bf16_value(s).reshape(2, 50) / 2.0
    lp = tv - np.log(np.exp(tv).sum(1, keepdims=True))
    lq = sv - np.log(np.exp(sv).sum(1, keepdims=True))
    assert np.allclose(k2, (np.exp(lp) * (lp - lq)).sum(1), rtol=1e-12, atol=1e-14)
    assert np.allclose(g2.reshape(2, 50), 0.25 * (np.exp(lq) - np.exp(lp)), rtol=1e-12, atol=1e-16)


def test_kl_is_non_negative_and_large_for_disjoint_peaks():
    t = np.full((1, 64), -20.0, np.float32)
    s = np.full((1, 64), -20.0, np.float32)
    t[0, 3] = 20.0
    s[0, 40] = 20.0
    kl, _ = O.qad_kl(bf16(t), bf16(s), 1, 64)
    assert 39.9 < kl[0] < 40.1                # about 40 nats: log p/q at the teacher's peak
    rng = np.random.default_rng(4)
    for _ in range(5):
        a, b = bf16(rng.normal(0, 3, (8, 33))), bf16(rng.normal(0, 3, (8, 33)))
        assert np.all(O.qad_kl(a, b, 8, 33, with_grad=False)[0] >= -1e-15)
