"""Hardware instruction semantics on the B200 against the oracle's scalar definitions and
IEEE host arithmetic: E2M1 / E4M3 conversions (rounding, ties, saturation, sign of zero),
their exact decodes, BF16 rounding, and the IEEE round-to-nearest arithmetic the kernels use
(reciprocal, division, packed .f32x2 mul/sub/add/fma), subnormals included."""
import ctypes
import struct
from fractions import Fraction as F

import numpy as np
import pytest
import torch

import oracle as O
from tests import exact as X
from tests.probe import build as probe_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def probe(gpu):
    L = ctypes.CDLL(probe_build.build())
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.probe_e2m1.argtypes = [vp, vp, i64, i32]
    L.probe_e4m3.argtypes = [vp, vp, i64]
    L.probe_decode.argtypes = [vp, vp]
    L.probe_bf16.argtypes = [vp, vp, i64]
    L.probe_arith.argtypes = [i32, vp, vp, vp, vp, i64]
    return L


def _run_conv(probe, fn, x: np.ndarray, out_dtype, *extra):
    xd = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    out = torch.empty(x.size, dtype=torch.uint8 if out_dtype == np.uint8 else torch.int16, device="cuda")
    assert getattr(probe, fn)(xd.data_ptr(), out.data_ptr(), x.size, *extra) == 0
    assert probe.probe_sync() == 0
    return out.cpu().numpy().view(out_dtype)


def _binades(lo_exp_field, hi_exp_field):
    """Every positive binary32 whose exponent field is in [lo, hi)."""
    bits = np.arange(lo_exp_field << 23, hi_exp_field << 23, dtype=np.uint32)
    return bits.view(np.float32)


def _samples(rng, n):
    u = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    return f[np.isfinite(f)]


def test_e2m1_exhaustive_against_oracle(probe):
    rng = np.random.default_rng(0)
    # every binary32 in [2^-3, 2^3) (all of E2M1's decisions: 0.25 ... 5 and saturation),
    # plus random patterns of every magnitude and sign, zeros and infinities
    x = np.concatenate([_binades(124, 130), _samples(rng, 4_000_000),
                        np.array([0.0, -0.0, np.inf, -np.inf, 6.0, -6.0, 1e-45, -1e-45], np.float32)])
    x = np.concatenate([x, -x[:1_000_000]])
    want = O.f32_to_e2m1_array(x)
    for high in (0, 1):
        got = _run_conv(probe, "probe_e2m1", x, np.uint8, high)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (high, x[bad[:10]], got[bad[:10]], want[bad[:10]])


def test_e4m3_exhaustive_against_oracle(probe):
    rng = np.random.default_rng(1)
    # every binary32 in [2^-11, 2^10) (E4M3 subnormals, normals, saturation past 448)
    x = np.concatenate([_binades(116, 137), _samples(rng, 4_000_000),
                        np.array([0.0, -0.0, np.inf, 448.0, 464.0, 480.0, 1e30], np.float32)])
    x = np.concatenate([x, -x[-3_000_000:]])
    want = O.f32_to_e4m3_array(x)
    got = _run_conv(probe, "probe_e4m3", x, np.uint8)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (x[bad[:10]], got[bad[:10]], want[bad[:10]])


def test_decodes_exact_and_nibble_order(probe):
    e2 = torch.empty(512, dtype=torch.float32, device="cuda")
    e4 = torch.empty(131072, dtype=torch.float32, device="cuda")
    assert probe.probe_decode(e2.data_ptr(), e4.data_ptr()) == 0
    e2 = e2.cpu().numpy().reshape(256, 2)
    e4 = e4.cpu().numpy().reshape(65536, 2)
    for b in range(256):
        lo, hi = O.e2m1_to_f32([b & 0xF])[0], O.e2m1_to_f32([b >> 4])[0]
        assert e2[b, 0] == lo and np.signbit(e2[b, 0]) == np.signbit(lo), b
        assert e2[b, 1] == hi and np.signbit(e2[b, 1]) == np.signbit(hi), b
    codes = np.arange(256, dtype=np.uint8)
    ref = O.e4m3_to_f32(codes)
    finite = np.isfinite(ref)
    lo_want = ref[np.arange(65536) & 0xFF]
    hi_want = ref[np.arange(65536) >> 8]
    mask = finite[np.arange(65536) & 0xFF] & finite[np.arange(65536) >> 8]
    assert np.array_equal(e4[mask, 0], lo_want[mask]) and np.array_equal(e4[mask, 1], hi_want[mask])


def test_bf16_rounding_against_oracle(probe):
    rng = np.random.default_rng(2)
    ties = ((rng.integers(0, 2**16, 200_000, dtype=np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([_samples(rng, 2_000_000), ties[np.isfinite(ties)],
                        np.array([3.3961776e38, 3.40282e38, -3.40282e38, 1e-45, -0.0], np.float32)])
    want = O.f32_to_bf16_array(x)
    got = _run_conv(probe, "probe_bf16", x, np.uint16)
    assert np.array_equal(got, want)


def _arith(probe, op, a, b, c):
    n = a.size
    ad, bd, cd = (torch.from_numpy(np.ascontiguousarray(v, np.float32)).cuda() for v in (a, b, c))
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    assert probe.probe_arith(op, ad.data_ptr(), bd.data_ptr(), cd.data_ptr(), out.data_ptr(), n) == 0
    assert probe.probe_sync() == 0
    return out.cpu().numpy()


def _operands(rng, n):
    """Finite operands across the range, a quarter of them subnormal."""
    a = _samples(rng, n)
    sub = (rng.integers(1, 2**23, n // 4, dtype=np.uint32)).view(np.float32)
    a = np.concatenate([a, sub])[: n // 2 * 2]
    return a[: a.size // 2 * 2]


@pytest.mark.parametrize("op", [0, 1, 2, 3, 4])
def test_ieee_round_to_nearest_ops(probe, op):
    rng = np.random.default_rng(10 + op)
    a = _operands(rng, 1_000_000)
    b = _operands(rng, a.size)[: a.size]
    a = a[: b.size]
    c = np.zeros_like(a)
    got = _arith(probe, op, a, b, c)
    with np.errstate(all="ignore"):
        want = {0: np.float32(1.0) / a, 1: a / b, 2: a * b, 3: a - b, 4: a + b}[op]
    same = (got.view(np.uint32) == want.view(np.uint32)) | (np.isnan(got) & np.isnan(want))
    assert same.all(), (op, a[~same][:5], b[~same][:5], got[~same][:5], want[~same][:5])


def test_packed_fma_is_single_rounding(probe):
    rng = np.random.default_rng(20)
    n = 40_000
    a = _operands(rng, n)[:n]
    b = np.float32(1.0) + rng.standard_normal(n).astype(np.float32) * np.float32(1e-3)
    c = (-(a.astype(np.float64) * b) * (1 + rng.standard_normal(n) * 1e-7)).astype(np.float32)
    keep = np.isfinite(a * b) & (np.abs(a) > 1e-30) & (np.abs(a) < 1e30)
    a, b, c = a[keep][:20000], b[keep][:20000], c[keep][:20000]
    got = _arith(probe, 5, a, b, c)
    for i in range(a.size):
        want = X.round_f32(F(float(a[i])) * F(float(b[i])) + F(float(c[i])))
        assert want is not None and F(float(got[i])) == want, (a[i], b[i], c[i], got[i], float(want))


def test_error_term_single_rounding(probe):
    """x - v*d as the kernels compute it (one fused multiply-add, fma.rn.f32x2 with -d) is
    the exact difference rounded once; the operands make that differ from rounding the
    product first, so the data tells the two apart."""
    rng = np.random.default_rng(31)
    n = 200_000
    v = rng.choice(np.array([0.5, 1, 1.5, 2, 3, 4, 6], np.float32), n).astype(np.float32)
    d = (np.float32(1.0) + rng.random(n, dtype=np.float32)).astype(np.float32)
    x = (v.astype(np.float64) * d * (1 + rng.standard_normal(n) * 1e-6)).astype(np.float32)
    got = _arith(probe, 5, v, -d, x)
    exact = x.astype(np.float64) - v.astype(np.float64) * d.astype(np.float64)   # exact: 24+3 bit product
    want = exact.astype(np.float32)
    two = x - v * d
    assert int((want.view(np.uint32) != two.view(np.uint32)).sum()) > 1000
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
