"""The division-free block-scale rule of the quantizer kernels, checked on the CPU against the
exact quotient.

The kernels compute s = E4M3(RN(m / beta)) without a division: a bracket lo = RN(m yl),
hi = RN(m yh) decides when E4M3(lo) == E4M3(hi); otherwise the two codes are adjacent and the
boundary M between them is hi with its significand cut to 5 bits, and the sign of the exact
d = m - beta M against +-beta ulp(M) / 2 (ties to the even code) decides. This file restates
that rule in numpy, independently of the kernels and of the oracle, and compares it with
E4M3 of the correctly rounded binary32 quotient (numpy's float32 division) on every BF16 block
maximum around every E4M3 boundary for a range of tensor scales, plus random ones. It also
checks the premise of the kernels' exactness argument: d is a binary32 number (so one fused
multiply-add gives it exactly) whenever the rule reaches it."""
import numpy as np
import torch

F32 = np.float32


def e4m3(v: np.ndarray) -> np.ndarray:
    """Binary32 (non-negative) -> E4M3 code, round to nearest even, saturating at 448."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).clamp(max=448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)


def boundaries() -> np.ndarray:
    v = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    return ((v[:-1] + v[1:]) / 2).astype(np.float32)


def rule(m: np.ndarray, beta: np.float32):
    """(codes by the kernels' rule, whether the boundary test was used, d as float64)."""
    y = F32(F32(1.0) / beta)
    yl, yh = F32(y * F32(1 - 2.0**-20)), F32(y * F32(1 + 2.0**-20))
    with np.errstate(over="ignore"):   # huge maxima: the products saturate to 448 like the quotient
        lo, hi = (m * yl).astype(np.float32), (m * yh).astype(np.float32)
    s_lo, s_hi = e4m3(lo), e4m3(hi)
    out = s_lo.copy()
    at = s_lo != s_hi
    mid = (hi[at].view(np.uint32) & np.uint32(0xFFF80000)).view(np.float32)
    d = m[at].astype(np.float64) - np.float64(beta) * mid.astype(np.float64)      # exact in binary64
    up = ((mid.view(np.uint32) & np.uint32(0x7F800000)) - np.uint32(24 << 23)).view(np.float32)
    bu = np.float64(beta) * up.astype(np.float64)                                 # exact
    odd = (s_lo[at] & 1) == 1
    take_hi = np.where(odd, d >= -bu, d > bu)
    out[at] = np.where(take_hi, s_hi[at], s_lo[at])
    return out, at, d


def test_rule_equals_e4m3_of_the_rounded_quotient():
    mids = boundaries()
    rng = np.random.default_rng(0)
    # tensor scales from BF16 amax values over a wide range, both modes' beta = K alpha
    amaxes = (np.arange(0x3000, 0x4700, 7, dtype=np.uint32) << 16).view(np.float32)
    n_boundary = n_total = 0
    for amax in amaxes:
        for six_m, k in ((F32(1536.0), F32(6.0)), (F32(1536.0), F32(4.0)), (F32(2688.0), F32(6.0))):
            beta = F32(k * F32(amax / six_m))
            if not (2.0**-90 <= beta <= 2.0**125):
                continue
            # BF16 neighbours of beta M for every boundary M, and random BF16 block maxima
            t = (np.float64(beta) * mids).astype(np.float32).view(np.uint32).astype(np.int64)
            near = np.concatenate([((t >> 16) + dk) << 16 for dk in (-2, -1, 0, 1, 2)])
            near = near[(near >= 0) & (near < 2**32)].astype(np.uint32)
            rand = (rng.integers(0x0080, 0x7F80, 64, dtype=np.uint32) << 16)
            m = np.concatenate([near, rand]).view(np.float32)
            m = m[np.isfinite(m) & (m >= 0)]
            with np.errstate(over="ignore"):
                want = e4m3((m / beta).astype(np.float32))
            got, at, d = rule(m, beta)
            assert np.array_equal(got, want), (amax, beta, m[got != want][:4])
            # the premise of the exactness argument: d is a binary32 number
            assert np.all(d.astype(np.float32).astype(np.float64) == d)
            n_boundary += int(at.sum())
            n_total += m.size
    print(f"{n_boundary} of {n_total} block maxima needed the boundary test")
    assert n_boundary > 10_000, n_boundary   # the boundary test was exercised, not just the bracket
    assert n_total > 500_000


# ---- the threshold form of the rule ------------------------------------------------------------

def e4m3_values() -> np.ndarray:
    return torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def thresholds(beta: np.float32) -> np.ndarray:
    """T[s] = the smallest BF16 value m >= 0 with E4M3(RN(m / beta)) >= s (as binary32; T[0] = 0,
    T[127] = +inf), from the E4M3 rounding boundary between codes s - 1 and s: ties go to the
    even code, so code s needs RN(m / beta) >= M (s even) or > M (s odd), i.e. m / beta at or
    past the binary32 midpoint next to M on the matching side. beta times that midpoint is exact
    in binary64; it is rounded up to binary32 and then to BF16, and stepped once more when a
    strict comparison meets it exactly."""
    v = e4m3_values().astype(np.float32)
    T = np.full(128, np.inf, np.float32)
    T[0] = 0.0
    if not beta > 0:
        return T
    for s in range(1, 127):
        M = np.float32((v[s - 1] + v[s]) / 2)
        odd = s & 1
        nb = np.nextafter(M, np.float32(np.inf) if odd else np.float32(0))
        V = np.float64(beta) * ((np.float64(M) + np.float64(nb)) / 2)
        with np.errstate(over="ignore"):
            vf = np.float32(V)
        if np.float64(vf) < V:
            vf = np.nextafter(vf, np.float32(np.inf))
        t = (int(vf.view(np.uint32)) + 0xFFFF) & 0xFFFF0000
        if odd and np.float64(np.uint32(t).view(np.float32)) == V:
            t += 0x10000
        T[s] = np.uint32(min(t, 0x7F800000)).view(np.float32)
    return T


def threshold_rule(m: np.ndarray, beta: np.float32, T: np.ndarray) -> np.ndarray:
    y = F32(F32(1.0) / beta)
    yl = F32(y * F32(1 - 2.0**-20))
    with np.errstate(over="ignore"):
        lo = (m * yl).astype(np.float32)
    s_lo = e4m3(lo)
    return s_lo + (m >= T[np.minimum(s_lo + 1, 127)]).astype(np.int64)


def test_threshold_rule_equals_e4m3_of_the_rounded_quotient_for_every_bf16_maximum():
    """Every positive finite BF16 value as a block maximum, under tensor scales of both modes
    (among them amaxes with short binary expansions, whose quotients hit E4M3 boundaries
    exactly): E4M3(lo) plus one threshold comparison equals E4M3(RN(m / beta))."""
    m = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(1)
    amaxes = np.concatenate([np.array([0.1171875, 5.5, 6.09375, 1.0, 448.0, 3.0e-5, 2.0**-100 * 3], np.float32),
                             (rng.integers(0x2000, 0x5F00, 40, dtype=np.uint32) << 16).view(np.float32)])
    hits = 0
    for amax in amaxes:
        for six_m, k in ((F32(1536.0), F32(6.0)), (F32(1536.0), F32(4.0)), (F32(2688.0), F32(6.0))):
            beta = F32(k * F32(amax / six_m))
            if not (2.0**-90 <= beta <= 2.0**125):
                continue
            T = thresholds(beta)
            with np.errstate(over="ignore"):
                want = e4m3((m / beta).astype(np.float32))
            got = threshold_rule(m, beta, T)
            assert np.array_equal(got, want), (amax, beta, m[got != want][:4], got[got != want][:4],
                                               want[got != want][:4])
            y = F32(F32(1.0) / beta)
            with np.errstate(over="ignore"):
                hits += int((e4m3((m * F32(y * F32(1 - 2.0**-20))).astype(np.float32)) != want).sum())
    assert hits > 300, hits     # the threshold comparison changed the code, not only the product
