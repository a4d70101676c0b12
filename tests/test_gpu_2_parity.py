"""GPU path vs the oracle, bit for bit, through the C ABI: every output (amax, tensor scale,
E4M3 scales, E2M1 codes, choice bits, fake-quant BF16, dequantized BF16) on the five
workloads' distributions at sizes the oracle finishes in seconds (several CTAs, grid-stride
passes, ragged tails, group boundaries inside a warp), random shapes, adversarial blocks,
and the edge cases of the method; plus guard canaries around every output, host-side
argument errors that leave outputs untouched, and non-default streams."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

MODES = [(0, 2), (1, 0), (1, 1), (1, 2)]      # scale-6; Four Over Six with max / MAE / MSE
MODE_IDS = ["scale6", "46max", "46mae", "46mse"]


# (config, rows, cols, groups): ragged block counts, group sizes that are not multiples of
# 32 blocks, and two cases large enough for several grid-stride passes per thread.
SMALL = [
    ("c1", 256, 1024, 1),
    ("c2", 517, 4080, 1),
    ("c3", 333, 4096, 1),
    ("c4", 129, 1008, 3),
    ("c5", 301, 8176, 1),
]
LARGE = [
    ("c5", 733, 8176, 1),      # 6.0 M elements, 374 k blocks (ragged)
    ("c4", 1001, 1008, 5),     # 5.0 M elements, 5 groups of 63 063 blocks
]


@pytest.mark.parametrize("mode,rule", MODES, ids=MODE_IDS)
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}x{c[3]}")
def test_parity_small(gpu, case, mode, rule):
    name, rows, cols, groups = case
    x, (g, r, c) = synth.make(name, rows=rows, cols=cols, groups=groups)
    U.check_case(x, g, r, c, mode, rule)


@pytest.mark.parametrize("mode,rule", [(0, 2), (1, 2), (1, 1)], ids=["scale6", "46mse", "46mae"])
@pytest.mark.parametrize("case", LARGE, ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}x{c[3]}")
def test_parity_grid_stride(gpu, case, mode, rule):
    name, rows, cols, groups = case
    x, (g, r, c) = synth.make(name, rows=rows, cols=cols, groups=groups)
    U.check_case(x, g, r, c, mode, rule, dequant=False)


@pytest.mark.parametrize("seed", range(24))
def test_parity_random_shapes(gpu, seed):
    x, (g, r, c) = synth.random_case(seed)
    mode, rule = MODES[seed % 4]
    U.check_case(x, g, r, c, mode, rule)


def _adversarial(M):
    """Blocks built to sit on decision boundaries. With amax = 6M the tensor scale is 1 and
    power-of-two block maxima give exact scaled values."""
    rng = np.random.default_rng(99)
    six_m = 6.0 * M
    blocks = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for s in [2.0 ** k for k in range(-3, 9)]:
        # one element at 6s (block maximum -> scale s for target 6), the rest on midpoints
        blocks.append([6 * s] + [mids[i % 7] * s * (-1) ** i for i in range(15)])
        # target-4 friendly: maximum 4s' and three-quarter values
        blocks.append([4 * s, 3 * s, -3 * s, 0.75 * 4 * s] + [2 * s, -1.5 * s] * 6)
        # values near 5/6 of the maximum: the pages' "size 5" gap
        blocks.append([6 * s, 5 * s, -5 * s, 4.5 * s, 5.5 * s, 4 * s] + [5 * s] * 10)
    blocks.append([1.0] * 16)                                          # all equal
    blocks.append([six_m] + [2.0 ** -60] * 15)                         # single outlier
    blocks.append([0.0, -0.0] * 8)                                     # signed zeros
    blocks.append([2.0 ** -130 * (i + 1) for i in range(16)])          # BF16 subnormals
    blocks.append([1e-6 * v for v in rng.standard_normal(16)])         # tiny: scale underflow
    blocks.append([3.3895e38, -3.3895e38] + [1e38] * 14)               # near BF16 max
    blocks.append([six_m * 0.75] * 8 + [six_m * 0.5] * 8)
    x = np.array([v for b in blocks for v in b], np.float32)
    return synth.to_bf16_bits(x)


@pytest.mark.parametrize("mode,rule", MODES, ids=MODE_IDS)
def test_parity_adversarial_blocks(gpu, mode, rule):
    M = 256.0 if mode == 1 else 448.0
    x = _adversarial(M)
    n = x.size
    # amax = 6M (tensor scale exactly 1) for exact ties; the true amax; a BF16-subnormal amax
    for amax in (6 * M, None):
        a = None if amax is None else np.array([amax], np.float32)
        U.check_case(x, 1, n // 16, 16, mode, rule, amax_np=a)
    tiny = synth.to_bf16_bits(np.float32(2.0 ** -130) * np.arange(1, 33, dtype=np.float32))
    U.check_case(tiny, 1, 2, 16, mode, rule)


@pytest.mark.parametrize("mode,rule", MODES, ids=MODE_IDS)
def test_parity_static_amax(gpu, mode, rule):
    """A calibrated (static) amax: below the true maximum (saturation), above it, and zero."""
    x, (g, r, c) = synth.make("c3", rows=64, cols=1024)
    true = O.amax(x, g, r, c)
    for factor in (0.25, 1.0, 3.0, 0.0):
        U.check_case(x, g, r, c, mode, rule, amax_np=(true * np.float32(factor)).astype(np.float32))


def test_zero_and_one_block_tensors(gpu):
    for mode, rule in MODES:
        zero = np.zeros(16 * 40, np.uint16)
        U.check_case(zero, 2, 20, 16, mode, rule)
        one = synth.to_bf16_bits(np.arange(-8, 8, dtype=np.float32))
        U.check_case(one, 1, 1, 16, mode, rule)


def test_empty_tensors(gpu):
    dummy = torch.zeros(16, dtype=torch.int16, device="cuda")
    # amax of an empty group is 0
    out = U.Guarded(12, fill=0x7F)
    nv.nvfp4_amax(dummy.data_ptr(), 3, 0, 64, out.ptr())
    torch.cuda.synchronize()
    assert out.guards_intact() and not out.numpy(np.float32).any()
    # quantize of an empty tensor writes only the tensor scales
    amax = torch.tensor([2688.0, 0.0, 5376.0], device="cuda")
    ts = U.Guarded(12)
    codes = U.Guarded(64, fill=0x11)
    nv.nvfp4_quantize(dummy.data_ptr(), 3, 0, 64, amax.data_ptr(), 0, 2, codes.ptr(), codes.ptr(), ts.ptr(), None)
    torch.cuda.synchronize()
    assert list(ts.numpy(np.float32)) == [1.0, 0.0, 2.0]
    assert ts.guards_intact() and codes.guards_intact() and (codes.numpy() == 0x11).all()
    # fake-quant and dequantize of an empty tensor do nothing
    y = U.Guarded(64, fill=0x22)
    nv.nvfp4_fakequant(dummy.data_ptr(), 1, 4, 0, amax.data_ptr(), 1, 2, y.ptr(), None)
    nv.nvfp4_dequantize(codes.ptr(), codes.ptr(), ts.ptr(), 1, 0, 16, y.ptr())
    torch.cuda.synchronize()
    assert (y.numpy() == 0x22).all() and y.guards_intact()


def test_errors_leave_outputs_untouched(gpu):
    x, (g, r, c) = synth.make("c1", rows=8, cols=64)
    xd = U.to_device_bf16(x)
    amax = torch.ones(1, device="cuda")
    codes, scales, ts, ch = U.Guarded(256, 0x33), U.Guarded(32, 0x33), U.Guarded(4, 0x33), U.Guarded(4, 0x33)
    for args, status in [
        ((xd.data_ptr(), 1, 8, 60), 2),                 # cols % 16 != 0
        ((xd.data_ptr() + 2, 1, 8, 64), 3),             # misaligned x
    ]:
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.nvfp4_quantize(*args, amax.data_ptr(), 1, 2, codes.ptr(), scales.ptr(), ts.ptr(), ch.ptr())
        assert e.value.status == status
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.nvfp4_quantize(xd.data_ptr(), 1, 8, 64, amax.data_ptr(), 1, 5, codes.ptr(), scales.ptr(), ts.ptr(),
                          ch.ptr())
    assert e.value.status == 5
    torch.cuda.synchronize()
    for b in (codes, scales, ts, ch):
        assert (b.numpy() == 0x33).all() and b.guards_intact()


def test_side_stream_and_choice_optional(gpu):
    x, (g, r, c) = synth.make("c2", rows=64, cols=4096)
    xd = U.to_device_bf16(x)
    amax = O.amax(x, g, r, c)
    want = O.quantize(x, g, r, c, amax, 1, 2)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got = U.gpu_quantize(xd, g, r, c, amax, 1, 2, with_choice=False, stream=s)
    for k in ("codes", "scales", "tscale"):
        U.assert_same(k, got[k], want[k])


def test_python_wrappers_round_trip(gpu):
    x, (g, r, c) = synth.make("c4", rows=64, cols=256, groups=4)
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16).reshape(g, r, c)
    q = nv.quantize(xt, "four_over_six", "mse", groups=g)
    y = nv.dequantize(q)
    fq = nv.fakequant(xt, "four_over_six", "mse", groups=g)
    torch.cuda.synchronize()
    assert torch.equal(y.view(-1).view(torch.int16), fq.reshape(-1).view(torch.int16))
    want = O.quantize(x, g, r, c, O.amax(x, g, r, c), 1, 2)
    U.assert_same("codes", q.codes.cpu().numpy(), want["codes"])
    U.assert_same("choice", q.choice.cpu().numpy(), want["choice"])


# ---- block maxima whose scale quotient RN(m / beta) lies exactly on an E4M3 rounding boundary ----

def _e4m3_boundaries() -> np.ndarray:
    """Midpoints between consecutive non-negative E4M3 values (exact in binary32)."""
    v = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    return ((v[:-1] + v[1:]) / 2).astype(np.float32)


def _boundary_groups(mode: int, n_groups: int):
    """(amax, [(m, exact)]) for tensor maxima amax whose betas send some BF16 block maxima m
    exactly onto an E4M3 boundary: m / beta equal to it (exact) or only rounded onto it."""
    mids = _e4m3_boundaries()
    ks = (6.0, 4.0) if mode == 1 else (6.0,)
    bits = np.arange(0x3D00, 0x41F0, dtype=np.uint32)                 # BF16 amax in [0.031, 30)
    found = []
    for amax in (bits << 16).view(np.float32):
        alpha = np.float32(O.tensor_scale(float(amax), mode))
        hits = []
        for k in ks:
            beta = np.float32(np.float32(k) * alpha)
            target = beta.astype(np.float64) * mids
            for rnd in (np.floor, np.ceil):                             # the two BF16 neighbours
                t = target.astype(np.float32).view(np.uint32).astype(np.int64)
                hi16 = rnd(t / 65536.0).astype(np.int64)
                m = (hi16.astype(np.uint32) << 16).view(np.float32)
                ok = (m > 0) & (m < amax) & ((m / beta).astype(np.float32) == mids)
                for mv, mid in zip(m[ok], mids[ok]):
                    hits.append((np.float32(mv), bool(np.float64(mv) == np.float64(beta) * np.float64(mid))))
        if hits:
            hits.sort(key=lambda h: h[1])                                # rounded-onto ones first
            found.append((np.float32(amax), hits))
    # most hits first, keeping both kinds
    found.sort(key=lambda f: -len(f[1]))
    exact = [f for f in found if any(e for _, e in f[1])][: n_groups // 2]
    rounded = [f for f in found if any(not e for _, e in f[1]) and f not in exact][: n_groups - len(exact)]
    return exact + rounded


def _boundary_tensor(groups, blocks_per_group: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    out = []
    for amax, hits in groups:
        blocks = [np.concatenate([[amax], rng.uniform(-1, 1, 15) * amax * 0.9])]
        for m, _ in hits[: blocks_per_group - 1]:
            b = rng.uniform(-1, 1, 16) * m * 0.95
            b[rng.integers(0, 16)] = m if rng.random() < 0.5 else -m
            blocks.append(b)
        while len(blocks) < blocks_per_group:
            blocks.append(rng.standard_normal(16) * amax * 0.1)
        out.append(np.concatenate(blocks))
    return synth.to_bf16_bits(np.concatenate(out).astype(np.float32))


@pytest.mark.parametrize("mode,rule", MODES, ids=MODE_IDS)
def test_parity_scale_on_e4m3_boundary(gpu, mode, rule):
    """Blocks whose scale quotient RN(m / beta) sits exactly on an E4M3 rounding boundary, where
    the division-free bracket cannot decide and the boundary test or the tie-to-even rule
    does: both the exact quotients and those rounded onto the boundary, each in its own
    group's tensor scale, through the grouped kernel (64 blocks per group) and the flat one
    (65)."""
    groups = _boundary_groups(mode, 24)
    for bpg in (64, 65):
        used = [e for _, h in groups for _, e in h[: bpg - 1]]
        assert sum(used) >= 100 and len(used) - sum(used) >= 20, (sum(used), len(used))
        x = _boundary_tensor(groups, bpg, seed=bpg)
        U.check_case(x, len(groups), bpg, 16, mode, rule)


# ---- amax and quantization in one launch (a grid-wide wait between them) ------------------------

# one group (ragged), several groups of whole warp words (one launch), and several groups whose
# block count is not a multiple of 32 (the two launches)
ONE_LAUNCH = [("c1", 256, 1024, 1), ("c2", 517, 4080, 1), ("c4", 128, 1024, 4), ("c4", 129, 1008, 3),
              ("c5", 301, 8176, 1)]


@pytest.mark.parametrize("mode,rule", MODES, ids=MODE_IDS)
@pytest.mark.parametrize("case", ONE_LAUNCH, ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}x{c[3]}")
def test_parity_amax_in_the_same_launch(gpu, case, mode, rule):
    name, rows, cols, groups = case
    x, (g, r, c) = synth.make(name, rows=rows, cols=cols, groups=groups)
    n, nb = g * r * c, g * r * c // 16
    want_amax = O.amax(x, g, r, c)
    want = O.quantize(x, g, r, c, want_amax, mode, rule)
    wfq = O.fakequant(x, g, r, c, want_amax, mode, rule)
    xd = U.to_device_bf16(x)
    amax, tscale = U.Guarded(4 * g), U.Guarded(4 * g)
    codes, scales, choice = U.Guarded(n // 2), U.Guarded(nb), U.Guarded((nb + 7) // 8)
    work = torch.zeros(2, dtype=torch.int32, device="cuda")     # [0] workspace, [1] status
    nv.nvfp4_amax_quantize(xd.data_ptr(), g, r, c, mode, rule, amax.ptr(), codes.ptr(), scales.ptr(), tscale.ptr(),
                           choice.ptr(), work[0:1].data_ptr(), work[1:2].data_ptr())
    torch.cuda.synchronize()
    assert work[1].item() == 0
    assert all(b.guards_intact() for b in (amax, tscale, codes, scales, choice)), "write outside an output buffer"
    U.assert_same("amax", amax.numpy(np.float32), want_amax)
    U.assert_same("tscale", tscale.numpy(np.float32), want["tscale"])
    for k, buf in (("codes", codes), ("scales", scales), ("choice", choice)):
        U.assert_same(k, buf.numpy(), want[k])
    # fake-quant, twice in a row on the library's own workspace word
    for _ in range(2):
        amax2, y, choice2 = U.Guarded(4 * g), U.Guarded(2 * n), U.Guarded((nb + 7) // 8)
        nv.nvfp4_amax_fakequant(xd.data_ptr(), g, r, c, mode, rule, amax2.ptr(), y.ptr(), choice2.ptr(), None,
                                work[1:2].data_ptr())
        torch.cuda.synchronize()
        assert work[1].item() == 0 and y.guards_intact() and choice2.guards_intact()
        U.assert_same("amax", amax2.numpy(np.float32), want_amax)
        U.assert_same("fakequant", y.numpy(np.uint16), wfq["fq"])
        U.assert_same("fakequant choice", choice2.numpy(), wfq["choice"])
