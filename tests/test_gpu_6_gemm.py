"""Block-scaled FP4 GEMM on the tensor cores (nvfp4_gemm, nvfp4_gemm_quantize_x).

Parity, from the most exact to the least:
  1. the operands the GEMM consumes (codes, tiled scales, tensor scales of nvfp4_quantize_gemm)
     equal the oracle's quantization bit for bit;
  2. the GEMM whose prologue quantizes the BF16 activations equals the GEMM on the
     separately quantized activations bit for bit (same arithmetic, same MMA sequence);
  3. y agrees with the oracle's exact product alpha_x alpha_w sum_k (v s)_x (v s)_w within a
     bound derived from FP32 accumulation: every one of the k / 64 MMAs adds its partial sum
     to the FP32 accumulator with a relative rounding below 2^-23, and the partial sums are
     themselves formed in at least FP32, so |y - exact| <= (k / 64 + 4) 2^-22 S, where
     S = alpha_x alpha_w sum_k |(v s)_x (v s)_w| (the same product on magnitudes).
Inputs: activations shaped like the 8192 x 4096 workload (Student-t(3) times a lognormal
per-channel scale), weights N(0, 0.02) with 0.1% outliers x20."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth
from tests.test_gpu_4_gemm_layout import tiled_from_rowmajor

pytestmark = pytest.mark.gpu

MODES = {"scale6": 0, "four_over_six": 1}
RULES = {"maxerr": 0, "mae": 1, "mse": 2}


def device_bf16(bits: np.ndarray, rows: int, cols: int):
    return torch.from_numpy(bits.view(np.int16).reshape(rows, cols)).cuda().view(torch.bfloat16)


def operands(m, n, k, seed):
    x, _ = synth.make("c3", rows=m, cols=k, seed=seed)
    w, _ = synth.make("c2", rows=n, cols=k, seed=seed + 1)
    return x, w


def oracle_quant(bits, rows, cols, mode, rule):
    a = O.amax(bits, 1, rows, cols)
    q = O.quantize(bits, 1, rows, cols, a, MODES[mode], RULES[rule])
    return q["codes"], q["scales"], q["tscale"][0]


def magnitude(codes):
    return (np.asarray(codes, np.uint8) & 0x77).astype(np.uint8)   # clear both nibbles' sign bits


SHAPES = [(128, 256, 256), (256, 512, 512), (384, 256, 1280), (128, 768, 4096), (512, 256, 2304)]


@pytest.mark.parametrize("m,n,k", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_gemm_parity(gpu, m, n, k):
    x, w = operands(m, n, k, seed=m + n + k)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq = nv.quantize_for_gemm(xd, "four_over_six", "mse")
    wq = nv.quantize_for_gemm(wd, "four_over_six", "mse")
    torch.cuda.synchronize()
    # 1. operands against the oracle
    xc, xs, xt = oracle_quant(x, m, k, "four_over_six", "mse")
    wc, ws, wt = oracle_quant(w, n, k, "four_over_six", "mse")
    assert np.array_equal(xq[0].cpu().numpy().ravel(), xc)
    assert np.array_equal(wq[0].cpu().numpy().ravel(), wc)
    assert np.array_equal(xq[1].cpu().numpy(), tiled_from_rowmajor(xs, m, k // 16))
    assert np.array_equal(wq[1].cpu().numpy(), tiled_from_rowmajor(ws, n, k // 16))
    assert xq[2].item() == xt and wq[2].item() == wt
    # 2. prologue-quantized activations give the same bits
    y = nv.gemm(xq, wq)
    y2 = nv.gemm_quantize_x(xd, wq, "four_over_six", "mse")
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    # 3. against the exact product
    want = O.gemm_nvfp4(xc, xs, xt, wc, ws, wt, m, n, k)
    s = O.gemm_nvfp4(magnitude(xc), xs, xt, magnitude(wc), ws, wt, m, n, k)
    got = y.cpu().numpy().astype(np.float64)
    bound = (k / 64 + 4) * 2.0 ** -22 * s + 1e-30
    err = np.abs(got - want)
    assert np.all(err <= bound), (float(np.max(err / bound)), float(np.max(err)))
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("mode,rule", [("four_over_six", "maxerr"), ("four_over_six", "mae"), ("scale6", "mse")])
def test_prologue_quantization_matches_separate_quantization(gpu, mode, rule):
    m, n, k = 256, 256, 768
    x, w = operands(m, n, k, seed=11)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    wq = nv.quantize_for_gemm(wd, "four_over_six", "mse")
    xq = nv.quantize_for_gemm(xd, mode, rule)
    y = nv.gemm(xq, wq)
    y2 = nv.gemm_quantize_x(xd, wq, mode, rule)
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    xc, xs, xt = oracle_quant(x, m, k, mode, rule)
    assert np.array_equal(xq[0].cpu().numpy().ravel(), xc)


def test_zero_and_one_hot_operands(gpu):
    """W with one 1.0 per row (code 2 at k = n, scale 1.0, alpha 1): y reproduces the exact
    quantized activations; an all-zero X gives exact zeros."""
    m, n, k = 128, 256, 256
    x, _ = operands(m, n, k, seed=3)
    xd = device_bf16(x, m, k)
    xq = nv.quantize_for_gemm(xd, "four_over_six", "mse")
    w4 = np.zeros((n, k), np.uint8)
    w4[np.arange(n), np.arange(n)] = 2
    wc = (w4[:, 0::2] | (w4[:, 1::2] << 4)).astype(np.uint8)
    ws = np.full((n, k // 16), 0x38, np.uint8)
    wq = (torch.from_numpy(wc).cuda(), torch.from_numpy(tiled_from_rowmajor(ws, n, k // 16)).cuda(),
          torch.ones(1, dtype=torch.float32, device="cuda"), None)
    y = nv.gemm(xq, wq).cpu().numpy().astype(np.float64)
    xc, xs, xt = oracle_quant(x, m, k, "four_over_six", "mse")
    want = O.gemm_nvfp4(xc, xs, xt, wc, ws, 1.0, m, n, k)
    assert np.array_equal(y, want.astype(np.float32).astype(np.float64))
    zq = nv.quantize_for_gemm(torch.zeros_like(xd), "four_over_six", "mse")
    assert torch.count_nonzero(nv.gemm(zq, wq)) == 0


def test_side_stream_and_status_word(gpu):
    m, n, k = 128, 256, 512
    x, w = operands(m, n, k, seed=5)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq = nv.quantize_for_gemm(xd)
    wq = nv.quantize_for_gemm(wd)
    torch.cuda.synchronize()
    y_ref = nv.gemm(xq, wq)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = torch.full((m, n), float("nan"), device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_gemm(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], m, n, k, y, status, s.cuda_stream)
    s.synchronize()
    assert status.item() == 0
    assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32))


def test_more_tiles_than_ctas(gpu):
    """2048 x 4096 x 512: 256 output tiles on one CTA per SM, so CTAs run one or two tiles and
    hand the accumulator over between them; every output against the exact product."""
    m, n, k = 2048, 4096, 512
    x, w = operands(m, n, k, seed=17)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    y = nv.gemm(xq, wq)
    y2 = nv.gemm_quantize_x(xd, wq)
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    xc, xs, xt = oracle_quant(x, m, k, "four_over_six", "mse")
    wc, ws, wt = oracle_quant(w, n, k, "four_over_six", "mse")
    want = O.gemm_nvfp4(xc, xs, xt, wc, ws, wt, m, n, k)
    s = O.gemm_nvfp4(magnitude(xc), xs, xt, magnitude(wc), ws, wt, m, n, k)
    err = np.abs(y.cpu().numpy().astype(np.float64) - want)
    assert np.all(err <= (k / 64 + 4) * 2.0 ** -22 * s + 1e-30)


@pytest.mark.slow
def test_bench_shape_sampled(gpu):
    """The bench's GEMM shape, 8192 x 4096 x 4096 (2048 tiles, about 14 per CTA): 512 sampled
    outputs (whole rows' worth of tiles included) against the exact product of the oracle's
    operands."""
    m, n, k = 8192, 4096, 4096
    rng = np.random.default_rng(8)
    x, w = operands(m, n, k, seed=23)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    y = nv.gemm(xq, wq).cpu().numpy().astype(np.float64)
    xc, xs, xt = oracle_quant(x, m, k, "four_over_six", "mse")
    wc, ws, wt = oracle_quant(w, n, k, "four_over_six", "mse")
    assert np.array_equal(xq[0].cpu().numpy().ravel(), xc) and np.array_equal(wq[0].cpu().numpy().ravel(), wc)
    rows = np.concatenate([rng.integers(0, m, 14), [0, m - 1]])
    cols = np.concatenate([rng.integers(0, n, 30), [0, n - 1]])
    xr, xsr = xc.reshape(m, k // 2)[rows], xs.reshape(m, k // 16)[rows]
    wr, wsr = wc.reshape(n, k // 2)[cols], ws.reshape(n, k // 16)[cols]
    want = O.gemm_nvfp4(xr, xsr, xt, wr, wsr, wt, len(rows), len(cols), k)
    s = O.gemm_nvfp4(magnitude(xr), xsr, xt, magnitude(wr), wsr, wt, len(rows), len(cols), k)
    got = y[np.ix_(rows, cols)]
    assert np.all(np.abs(got - want) <= (k / 64 + 4) * 2.0 ** -22 * s + 1e-30)
    assert np.all(np.isfinite(y))


RAGGED = [(1, 128, 256), (200, 384, 512), (130, 640, 768), (385, 256, 256)]


@pytest.mark.parametrize("m,n,k", RAGGED, ids=[f"{m}x{n}x{k}" for m, n, k in RAGGED])
def test_ragged_rows_and_half_column_tiles(gpu, m, n, k):
    """Row counts that are not multiples of 128 (the last row tile is part zeros and only rows
    below m are stored) and column counts that end in half a 256-column tile; rows of y past m
    and the guard bytes after y stay untouched."""
    x, w = operands(m, n, k, seed=m + 3 * n + k)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    ybuf = torch.full((m * n + 1024,), float("nan"), dtype=torch.float32, device="cuda")
    y = ybuf[: m * n].view(m, n)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_gemm(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], m, n, k, y, status)
    y2 = nv.gemm_quantize_x(xd, wq)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.isnan(ybuf[m * n:]).all(), "write past the end of y"
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    xc, xs, xt = oracle_quant(x, m, k, "four_over_six", "mse")
    wc, ws, wt = oracle_quant(w, n, k, "four_over_six", "mse")
    want = O.gemm_nvfp4(xc, xs, xt, wc, ws, wt, m, n, k)
    s = O.gemm_nvfp4(magnitude(xc), xs, xt, magnitude(wc), ws, wt, m, n, k)
    got = y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - want) <= (k / 64 + 4) * 2.0 ** -22 * s + 1e-30)
