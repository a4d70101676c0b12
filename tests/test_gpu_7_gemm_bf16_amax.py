"""FP4 GEMM with a BF16 result and its amax fused into the epilogue (nvfp4_gemm_bf16).

What must hold, and how each is checked:
  1. y equals the BF16 round-to-nearest-even of nvfp4_gemm's FP32 output bit for bit (same
     kernel, same MMA sequence; torch's float32 -> bfloat16 conversion rounds to nearest even);
  2. y_amax equals max |y| over the BF16 values written, bit for bit, which is also what
     nvfp4_amax computes on y and what the oracle's amax computes on y's bits;
  3. the chain GEMM -> fused amax -> quantization of y for the next GEMM gives the oracle's
     codes, scales and tensor scale for y, bit for bit (the next layer's quantization needs no
     separate amax pass);
  4. y agrees with the oracle's exact product within the FP32 accumulation bound of
     tests/test_gpu_6_gemm.py plus one BF16 rounding (relative 2^-8).
Edge cases: ragged row counts and half column tiles (guard bytes after y untouched), an empty
product (amax 0), zero operands, y_amax omitted."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from tests.test_gpu_6_gemm import device_bf16, magnitude, operands, oracle_quant

pytestmark = pytest.mark.gpu

SHAPES = [(128, 256, 256), (256, 512, 512), (384, 256, 1280), (1, 128, 256), (200, 384, 512), (130, 640, 768),
          (385, 256, 256), (2048, 4096, 512)]


def run_bf16(xq, wq, m, n, k, guard=1024, with_amax=True):
    ybuf = torch.full((m * n + guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = ybuf[: m * n].view(m, n)
    y_amax = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda") if with_amax else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_gemm_bf16(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], m, n, k, y, y_amax, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.isnan(ybuf[m * n:]).all(), "write past the end of y"
    return y, y_amax


@pytest.mark.parametrize("m,n,k", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_bf16_output_and_fused_amax(gpu, m, n, k):
    x, w = operands(m, n, k, seed=2 * m + n + k)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    y32 = nv.gemm(xq, wq)
    y, y_amax = run_bf16(xq, wq, m, n, k)
    # 1. the rounded FP32 output
    assert torch.equal(y.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
    # 2. the amax of what was written, three ways
    top = y.float().abs().max().reshape(1)
    assert torch.equal(y_amax.view(torch.int32), top.view(torch.int32))
    assert torch.equal(y_amax.view(torch.int32), nv.amax(y, 1).view(torch.int32))
    ybits = y.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    assert np.float32(O.amax(ybits, 1, m, n)[0]).view(np.int32) == y_amax.view(torch.int32).item()
    # 4. against the exact product
    xc, xs, xt = oracle_quant(x, m, k, "four_over_six", "mse")
    wc, ws, wt = oracle_quant(w, n, k, "four_over_six", "mse")
    want = O.gemm_nvfp4(xc, xs, xt, wc, ws, wt, m, n, k)
    s = O.gemm_nvfp4(magnitude(xc), xs, xt, magnitude(wc), ws, wt, m, n, k)
    bound = (k / 64 + 4) * 2.0 ** -22 * s + 1e-30
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - want) <= bound + 2.0 ** -8 * (np.abs(want) + bound))


def test_chain_gemm_amax_quantize(gpu):
    """y = gemm_bf16(Xq, Wq) with its amax, then y quantized for the next GEMM with that amax
    (no amax pass over y): the oracle, given y's bits, computes the same amax and the same
    codes, scales and tensor scale."""
    m, n, k = 256, 1024, 512
    x, w = operands(m, n, k, seed=41)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    y, y_amax = nv.gemm_bf16(xq, wq)
    yq = nv.quantize_for_gemm(y, "four_over_six", "mse", amax_values=y_amax)
    torch.cuda.synchronize()
    ybits = y.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    yc, ys, yt = oracle_quant(ybits, m, n, "four_over_six", "mse")
    from tests.test_gpu_4_gemm_layout import tiled_from_rowmajor
    assert np.array_equal(yq[0].cpu().numpy().ravel(), yc)
    assert np.array_equal(yq[1].cpu().numpy(), tiled_from_rowmajor(ys, m, n // 16))
    assert yq[2].item() == yt


def test_empty_zero_and_no_amax(gpu):
    m, n, k = 128, 256, 256
    x, w = operands(m, n, k, seed=43)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    # an empty product still writes its amax: 0
    y_amax = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm_bf16(xq[0], xq[1], xq[2], wq[0], wq[1], wq[2], 0, n, k, None, y_amax)
    torch.cuda.synchronize()
    assert y_amax.item() == 0.0 and not torch.signbit(y_amax).item()
    # without an amax the values are the same
    y_a, _ = run_bf16(xq, wq, m, n, k)
    y_b, none = run_bf16(xq, wq, m, n, k, with_amax=False)
    assert none is None and torch.equal(y_a.view(torch.int16), y_b.view(torch.int16))
    # zero activations: +0 everywhere, amax +0
    zq = nv.quantize_for_gemm(torch.zeros_like(xd))
    y0, a0 = run_bf16(zq, wq, m, n, k)
    assert torch.count_nonzero(y0.view(torch.int16)) == 0 and a0.view(torch.int32).item() == 0


def test_side_stream(gpu):
    m, n, k = 256, 512, 512
    x, w = operands(m, n, k, seed=47)
    xd, wd = device_bf16(x, m, k), device_bf16(w, n, k)
    xq, wq = nv.quantize_for_gemm(xd), nv.quantize_for_gemm(wd)
    y_ref, a_ref = nv.gemm_bf16(xq, wq)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y, a = nv.gemm_bf16(xq, wq, s.cuda_stream)
    s.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)) and torch.equal(a, a_ref)
