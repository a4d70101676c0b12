"""Quantization for Blackwell block-scaled FP4 GEMMs (nvfp4_quantize_gemm).

Parity: codes, tensor scale and choice bits equal the oracle's; the tiled scales equal the
oracle's row-major scales moved by the tiled layout (written out here from its definition:
128 x 4 tiles of 512 bytes, row r / column c at (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4),
with zero padding. Use: two operands quantized this way go through a library NVFP4 GEMM
(cuBLASLt via torch's scaled_mm, used here only to check the operand format) and must match
a float64 GEMM of their exactly decoded values.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def tiled_from_rowmajor(s_rm: np.ndarray, rows: int, bpr: int) -> np.ndarray:
    n_ct = (bpr + 3) // 4
    out = np.zeros(((rows + 127) // 128) * 128 * n_ct * 4, np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(bpr)[None, :]
    off = ((r // 128) * n_ct + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)
    out[off.ravel()] = s_rm.reshape(rows, bpr).ravel()
    return out


def run_gemm_quant(x, rows, cols, mode, rule, amax_np):
    xd = U.to_device_bf16(x)
    amax_d = torch.from_numpy(np.ascontiguousarray(amax_np, np.float32)).cuda()
    nb = rows * cols // 16
    codes = U.Guarded(rows * cols // 2)
    scales = U.Guarded(nv.gemm_scale_bytes(rows, cols), fill=0x5A)
    tscale = U.Guarded(4)
    choice = U.Guarded((nb + 7) // 8)
    nv.nvfp4_quantize_gemm(xd.data_ptr(), rows, cols, amax_d.data_ptr(), mode, rule, codes.ptr(), scales.ptr(),
                           tscale.ptr(), choice.ptr())
    torch.cuda.synchronize()
    assert all(b.guards_intact() for b in (codes, scales, tscale, choice))
    return codes.numpy(), scales.numpy(), tscale.numpy(np.float32), choice.numpy()


@pytest.mark.parametrize("rows,cols", [(1, 16), (100, 48), (129, 64), (300, 1024), (256, 4080), (1000, 512)])
@pytest.mark.parametrize("mode,rule", [(0, 2), (1, 0), (1, 1), (1, 2)], ids=["scale6", "46max", "46mae", "46mse"])
def test_tiled_scales_parity(gpu, rows, cols, mode, rule):
    x, _ = synth.make("c3", rows=rows, cols=cols)
    amax = O.amax(x, 1, rows, cols)
    want = O.quantize(x, 1, rows, cols, amax, mode, rule)
    codes, scales, tscale, choice = run_gemm_quant(x, rows, cols, mode, rule, amax)
    U.assert_same("codes", codes, want["codes"])
    U.assert_same("tscale", tscale, want["tscale"])
    U.assert_same("choice", choice, want["choice"])
    U.assert_same("tiled scales", scales, tiled_from_rowmajor(want["scales"], rows, cols // 16))


E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def decode_exact(codes: np.ndarray, scales_rm: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Exact decoded values v * s (float64), without the tensor scale."""
    lo = E2M1[codes & 0xF]
    hi = E2M1[codes >> 4]
    v = np.stack([lo, hi], axis=-1).reshape(rows, cols)
    s = O.e4m3_to_f32(scales_rm).astype(np.float64).reshape(rows, cols // 16)
    return v * np.repeat(s, 16, axis=1)


@pytest.mark.parametrize("m,n,k", [(256, 256, 2048), (128, 384, 512), (384, 128, 1024)])
def test_block_scaled_gemm_consumes_the_operands(gpu, m, n, k):
    import torch.nn.functional as F

    a, _ = synth.make("c3", rows=m, cols=k)          # activations
    b, _ = synth.make("c2", rows=n, cols=k)          # weights
    ops = []
    for x, rows in ((a, m), (b, n)):
        amax = O.amax(x, 1, rows, k)
        codes, scales, tscale, _ = run_gemm_quant(x, rows, k, 1, 2, amax)
        rm = O.quantize(x, 1, rows, k, amax, 1, 2)
        ops.append((codes, scales, float(tscale[0]), decode_exact(codes, rm["scales"], rows, k)))
    (ca, sa, ta, va), (cb, sb, tb, vb) = ops
    A = torch.from_numpy(ca).cuda().view(m, k // 2).view(torch.float4_e2m1fn_x2)
    B = torch.from_numpy(cb).cuda().view(n, k // 2).view(torch.float4_e2m1fn_x2)
    SA = torch.from_numpy(sa).cuda().view(torch.float8_e4m3fn)
    SB = torch.from_numpy(sb).cuda().view(torch.float8_e4m3fn)
    d = F.scaled_mm(A, B.t(), SA, F.ScalingType.BlockWise1x16, SB, F.ScalingType.BlockWise1x16,
                    swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                    output_dtype=torch.bfloat16)
    got = d.float().cpu().numpy().astype(np.float64) * ta * tb
    ref = (va @ vb.T) * ta * tb
    bound = (np.abs(va) @ np.abs(vb).T) * ta * tb * 2.0 ** -7 + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), (float(err.max()), float((err / bound).max()))
    # the bound is not vacuous: the result is far larger than the error
    assert np.mean(np.abs(ref)) > 0 and np.max(np.abs(got - ref)) < 0.05 * np.max(np.abs(ref))
