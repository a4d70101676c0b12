"""Python binding of libnvfp4.so (include/nvfp4.h): BF16 -> NVFP4 quantization on B200.

The functions named ``nvfp4_*`` mirror the C ABI one to one and only marshal arguments:
torch CUDA tensors in, device pointers and the current CUDA stream out. Every step of the
computation runs in the library's sm_100a kernels; there is no CPU path. If the shared
library is missing, ``load()`` raises.

The convenience wrappers ``quantize``, ``fakequant`` and ``dequantize`` allocate outputs
with torch and call the same entry points.

Sources: "Four Over Six: More Accurate NVFP4 Quantization with Adaptive Block Scaling"
(gist.science explainer), technical summary (Problem definition; Method; Implementation
details); "Quantization-Aware Distillation for NVFP4 Inference Accuracy Recovery" §3.3
(blocks of 16).
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple

__all__ = [
    "load", "library_path", "Nvfp4Error", "Nvfp4TimeoutError",
    "SCALE6", "FOUR_OVER_SIX", "RULE_MAXERR", "RULE_MAE", "RULE_MSE",
    "nvfp4_amax", "nvfp4_quantize", "nvfp4_dequantize", "nvfp4_fakequant", "nvfp4_amax_quantize",
    "nvfp4_amax_fakequant", "QUANT_TIMEOUT", "nvfp4_quantize_gemm", "nvfp4_qad_kl",
    "nvfp4_gemm", "nvfp4_gemm_bf16", "nvfp4_gemm_quantize_x", "GEMM_TIMEOUT", "nvfp4_status_string", "nvfp4_version",
    "Quantized", "amax", "quantize", "fakequant", "dequantize", "amax_quantize", "amax_fakequant", "quantize_for_gemm", "gemm_scale_bytes",
    "qad_kl", "fakequant_ste", "gemm", "gemm_bf16", "gemm_quantize_x",
]

GEMM_TIMEOUT = 1   # bit of a GEMM's status word: a bounded wait for the tensor core timed out
QUANT_TIMEOUT = 2  # bit of a quantizer's status word: the grid-wide wait of a one-launch amax timed out

SCALE6, FOUR_OVER_SIX = 0, 1
RULE_MAXERR, RULE_MAE, RULE_MSE = 0, 1, 2
_MODES = {"scale6": SCALE6, "four_over_six": FOUR_OVER_SIX, "4/6": FOUR_OVER_SIX}
_RULES = {"maxerr": RULE_MAXERR, "max": RULE_MAXERR, "mae": RULE_MAE, "mse": RULE_MSE}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "lib", "libnvfp4.so")
_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, func: str):
        self.status = status
        super().__init__(f"{func}: {nvfp4_status_string(status)} (status {status})")


class Nvfp4TimeoutError(RuntimeError):
    """A kernel's bounded wait timed out, as its status word reports (its outputs are partial)."""


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libnvfp4.so (built by ``python -m nvfp4_block_scaled_13_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libnvfp4.so not built: {_LIB_PATH} is missing "
                              "(run python -m nvfp4_block_scaled_13_b200.build)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.nvfp4_amax.argtypes = [vp, i64, i64, i64, vp, vp]
        L.nvfp4_quantize.argtypes = [vp, i64, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp]
        L.nvfp4_dequantize.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp]
        L.nvfp4_fakequant.argtypes = [vp, i64, i64, i64, vp, i32, i32, vp, vp, vp]
        L.nvfp4_quantize_gemm.argtypes = [vp, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp]
        L.nvfp4_qad_kl.argtypes = [vp, vp, i64, i64, ctypes.c_float, ctypes.c_float, vp, vp, vp]
        L.nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp]
        L.nvfp4_gemm_bf16.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp]
        L.nvfp4_amax_quantize.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.nvfp4_amax_fakequant.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
        L.nvfp4_gemm_quantize_x.argtypes = [vp, vp, i32, i32, vp, vp, vp, i64, i64, i64, vp, vp, vp]
        for f in (L.nvfp4_amax, L.nvfp4_quantize, L.nvfp4_dequantize, L.nvfp4_fakequant, L.nvfp4_quantize_gemm,
                  L.nvfp4_qad_kl, L.nvfp4_gemm, L.nvfp4_gemm_bf16, L.nvfp4_gemm_quantize_x, L.nvfp4_amax_quantize,
                  L.nvfp4_amax_fakequant):
            f.restype = i32
        L.nvfp4_status_string.argtypes, L.nvfp4_status_string.restype = [i32], ctypes.c_char_p
        L.nvfp4_version.argtypes, L.nvfp4_version.restype = [], i32
        _lib = L
    return _lib


# ---- marshalling helpers -------------------------------------------------------------------

def _ptr(t):
    """Device pointer of a CUDA tensor (None -> NULL). Raw integers pass through."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("nvfp4: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("nvfp4: tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, func: str):
    if status != 0:
        raise Nvfp4Error(status, func)


def _mode(m):
    return _MODES[m] if isinstance(m, str) else int(m)


def _rule(r):
    return _RULES[r] if isinstance(r, str) else int(r)


# ---- the C ABI, one to one -------------------------------------------------------------------

def nvfp4_amax(x, groups, rows, cols, amax, stream=None):
    _check(load().nvfp4_amax(_ptr(x), groups, rows, cols, _ptr(amax), _stream(stream)), "nvfp4_amax")


def nvfp4_quantize(x, groups, rows, cols, amax, mode, rule, codes, scales, tscale, choice=None, stream=None):
    _check(load().nvfp4_quantize(_ptr(x), groups, rows, cols, _ptr(amax), _mode(mode), _rule(rule),
                                 _ptr(codes), _ptr(scales), _ptr(tscale), _ptr(choice), _stream(stream)),
           "nvfp4_quantize")


def nvfp4_dequantize(codes, scales, tscale, groups, rows, cols, y, stream=None):
    _check(load().nvfp4_dequantize(_ptr(codes), _ptr(scales), _ptr(tscale), groups, rows, cols, _ptr(y),
                                   _stream(stream)), "nvfp4_dequantize")


def nvfp4_fakequant(x, groups, rows, cols, amax, mode, rule, y, choice=None, stream=None):
    _check(load().nvfp4_fakequant(_ptr(x), groups, rows, cols, _ptr(amax), _mode(mode), _rule(rule),
                                  _ptr(y), _ptr(choice), _stream(stream)), "nvfp4_fakequant")


def nvfp4_amax_quantize(x, groups, rows, cols, mode, rule, amax, codes, scales, tscale, choice=None, workspace=None,
                        status=None, stream=None):
    _check(load().nvfp4_amax_quantize(_ptr(x), groups, rows, cols, _mode(mode), _rule(rule), _ptr(amax), _ptr(codes),
                                      _ptr(scales), _ptr(tscale), _ptr(choice), _ptr(workspace), _ptr(status),
                                      _stream(stream)), "nvfp4_amax_quantize")


def nvfp4_amax_fakequant(x, groups, rows, cols, mode, rule, amax, y, choice=None, workspace=None, status=None,
                         stream=None):
    _check(load().nvfp4_amax_fakequant(_ptr(x), groups, rows, cols, _mode(mode), _rule(rule), _ptr(amax), _ptr(y),
                                       _ptr(choice), _ptr(workspace), _ptr(status), _stream(stream)),
           "nvfp4_amax_fakequant")


def nvfp4_gemm(x_codes, x_scales, x_tscale, w_codes, w_scales, w_tscale, m, n, k, y, status=None, stream=None):
    _check(load().nvfp4_gemm(_ptr(x_codes), _ptr(x_scales), _ptr(x_tscale), _ptr(w_codes), _ptr(w_scales),
                             _ptr(w_tscale), m, n, k, _ptr(y), _ptr(status), _stream(stream)), "nvfp4_gemm")


def nvfp4_gemm_bf16(x_codes, x_scales, x_tscale, w_codes, w_scales, w_tscale, m, n, k, y, y_amax=None,
                    status=None, stream=None):
    _check(load().nvfp4_gemm_bf16(_ptr(x_codes), _ptr(x_scales), _ptr(x_tscale), _ptr(w_codes), _ptr(w_scales),
                                  _ptr(w_tscale), m, n, k, _ptr(y), _ptr(y_amax), _ptr(status), _stream(stream)),
           "nvfp4_gemm_bf16")


def nvfp4_gemm_quantize_x(x, x_amax, mode, rule, w_codes, w_scales, w_tscale, m, n, k, y, status=None,
                          stream=None):
    _check(load().nvfp4_gemm_quantize_x(_ptr(x), _ptr(x_amax), _mode(mode), _rule(rule), _ptr(w_codes),
                                        _ptr(w_scales), _ptr(w_tscale), m, n, k, _ptr(y), _ptr(status),
                                        _stream(stream)), "nvfp4_gemm_quantize_x")


def nvfp4_quantize_gemm(x, rows, cols, amax, mode, rule, codes, scales, tscale, choice=None, stream=None):
    _check(load().nvfp4_quantize_gemm(_ptr(x), rows, cols, _ptr(amax), _mode(mode), _rule(rule), _ptr(codes),
                                      _ptr(scales), _ptr(tscale), _ptr(choice), _stream(stream)),
           "nvfp4_quantize_gemm")


def nvfp4_qad_kl(teacher, student, rows, vocab, tau, grad_scale, kl, grad=None, stream=None):
    _check(load().nvfp4_qad_kl(_ptr(teacher), _ptr(student), rows, vocab, float(tau), float(grad_scale), _ptr(kl),
                               _ptr(grad), _stream(stream)), "nvfp4_qad_kl")


def nvfp4_status_string(status: int) -> str:
    return load().nvfp4_status_string(int(status)).decode()


def nvfp4_version() -> int:
    return load().nvfp4_version()


# ---- convenience wrappers (torch allocates, the library computes) -----------------------------

class Quantized(NamedTuple):
    codes: "object"      # uint8 [groups*rows*cols/2]
    scales: "object"     # uint8 [groups*rows*cols/16] (E4M3 bits)
    tscale: "object"     # float32 [groups]
    choice: "object"     # uint8 [ceil(blocks/8)] or None
    shape: tuple         # (groups, rows, cols)


def _shape3(x, groups):
    if x.dtype.itemsize != 2:
        raise ValueError("nvfp4: x must be BF16 (or its uint16/int16 bits)")
    cols = x.shape[-1] if x.dim() > 0 else 0
    n = x.numel()
    if groups < 1 or (cols and n % (groups * cols)):
        raise ValueError("nvfp4: numel must be a multiple of groups * cols")
    rows = n // (groups * cols) if cols else 0
    return groups, rows, cols


def amax(x, groups: int = 1, stream=None):
    import torch

    g, r, c = _shape3(x, groups)
    out = torch.empty(g, dtype=torch.float32, device=x.device)
    nvfp4_amax(x, g, r, c, out, stream)
    return out


def quantize(x, mode="four_over_six", rule="mse", groups: int = 1, amax_values=None, with_choice=True,
             stream=None) -> Quantized:
    import torch

    g, r, c = _shape3(x, groups)
    if amax_values is None:
        amax_values = amax(x, groups, stream)
    n = g * r * c
    nb = n // 16
    dev = x.device
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(nb, dtype=torch.uint8, device=dev)
    tscale = torch.empty(g, dtype=torch.float32, device=dev)
    choice = torch.empty(max(1, (nb + 7) // 8), dtype=torch.uint8, device=dev) if with_choice else None
    nvfp4_quantize(x, g, r, c, amax_values, mode, rule, codes, scales, tscale, choice, stream)
    return Quantized(codes, scales, tscale, choice, (g, r, c))


def dequantize(q: Quantized, out=None, stream=None):
    import torch

    g, r, c = q.shape
    if out is None:
        out = torch.empty((g * r, c) if c else (0,), dtype=torch.bfloat16, device=q.codes.device)
    nvfp4_dequantize(q.codes, q.scales, q.tscale, g, r, c, out, stream)
    return out


def fakequant(x, mode="four_over_six", rule="mse", groups: int = 1, amax_values=None, out=None, choice=None,
              stream=None):
    import torch

    g, r, c = _shape3(x, groups)
    if amax_values is None:
        amax_values = amax(x, groups, stream)
    if out is None:
        out = torch.empty_like(x, dtype=torch.bfloat16)
    nvfp4_fakequant(x, g, r, c, amax_values, mode, rule, out, choice, stream)
    return out


def amax_quantize(x, mode="four_over_six", rule="mse", groups: int = 1, with_choice=True, stream=None):
    """(Quantized, amax): the tensor amax and the quantization in one launch. Raises if the
    launch's grid-wide wait timed out."""
    import torch

    g, r, c = _shape3(x, groups)
    n = g * r * c
    nb = n // 16
    dev = x.device
    amax_out = torch.empty(g, dtype=torch.float32, device=dev)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(nb, dtype=torch.uint8, device=dev)
    tscale = torch.empty(g, dtype=torch.float32, device=dev)
    choice = torch.empty(max(1, (nb + 7) // 8), dtype=torch.uint8, device=dev) if with_choice else None
    work = torch.empty(2, dtype=torch.int32, device=dev)   # [0] barrier counter, [1] status
    work[1:].zero_()
    nvfp4_amax_quantize(x, g, r, c, mode, rule, amax_out, codes, scales, tscale, choice, work[0:1], work[1:2], stream)
    if int(work[1].item()) & QUANT_TIMEOUT:
        raise Nvfp4TimeoutError("nvfp4_amax_quantize: the grid-wide wait timed out")
    return Quantized(codes, scales, tscale, choice, (g, r, c)), amax_out


def amax_fakequant(x, mode="four_over_six", rule="mse", groups: int = 1, out=None, choice=None, stream=None):
    """(fake-quantized BF16, amax) in one launch."""
    import torch

    g, r, c = _shape3(x, groups)
    amax_out = torch.empty(g, dtype=torch.float32, device=x.device)
    if out is None:
        out = torch.empty_like(x, dtype=torch.bfloat16)
    work = torch.zeros(2, dtype=torch.int32, device=x.device)
    nvfp4_amax_fakequant(x, g, r, c, mode, rule, amax_out, out, choice, work[0:1], work[1:2], stream)
    if int(work[1].item()) & QUANT_TIMEOUT:
        raise Nvfp4TimeoutError("nvfp4_amax_fakequant: the grid-wide wait timed out")
    return out, amax_out


def gemm_scale_bytes(rows: int, cols: int) -> int:
    """Size of the tiled scale buffer of nvfp4_quantize_gemm: roundup(rows, 128) * roundup(cols / 16, 4)."""
    return (rows + 127) // 128 * 128 * ((cols // 16 + 3) // 4 * 4)


def quantize_for_gemm(x, mode="four_over_six", rule="mse", amax_values=None, with_choice=False, stream=None):
    """Quantize a 2-D BF16 matrix as a K-major block-scaled FP4 GEMM operand. Returns
    (codes [rows, cols/2] uint8, tiled scales uint8, tscale [1] float32, choice or None)."""
    import torch

    if x.dim() != 2:
        raise ValueError("quantize_for_gemm: x must be 2-D [rows, cols]")
    rows, cols = x.shape
    if amax_values is None:
        amax_values = amax(x, 1, stream)
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(gemm_scale_bytes(rows, cols), dtype=torch.uint8, device=dev)
    tscale = torch.empty(1, dtype=torch.float32, device=dev)
    nb = rows * cols // 16
    choice = torch.empty(max(1, (nb + 7) // 8), dtype=torch.uint8, device=dev) if with_choice else None
    nvfp4_quantize_gemm(x, rows, cols, amax_values, mode, rule, codes, scales, tscale, choice, stream)
    return codes, scales, tscale, choice


def gemm(xq, wq, stream=None):
    """y = Xq Wq^T (FP32) of two operands returned by quantize_for_gemm, on the FP4 tensor
    cores. Raises if the kernel reports a timed-out wait."""
    import torch

    (xc, xs, xt, _), (wc, ws, wt, _) = xq, wq
    m, n, k = xc.shape[0], wc.shape[0], 2 * xc.shape[1]
    y = torch.empty((m, n), dtype=torch.float32, device=xc.device)
    status = torch.zeros(1, dtype=torch.int32, device=xc.device)
    nvfp4_gemm(xc, xs, xt, wc, ws, wt, m, n, k, y, status, stream)
    if int(status.item()) & GEMM_TIMEOUT:
        raise Nvfp4TimeoutError("nvfp4_gemm: a wait for the tensor core timed out")
    return y


def gemm_bf16(xq, wq, stream=None):
    """(y, y_amax): y = Xq Wq^T rounded to BF16 and its absolute maximum [1] (float32), found in
    the GEMM's epilogue, ready to be the amax of y's own quantization."""
    import torch

    (xc, xs, xt, _), (wc, ws, wt, _) = xq, wq
    m, n, k = xc.shape[0], wc.shape[0], 2 * xc.shape[1]
    y = torch.empty((m, n), dtype=torch.bfloat16, device=xc.device)
    y_amax = torch.empty(1, dtype=torch.float32, device=xc.device)
    status = torch.zeros(1, dtype=torch.int32, device=xc.device)
    nvfp4_gemm_bf16(xc, xs, xt, wc, ws, wt, m, n, k, y, y_amax, status, stream)
    if int(status.item()) & GEMM_TIMEOUT:
        raise Nvfp4TimeoutError("nvfp4_gemm_bf16: a wait for the tensor core timed out")
    return y, y_amax


def gemm_quantize_x(x, wq, mode="four_over_six", rule="mse", amax_values=None, stream=None):
    """y = Q(x) Wq^T (FP32), x [m, k] BF16 quantized inside the GEMM's prologue."""
    import torch

    wc, ws, wt, _ = wq
    m, k = x.shape
    n = wc.shape[0]
    if amax_values is None:
        amax_values = amax(x, 1, stream)
    y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    nvfp4_gemm_quantize_x(x, amax_values, mode, rule, wc, ws, wt, m, n, k, y, status, stream)
    if int(status.item()) & GEMM_TIMEOUT:
        raise Nvfp4TimeoutError("nvfp4_gemm_quantize_x: a wait for the tensor core timed out")
    return y


def qad_kl(teacher, student, tau: float = 1.0, grad_scale=None, with_grad: bool = True, stream=None):
    """Per-row KL(softmax(teacher / tau) || softmax(student / tau)) of [rows, vocab] BF16 logits,
    and (optionally) grad_scale * (q - p), the gradient of the mean loss when grad_scale is
    1 / (tau * rows) (the default)."""
    import torch

    vocab = teacher.shape[-1]
    rows = teacher.numel() // vocab
    if student.shape != teacher.shape:
        raise ValueError("qad_kl: teacher and student shapes differ")
    if grad_scale is None:
        grad_scale = 1.0 / (tau * max(rows, 1))
    kl = torch.empty(rows, dtype=torch.float32, device=teacher.device)
    grad = torch.empty_like(student, dtype=torch.bfloat16) if with_grad else None
    nvfp4_qad_kl(teacher, student, rows, vocab, tau, grad_scale, kl, grad, stream)
    return kl, grad


def fakequant_ste(x, mode="four_over_six", rule="mse", groups: int = 1, amax_values=None):
    """Simulated NVFP4 quantization for a QAD student: the forward is nvfp4_fakequant, the
    backward passes the gradient through unchanged (straight-through)."""
    import torch

    class _FakeQuantSTE(torch.autograd.Function):
        @staticmethod
        def forward(ctx, inp):
            return fakequant(inp, mode, rule, groups, amax_values)

        @staticmethod
        def backward(ctx, g):
            return g

    return _FakeQuantSTE.apply(x)
