"""ctypes front end of the C oracle (oracle/nvfp4_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``. The product package never
imports it, and it never imports the product package.

All arrays are numpy arrays on the host. BF16 tensors travel as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

SCALE6, FOUR_OVER_SIX = 0, 1
RULE_MAXERR, RULE_MAE, RULE_MSE = 0, 1, 2

_lib = None


class Candidate(ctypes.Structure):
    _fields_ = [
        ("beta", ctypes.c_float),
        ("t", ctypes.c_float),
        ("s", ctypes.c_uint8),
        ("d", ctypes.c_float),
        ("r", ctypes.c_float),
        ("code", ctypes.c_uint8 * 16),
        ("q", ctypes.c_float * 16),
        ("e", ctypes.c_float * 16),
        ("err", ctypes.c_float),
    ]


def lib():
    global _lib
    if _lib is None:
        # NVO_ORACLE_LIB lets the mutation test load a deliberately broken copy of the oracle
        path = os.environ.get("NVO_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        f32, u8, u16, i64, i32, vp = (ctypes.c_float, ctypes.c_uint8, ctypes.c_uint16,
                                      ctypes.c_int64, ctypes.c_int, ctypes.c_void_p)
        L.nvo_bf16_to_f32.argtypes, L.nvo_bf16_to_f32.restype = [u16], f32
        L.nvo_f32_to_bf16_rne.argtypes, L.nvo_f32_to_bf16_rne.restype = [f32], u16
        L.nvo_f32_to_e4m3_satfinite.argtypes, L.nvo_f32_to_e4m3_satfinite.restype = [f32], u8
        L.nvo_e4m3_to_f32.argtypes, L.nvo_e4m3_to_f32.restype = [u8], f32
        L.nvo_f32_to_e2m1_satfinite.argtypes, L.nvo_f32_to_e2m1_satfinite.restype = [f32], u8
        L.nvo_e2m1_to_f32.argtypes, L.nvo_e2m1_to_f32.restype = [u8], f32
        for name in ("nvo_f32_to_e2m1_array", "nvo_f32_to_e4m3_array", "nvo_f32_to_bf16_array"):
            getattr(L, name).argtypes, getattr(L, name).restype = [vp, vp, i64], None
        L.nvo_qad_kl.argtypes = [vp, vp, i64, i64, ctypes.c_double, ctypes.c_double, vp, vp]
        L.nvo_qad_kl.restype = None
        L.nvo_block_candidate.argtypes = [vp, f32, f32, i32, ctypes.POINTER(Candidate)]
        L.nvo_block_candidate.restype = None
        L.nvo_amax.argtypes, L.nvo_amax.restype = [vp, i64, i64, i64, vp], None
        L.nvo_tensor_scale.argtypes, L.nvo_tensor_scale.restype = [f32, i32], f32
        L.nvo_quantize.argtypes = [vp, i64, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp]
        L.nvo_quantize.restype = None
        L.nvo_quantize_ex.argtypes = [vp, i64, i64, i64, vp, f32, i32, i32, vp, vp, vp, vp, vp]
        L.nvo_quantize_ex.restype = None
        L.nvo_dequantize.argtypes = [vp, vp, vp, i64, i64, i64, vp]
        L.nvo_dequantize.restype = None
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check_x(x, groups, rows, cols):
    assert x.dtype == np.uint16 and x.flags.c_contiguous
    assert x.size == groups * rows * cols and cols % 16 == 0


# ---- scalar conversions (vectorised over numpy arrays with plain loops) ------------------

def f32_to_e2m1(y) -> np.ndarray:
    y = np.asarray(y, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.nvo_f32_to_e2m1_satfinite(float(v)) for v in y], dtype=np.uint8)


def e2m1_to_f32(c) -> np.ndarray:
    L = lib()
    return np.array([L.nvo_e2m1_to_f32(int(v)) for v in np.asarray(c).ravel()], dtype=np.float32)


def f32_to_e4m3(t) -> np.ndarray:
    t = np.asarray(t, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.nvo_f32_to_e4m3_satfinite(float(v)) for v in t], dtype=np.uint8)


def e4m3_to_f32(s) -> np.ndarray:
    L = lib()
    return np.array([L.nvo_e4m3_to_f32(int(v)) for v in np.asarray(s).ravel()], dtype=np.float32)


def f32_to_bf16(f) -> np.ndarray:
    f = np.asarray(f, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.nvo_f32_to_bf16_rne(float(v)) for v in f], dtype=np.uint16)


def f32_to_e2m1_array(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.size, np.uint8)
    lib().nvo_f32_to_e2m1_array(_ptr(a), _ptr(out), a.size)
    return out


def f32_to_e4m3_array(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.size, np.uint8)
    lib().nvo_f32_to_e4m3_array(_ptr(a), _ptr(out), a.size)
    return out


def f32_to_bf16_array(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.size, np.uint16)
    lib().nvo_f32_to_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


def block_candidate(x16, alpha: float, K: float, rule: int) -> Candidate:
    xb = np.ascontiguousarray(np.asarray(x16, dtype=np.float32).ravel())
    assert xb.size == 16
    c = Candidate()
    lib().nvo_block_candidate(_ptr(xb), float(alpha), float(K), int(rule), ctypes.byref(c))
    return c


# ---- tensors ------------------------------------------------------------------------------

def amax(x: np.ndarray, groups: int, rows: int, cols: int) -> np.ndarray:
    _check_x(x, groups, rows, cols)
    out = np.zeros(groups, dtype=np.float32)
    lib().nvo_amax(_ptr(x), groups, rows, cols, _ptr(out))
    return out


def tensor_scale(amax_value: float, mode: int) -> np.float32:
    return np.float32(lib().nvo_tensor_scale(float(amax_value), int(mode)))


def _alloc_outputs(groups, rows, cols, fakequant):
    n = groups * rows * cols
    nb = n // 16
    if fakequant:
        return dict(fq=np.zeros(n, np.uint16), choice=np.zeros((nb + 7) // 8, np.uint8))
    return dict(codes=np.zeros(n // 2, np.uint8), scales=np.zeros(nb, np.uint8),
                tscale=np.zeros(groups, np.float32), choice=np.zeros((nb + 7) // 8, np.uint8))


def quantize(x, groups, rows, cols, amax_arr, mode, rule):
    """Returns dict(codes, scales, tscale, choice)."""
    _check_x(x, groups, rows, cols)
    a = np.ascontiguousarray(amax_arr, dtype=np.float32)
    o = _alloc_outputs(groups, rows, cols, False)
    lib().nvo_quantize(_ptr(x), groups, rows, cols, _ptr(a), mode, rule,
                       _ptr(o["codes"]), _ptr(o["scales"]), _ptr(o["tscale"]), _ptr(o["choice"]), None)
    return o


def fakequant(x, groups, rows, cols, amax_arr, mode, rule):
    """Returns dict(fq, choice)."""
    _check_x(x, groups, rows, cols)
    a = np.ascontiguousarray(amax_arr, dtype=np.float32)
    o = _alloc_outputs(groups, rows, cols, True)
    lib().nvo_quantize(_ptr(x), groups, rows, cols, _ptr(a), mode, rule,
                       None, None, None, _ptr(o["choice"]), _ptr(o["fq"]))
    return o


def quantize_ex(x, groups, rows, cols, amax_arr, fp8_max, cand_mask, rule, with_fq=False):
    _check_x(x, groups, rows, cols)
    a = np.ascontiguousarray(amax_arr, dtype=np.float32)
    o = _alloc_outputs(groups, rows, cols, False)
    fq = np.zeros(groups * rows * cols, np.uint16) if with_fq else None
    lib().nvo_quantize_ex(_ptr(x), groups, rows, cols, _ptr(a), float(fp8_max), int(cand_mask), rule,
                          _ptr(o["codes"]), _ptr(o["scales"]), _ptr(o["tscale"]), _ptr(o["choice"]), _ptr(fq))
    if with_fq:
        o["fq"] = fq
    return o


def dequantize(codes, scales, tscale, groups, rows, cols):
    y = np.zeros(groups * rows * cols, np.uint16)
    lib().nvo_dequantize(_ptr(np.ascontiguousarray(codes)), _ptr(np.ascontiguousarray(scales)),
                         _ptr(np.ascontiguousarray(tscale, dtype=np.float32)), groups, rows, cols, _ptr(y))
    return y


def library_path() -> str:
    return _build.LIB if os.path.exists(_build.LIB) else _build.build()


def qad_kl(teacher: np.ndarray, student: np.ndarray, rows: int, vocab: int, tau: float = 1.0,
           grad_scale: float = 1.0, with_grad: bool = True):
    """Per-row KL(softmax(teacher/tau) || softmax(student/tau)) and grad_scale * (q - p), binary64."""
    t = np.ascontiguousarray(teacher, dtype=np.uint16)
    s = np.ascontiguousarray(student, dtype=np.uint16)
    assert t.size == rows * vocab and s.size == rows * vocab
    kl = np.zeros(rows, np.float64)
    g = np.zeros(rows * vocab, np.float64) if with_grad else None
    lib().nvo_qad_kl(_ptr(t), _ptr(s), rows, vocab, float(tau), float(grad_scale), _ptr(kl), _ptr(g))
    return kl, g


def unpack_e2m1(codes: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Packed E2M1 codes [rows, cols/2] bytes (element 2j in the low nibble, 2j + 1 in the
    high nibble) -> the 4-bit codes [rows, cols] as uint8."""
    c = np.ascontiguousarray(codes, dtype=np.uint8).reshape(rows, cols // 2)
    out = np.empty((rows, cols), np.uint8)
    out[:, 0::2] = c & 0x0F
    out[:, 1::2] = c >> 4
    return out


def gemm_nvfp4(a_codes, a_scales, a_alpha, b_codes, b_scales, b_alpha, m: int, n: int, k: int) -> np.ndarray:
    """Y[m, n] = a_alpha * b_alpha * sum_k A[m, k] * B[n, k] in binary64, the product that a
    block-scaled FP4 tensor-core GEMM forms from two NVFP4 operands ("Four Over Six",
    Implementation details: NVFP4 operands on Blackwell's FP4 tensor cores; Problem definition:
    a stored value is v(code) * E4M3 block scale * FP32 tensor scale). A[m, k] =
    v(code) * f32(scale of block k / 16), exact in binary64; codes are [rows, k/2] bytes with
    element 2j in the low nibble, scales row-major [rows, k/16] E4M3 bytes. The sum over k is
    a float64 matrix product. It is not exact in general: every term is a multiple of 2^-20
    (code values are multiples of 1/2, E4M3 scales of 2^-9) with at most 12 significant bits,
    so the sum is exact only while every partial sum stays below 2^33; beyond that, the usual
    dot-product bound gives |error| <= k * 2^-53 * sum_k |A[m, k] B[n, k]|, about 2^-41 of
    sum |terms| at k = 4096, far below the binary32 accumulation bound the tests compare
    against (k * 2^-24 * sum |terms|). The tensor scales multiply once at the end."""
    v = e2m1_to_f32(np.arange(16)).astype(np.float64)           # the oracle's decodes, as tables
    sv = e4m3_to_f32(np.arange(256)).astype(np.float64)

    def values(codes, scales, rows):
        x = v[unpack_e2m1(codes, rows, k)]
        return x * np.repeat(sv[np.asarray(scales, np.uint8).reshape(rows, k // 16)], 16, axis=1)

    a, b = values(a_codes, a_scales, m), values(b_codes, b_scales, n)
    return (a @ b.T) * (float(np.float32(a_alpha)) * float(np.float32(b_alpha)))
