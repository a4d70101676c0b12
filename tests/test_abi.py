"""The C-ABI boundary without a GPU: the library loads, exports every symbol its header
declares, and rejects invalid arguments on the host before enqueuing anything."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_13_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions(path):
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_functions(os.path.join(ROOT, "include", "nvfp4.h"))
    assert names == ["nvfp4_amax", "nvfp4_amax_fakequant", "nvfp4_amax_quantize", "nvfp4_dequantize", "nvfp4_fakequant", "nvfp4_gemm", "nvfp4_gemm_bf16", "nvfp4_gemm_quantize_x",
                     "nvfp4_qad_kl", "nvfp4_quantize", "nvfp4_quantize_gemm", "nvfp4_status_string",
                     "nvfp4_version"]


def test_library_exports_every_declared_symbol():
    lib = nv.load()
    for name in header_functions(os.path.join(ROOT, "include", "nvfp4.h")):
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    assert nv.nvfp4_version() == 100
    assert nv.nvfp4_status_string(0) == "ok"
    for s in range(1, 8):
        assert nv.nvfp4_status_string(s) not in ("ok", "unknown nvfp4_status")
    assert nv.nvfp4_status_string(99) == "unknown nvfp4_status"


# Fake device addresses: validation rejects these calls before any CUDA call is made.
A = 1 << 20          # 32-byte aligned


@pytest.mark.parametrize("call,expected", [
    # nvfp4_amax(x, G, R, C, amax, stream)
    (lambda L: L.nvfp4_amax(A, 1, 4, 32, None, None), 1),
    (lambda L: L.nvfp4_amax(None, 1, 4, 32, A, None), 1),
    (lambda L: L.nvfp4_amax(A, 0, 4, 32, A, None), 2),
    (lambda L: L.nvfp4_amax(A, 1, -1, 32, A, None), 2),
    (lambda L: L.nvfp4_amax(A, 1, 4, 24, A, None), 2),
    (lambda L: L.nvfp4_amax(A + 16, 1, 4, 32, A, None), 3),
    (lambda L: L.nvfp4_amax(A, 1, 4, 32, A + 2, None), 3),
    (lambda L: L.nvfp4_amax(A, 1 << 40, 1 << 20, 1 << 20, A, None), 2),
    # nvfp4_quantize(x, G, R, C, amax, mode, rule, codes, scales, tscale, choice, stream)
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, None, 1, 2, A, A, A, None, None), 1),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, 2, None, A, A, None, None), 1),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, 2, A, None, A, None, None), 1),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, 2, A, A, None, None, None), 1),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 33, A, 1, 2, A, A, A, None, None), 2),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 2, 2, A, A, A, None, None), 4),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, 3, A, A, A, None, None), 5),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, -1, A, A, A, None, None), 5),
    (lambda L: L.nvfp4_quantize(A + 2, 1, 4, 32, A, 1, 2, A, A, A, None, None), 3),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, 2, A + 4, A, A, None, None), 3),
    (lambda L: L.nvfp4_quantize(A, 1, 4, 32, A, 1, 2, A, A, A, A + 1, None), 3),
    # nvfp4_dequantize(codes, scales, tscale, G, R, C, y, stream)
    (lambda L: L.nvfp4_dequantize(None, A, A, 1, 4, 32, A, None), 1),
    (lambda L: L.nvfp4_dequantize(A, A, A, 1, 4, 32, None, None), 1),
    (lambda L: L.nvfp4_dequantize(A, A, A, 1, 4, 31, A, None), 2),
    (lambda L: L.nvfp4_dequantize(A, A, A, 1, 4, 32, A + 8, None), 3),
    # nvfp4_quantize_gemm(x, R, C, amax, mode, rule, codes, scales, tscale, choice, stream)
    (lambda L: L.nvfp4_quantize_gemm(A, 4, 32, None, 1, 2, A, A, A, None, None), 1),
    (lambda L: L.nvfp4_quantize_gemm(A, 4, 32, A, 1, 2, A, None, A, None, None), 1),
    (lambda L: L.nvfp4_quantize_gemm(A, 4, 40, A, 1, 2, A, A, A, None, None), 2),
    (lambda L: L.nvfp4_quantize_gemm(A, 1 << 20, 1 << 15, A, 1, 2, A, A, A, None, None), 2),
    (lambda L: L.nvfp4_quantize_gemm(A, 4, 32, A, 3, 2, A, A, A, None, None), 4),
    (lambda L: L.nvfp4_quantize_gemm(A, 4, 32, A, 1, 7, A, A, A, None, None), 5),
    (lambda L: L.nvfp4_quantize_gemm(A + 8, 4, 32, A, 1, 2, A, A, A, None, None), 3),
    # nvfp4_qad_kl(teacher, student, rows, vocab, tau, grad_scale, kl, grad, stream)
    (lambda L: L.nvfp4_qad_kl(A, A, 4, 0, 1.0, 1.0, A, None, None), 2),
    (lambda L: L.nvfp4_qad_kl(A, A, -1, 8, 1.0, 1.0, A, None, None), 2),
    (lambda L: L.nvfp4_qad_kl(A, A, 4, 8, 0.0, 1.0, A, None, None), 7),
    (lambda L: L.nvfp4_qad_kl(A, A, 4, 8, float("inf"), 1.0, A, None, None), 7),
    (lambda L: L.nvfp4_qad_kl(A, A, 4, 8, 1.0, float("nan"), A, None, None), 7),
    (lambda L: L.nvfp4_qad_kl(None, A, 4, 8, 1.0, 1.0, A, None, None), 1),
    (lambda L: L.nvfp4_qad_kl(A, A, 4, 8, 1.0, 1.0, None, None, None), 1),
    (lambda L: L.nvfp4_qad_kl(A + 1, A, 4, 8, 1.0, 1.0, A, None, None), 3),
    (lambda L: L.nvfp4_qad_kl(A, A, 4, 8, 1.0, 1.0, A + 2, None, None), 3),
    # nvfp4_gemm(xc, xs, xt, wc, ws, wt, m, n, k, y, status, stream)
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 128, 256, 200, A, None, None), 2),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 128, 192, 256, A, None, None), 2),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, -1, 256, 256, A, None, None), 2),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 128, 256, 0, A, None, None), 2),
    (lambda L: L.nvfp4_gemm(None, A, A, A, A, A, 128, 256, 256, A, None, None), 1),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 128, 256, 256, None, None, None), 1),
    (lambda L: L.nvfp4_gemm(A + 8, A, A, A, A, A, 128, 256, 256, A, None, None), 3),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 128, 256, 256, A, A + 2, None), 3),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 128, 256, 256, A + 16, None, None), 3),
    (lambda L: L.nvfp4_gemm(A, A, A, A, A, A, 0, 256, 256, None, None, None), 0),
    # nvfp4_gemm_bf16(xc, xs, xt, wc, ws, wt, m, n, k, y, y_amax, status, stream)
    (lambda L: L.nvfp4_gemm_bf16(A, A, A, A, A, A, 128, 256, 200, A, A, None, None), 2),
    (lambda L: L.nvfp4_gemm_bf16(A, A, A, A, A, A, 128, 192, 256, A, A, None, None), 2),
    (lambda L: L.nvfp4_gemm_bf16(None, A, A, A, A, A, 128, 256, 256, A, A, None, None), 1),
    (lambda L: L.nvfp4_gemm_bf16(A, A, A, A, A, A, 128, 256, 256, None, A, None, None), 1),
    (lambda L: L.nvfp4_gemm_bf16(A, A, A, A, A, A, 128, 256, 256, A + 16, A, None, None), 3),
    (lambda L: L.nvfp4_gemm_bf16(A, A, A, A, A, A, 128, 256, 256, A, A + 2, None, None), 3),
    (lambda L: L.nvfp4_gemm_bf16(A, A, A, A, A, A, 0, 256, 256, None, None, None, None), 0),
    # nvfp4_gemm_quantize_x(x, amax, mode, rule, wc, ws, wt, m, n, k, y, status, stream)
    (lambda L: L.nvfp4_gemm_quantize_x(A, A, 2, 2, A, A, A, 128, 256, 256, A, None, None), 4),
    (lambda L: L.nvfp4_gemm_quantize_x(A, A, 1, 3, A, A, A, 128, 256, 256, A, None, None), 5),
    (lambda L: L.nvfp4_gemm_quantize_x(A, A, 1, 2, A, A, A, 128, 64, 256, A, None, None), 2),
    (lambda L: L.nvfp4_gemm_quantize_x(A, A, 1, 2, A, A, A, 100, 128, 320, A, None, None), 2),
    (lambda L: L.nvfp4_gemm_quantize_x(None, A, 1, 2, A, A, A, 128, 256, 256, A, None, None), 1),
    (lambda L: L.nvfp4_gemm_quantize_x(A, None, 1, 2, A, A, A, 128, 256, 256, A, None, None), 1),
    (lambda L: L.nvfp4_gemm_quantize_x(A + 16, A, 1, 2, A, A, A, 128, 256, 256, A, None, None), 3),
    # nvfp4_amax_quantize(x, G, R, C, mode, rule, amax, codes, scales, tscale, choice, workspace, status, stream)
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 2, None, A, A, A, None, None, None, None), 1),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 2, A, None, A, A, None, None, None, None), 1),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 2, A, A, A, None, None, None, None, None), 1),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 33, 1, 2, A, A, A, A, None, None, None, None), 2),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 3, 2, A, A, A, A, None, None, None, None), 4),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 3, A, A, A, A, None, None, None, None), 5),
    (lambda L: L.nvfp4_amax_quantize(A + 2, 1, 4, 32, 1, 2, A, A, A, A, None, None, None, None), 3),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 2, A + 2, A, A, A, None, None, None, None), 3),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 2, A, A, A, A, None, A + 2, None, None), 3),
    (lambda L: L.nvfp4_amax_quantize(A, 1, 4, 32, 1, 2, A, A, A, A, None, None, A + 1, None), 3),
    # nvfp4_amax_fakequant(x, G, R, C, mode, rule, amax, y, choice, workspace, status, stream)
    (lambda L: L.nvfp4_amax_fakequant(A, 1, 4, 32, 1, 2, None, A, None, None, None, None), 1),
    (lambda L: L.nvfp4_amax_fakequant(A, 1, 4, 32, 1, 2, A, None, None, None, None, None), 1),
    (lambda L: L.nvfp4_amax_fakequant(A, 1, 4, 31, 1, 2, A, A, None, None, None, None), 2),
    (lambda L: L.nvfp4_amax_fakequant(A, 1, 4, 32, 1, 9, A, A, None, None, None, None), 5),
    (lambda L: L.nvfp4_amax_fakequant(A, 1, 4, 32, 1, 2, A, A + 16, None, None, None, None), 3),
    # nvfp4_fakequant(x, G, R, C, amax, mode, rule, y, choice, stream)
    (lambda L: L.nvfp4_fakequant(A, 1, 4, 32, A, 1, 2, None, None, None), 1),
    (lambda L: L.nvfp4_fakequant(A, 1, 4, 32, A, 7, 2, A, None, None), 4),
    (lambda L: L.nvfp4_fakequant(A, 1, 4, 32, A, 1, 9, A, None, None), 5),
    (lambda L: L.nvfp4_fakequant(A, 1, 4, 32, A, 1, 2, A + 16, None, None), 3),
])
def test_invalid_arguments_rejected_on_host(call, expected):
    assert call(nv.load()) == expected


def test_rule_ignored_in_scale6_mode_but_mode_checked():
    L = nv.load()
    # invalid rule with scale-6 mode passes validation; a NULL x then fails with ERR_NULL
    assert L.nvfp4_quantize(None, 1, 4, 32, A, 0, 77, A, A, A, None, None) == 1


def test_python_wrappers_refuse_cpu_tensors():
    import torch

    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        nv.amax(x)


def test_oracle_library_exports_its_header():
    import oracle

    L = oracle.lib()
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "oracle", "nvfp4_oracle.h")).read(), flags=re.S)
    for name in set(re.findall(r"\b(nvo_\w+)\s*\(", text)):
        assert hasattr(L, name), name


def test_product_does_not_import_oracle():
    """The product package and its build never touch the oracle."""
    pkg = os.path.join(ROOT, "nvfp4_block_scaled_13_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "nvfp4_oracle" not in text and "nvo_" not in text, f
