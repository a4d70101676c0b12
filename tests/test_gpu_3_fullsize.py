"""The five workloads at full size, launched exactly as the bench launches them.

The oracle computes the exact amax of the whole tensor and then quantizes sampled rows one
by one (each row depends only on its group's amax), so every sampled output is compared bit
for bit. Properties that hold at any size are checked on the whole tensor: the round trip
dequantize(quantize(x)) equals fakequant(x) bitwise, the block holding the group maximum
gets the largest scale its target allows, and the choice bits are all zero in scale-6 mode.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

SWEEP = {
    "c1": [(0, 2), (1, 2)],
    "c2": [(1, 2)],
    "c3": [(1, 1)],
    "c4": [(1, 2)],
    "c5": [(0, 2), (1, 0), (1, 1), (1, 2)],
}
N_SAMPLE_ROWS = 24


def _bits(choice: np.ndarray, start: int, count: int) -> np.ndarray:
    return np.unpackbits(choice, bitorder="little")[start:start + count]


@pytest.fixture(scope="module", params=sorted(SWEEP))
def workload(request, gpu):
    name = request.param
    x, (g, r, c) = synth.make(name)
    xd = U.to_device_bf16(x)
    amax_ref = O.amax(x, g, r, c)
    yield name, x, xd, (g, r, c), amax_ref
    del xd
    torch.cuda.empty_cache()


def test_fullsize(workload):
    name, x, xd, (g, r, c), amax_ref = workload
    n = g * r * c
    nb = n // 16
    bpr = c // 16
    amax_d = torch.empty(g, dtype=torch.float32, device="cuda")
    nv.nvfp4_amax(xd, g, r, c, amax_d)
    torch.cuda.synchronize()
    U.assert_same("amax", amax_d.cpu().numpy(), amax_ref)
    rng = np.random.default_rng(7)
    rows_total = g * r
    sample = np.unique(np.concatenate([[0, rows_total - 1, r - 1, r], rng.integers(0, rows_total, N_SAMPLE_ROWS)]))
    sample = sample[sample < rows_total]
    for mode, rule in SWEEP[name]:
        codes = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        scales = torch.empty(nb, dtype=torch.uint8, device="cuda")
        tscale = torch.empty(g, dtype=torch.float32, device="cuda")
        choice = torch.empty((nb + 7) // 8, dtype=torch.uint8, device="cuda")
        nv.nvfp4_quantize(xd, g, r, c, amax_d, mode, rule, codes, scales, tscale, choice)
        fq = torch.empty(n, dtype=torch.int16, device="cuda")
        fq_choice = torch.empty_like(choice)
        nv.nvfp4_fakequant(xd, g, r, c, amax_d, mode, rule, fq, fq_choice)
        y = torch.empty(n, dtype=torch.int16, device="cuda")
        nv.nvfp4_dequantize(codes, scales, tscale, g, r, c, y)
        torch.cuda.synchronize()
        # properties of the whole tensor
        assert torch.equal(y, fq), "dequantize(quantize(x)) != fakequant(x)"
        assert torch.equal(choice, fq_choice)
        if mode == 0:
            assert not bool(choice.any())
        codes_h, scales_h, choice_h = codes.cpu().numpy(), scales.cpu().numpy(), choice.cpu().numpy()
        fq_h = fq.cpu().numpy().view(np.uint16)
        ts_want = np.array([O.tensor_scale(a, mode) for a in amax_ref], np.float32)
        U.assert_same("tscale", tscale.cpu().numpy(), ts_want)
        # the block holding each group's maximum: scale 448 (scale-6) or 256/384 (4/6)
        xg = x.reshape(g, -1)
        for gi in range(min(g, 8)):
            top = gi * (r * c // 16) + int(np.argmax(xg[gi] & 0x7FFF)) // 16
            if amax_ref[gi] > 2.0 ** -100:
                want_s = (0x7E,) if mode == 0 else (0x78, 0x7C)
                assert scales_h[top] in want_s, (gi, hex(scales_h[top]))
        # sampled rows, bit for bit
        for row in sample:
            gi = row // r
            xr = np.ascontiguousarray(x[row * c:(row + 1) * c])
            want = O.quantize(xr, 1, 1, c, amax_ref[gi:gi + 1], mode, rule)
            U.assert_same(f"codes row {row}", codes_h[row * c // 2:(row + 1) * c // 2], want["codes"])
            U.assert_same(f"scales row {row}", scales_h[row * bpr:(row + 1) * bpr], want["scales"])
            U.assert_same(f"choice row {row}", _bits(choice_h, row * bpr, bpr), _bits(want["choice"], 0, bpr))
            if name == "c3":
                wfq = O.fakequant(xr, 1, 1, c, amax_ref[gi:gi + 1], mode, rule)["fq"]
                U.assert_same(f"fakequant row {row}", fq_h[row * c:(row + 1) * c], wfq)
        del codes, scales, tscale, choice, fq, fq_choice, y
