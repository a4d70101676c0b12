"""The five workloads at full size, launched as the bench launches them, compared whole.

Every output of every (mode, rule) the workload sweeps is compared bit for bit with the
oracle over the whole tensor: the exact amax, the tensor scale, every code, scale and choice
bit, and (the activation workload, whose product is the QAD student's forward) every
fake-quant value. The oracle runs as independent row ranges on the host's threads (blocks
depend only on their group's amax). The whole-tensor properties stay as a second line:
dequantize(quantize(x)) equals fakequant(x), and the block holding each group's maximum
gets the largest scale its target allows.
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
FAKEQUANT_ORACLE = {"c3"}      # the workload whose output is the fake-quant BF16


@pytest.fixture(scope="module", params=sorted(SWEEP))
def workload(request, gpu):
    name = request.param
    x, (g, r, c) = synth.make(name)
    xd = U.to_device_bf16(x)
    amax_ref = O.amax(x, g, r, c)
    yield name, x, xd, (g, r, c), amax_ref
    del xd
    torch.cuda.empty_cache()


def test_fullsize_whole_tensor(workload):
    name, x, xd, (g, r, c), amax_ref = workload
    n = g * r * c
    nb = n // 16
    amax_d = torch.empty(g, dtype=torch.float32, device="cuda")
    nv.nvfp4_amax(xd, g, r, c, amax_d)
    torch.cuda.synchronize()
    U.assert_same("amax", amax_d.cpu().numpy(), amax_ref)
    for mode, rule in SWEEP[name]:
        tag = f"{name} mode {mode} rule {rule}"
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
        assert torch.equal(y, fq), f"{tag}: dequantize(quantize(x)) != fakequant(x)"
        assert torch.equal(choice, fq_choice), tag
        del y
        want = U.oracle_whole(x, g, r, c, amax_ref, mode, rule)
        U.assert_same(f"{tag} tscale", tscale.cpu().numpy(), want["tscale"])
        scales_h = scales.cpu().numpy()
        U.assert_same(f"{tag} scales", scales_h, want["scales"])
        U.assert_same(f"{tag} codes", codes.cpu().numpy(), want["codes"])
        U.assert_same(f"{tag} choice", choice.cpu().numpy(), want["choice"])
        if mode == 0:
            assert not want["choice"].any()
        del want
        if name in FAKEQUANT_ORACLE:
            wfq = U.oracle_whole(x, g, r, c, amax_ref, mode, rule, fakequant=True)
            U.assert_same(f"{tag} fakequant", fq.cpu().numpy().view(np.uint16), wfq["fq"])
            U.assert_same(f"{tag} fakequant choice", fq_choice.cpu().numpy(), wfq["choice"])
            del wfq
        # the block holding each group's maximum: scale 448 (scale-6) or 256/384 (4/6)
        xg = x.reshape(g, -1)
        for gi in range(min(g, 8)):
            top = gi * (r * c // 16) + int(np.argmax(xg[gi] & 0x7FFF)) // 16
            if amax_ref[gi] > 2.0 ** -100:
                want_s = (0x7E,) if mode == 0 else (0x78, 0x7C)
                assert scales_h[top] in want_s, (gi, hex(scales_h[top]))
        del codes, scales, tscale, choice, fq, fq_choice
