"""nvfp4_amax_quantize / nvfp4_amax_fakequant without a workspace allocate nothing.

Some callers cannot call cudaMalloc: code running while a CUDA graph is being captured in the
global capture mode, serving runtimes that reserve all device memory for their own pool at
start-up, and plain C callers that receive device buffers but hold no allocator. For them the
one-launch amax + quantize takes NULL for its workspace and then uses one static device word
of the library (the grid-wide barrier's counter) instead of caller memory.

This test calls that no-allocation form twice in a row, on two different tensors, and checks
each result bit for bit against the same entry point given a caller's workspace (the parity
tests of the quantizer use exact comparison, so the tolerance here is zero as well). It also
checks that the one-launch kernel really ran (the caller's barrier counter holds the number of
CTAs that arrived; the two-launch fallback would leave it at zero) and that the calls left the
torch allocator untouched. The file is collected last so that a run stopping at the first
failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth

pytestmark = pytest.mark.gpu

MODE, RULE = 1, 2      # Four Over Six, MSE


def _outputs(g, n, nb):
    return dict(amax=torch.empty(g, device="cuda"), codes=torch.empty(n // 2, dtype=torch.uint8, device="cuda"),
                scales=torch.empty(nb, dtype=torch.uint8, device="cuda"), tscale=torch.empty(g, device="cuda"),
                choice=torch.empty((nb + 7) // 8, dtype=torch.uint8, device="cuda"),
                y=torch.empty(n, dtype=torch.int16, device="cuda"),
                fq_amax=torch.empty(g, device="cuda"), fq_choice=torch.empty((nb + 7) // 8, dtype=torch.uint8,
                                                                             device="cuda"))


def _run(xd, shape, o, workspace, status):
    g, r, c = shape
    nv.nvfp4_amax_quantize(xd, g, r, c, MODE, RULE, o["amax"], o["codes"], o["scales"], o["tscale"], o["choice"],
                           workspace, status)
    nv.nvfp4_amax_fakequant(xd, g, r, c, MODE, RULE, o["fq_amax"], o["y"], o["fq_choice"], workspace, status)


def test_no_workspace_allocates_nothing_and_matches_the_workspace_form(gpu):
    cases = []
    for name, kw in (("c3", dict(rows=512, cols=4096)), ("c4", dict(rows=256, cols=1024, groups=4))):
        x, shape = synth.make(name, **kw)
        cases.append((x, shape, torch.from_numpy(x.view(np.int16)).cuda()))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got, want = [], []
    for x, (g, r, c), xd in cases:
        n = g * r * c
        got.append(_outputs(g, n, n // 16))
        want.append(_outputs(g, n, n // 16))
    torch.cuda.synchronize()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for (x, shape, xd), o in zip(cases, got):          # two no-allocation calls in a row
        _run(xd, shape, o, None, status)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0, "the torch allocator was used"
    assert torch.cuda.memory_reserved() == reserved0, "the torch allocator reserved memory"
    assert status.item() == 0
    for (x, shape, xd), o in zip(cases, want):          # the same entry point with a caller's workspace
        work = torch.zeros(1, dtype=torch.int32, device="cuda")
        _run(xd, shape, o, work, status)
        torch.cuda.synchronize()
        assert work.item() > 1, "the one-launch kernel did not run (two-launch fallback)"
    assert status.item() == 0
    for (x, (g, r, c), xd), a, b in zip(cases, got, want):
        for k in a:
            assert torch.equal(a[k], b[k]), k
        # and both equal the oracle
        amax = O.amax(x, g, r, c)
        assert np.array_equal(a["amax"].cpu().numpy(), amax)
        ref = O.quantize(x, g, r, c, amax, MODE, RULE)
        assert np.array_equal(a["codes"].cpu().numpy(), ref["codes"])
        assert np.array_equal(a["scales"].cpu().numpy(), ref["scales"])
        assert np.array_equal(a["choice"].cpu().numpy(), ref["choice"])
