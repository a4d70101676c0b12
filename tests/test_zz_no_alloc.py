"""The entry points that use scratch memory, called without a workspace, allocate nothing.

nvfp4_amax_quantize and nvfp4_amax_fakequant need one device word for their grid-wide
barrier. Given NULL instead of a workspace they use a word of library memory (a static device
array), so a call makes no allocation of its own: the device's free memory is the same before
and after many calls, the torch allocator is untouched, and the results equal those of calls
with a caller's workspace."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
from nvfp4_block_scaled_13_b200 import synth

pytestmark = pytest.mark.gpu


def test_one_launch_amax_without_workspace_allocates_nothing(gpu):
    x, (g, r, c) = synth.make("c3", rows=512, cols=4096)
    n, nb = g * r * c, g * r * c // 16
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    outs = [dict(amax=torch.empty(g, device="cuda"), codes=torch.empty(n // 2, dtype=torch.uint8, device="cuda"),
                 scales=torch.empty(nb, dtype=torch.uint8, device="cuda"), tscale=torch.empty(g, device="cuda"),
                 choice=torch.empty((nb + 7) // 8, dtype=torch.uint8, device="cuda"),
                 y=torch.empty(n, dtype=torch.int16, device="cuda")) for _ in range(2)]
    work = torch.zeros(2, dtype=torch.int32, device="cuda")

    def run(o, workspace):
        nv.nvfp4_amax_quantize(xd, g, r, c, 1, 2, o["amax"], o["codes"], o["scales"], o["tscale"], o["choice"],
                               workspace, work[1:2])
        nv.nvfp4_amax_fakequant(xd, g, r, c, 1, 2, o["amax"], o["y"], None, workspace, work[1:2])

    run(outs[0], None)   # loads the module and its static data
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(20):
        run(outs[0], None)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0, "device memory was allocated"
    assert torch.cuda.memory_allocated() == alloc0
    assert work[1].item() == 0
    run(outs[1], work[0:1])
    torch.cuda.synchronize()
    for k in outs[0]:
        assert torch.equal(outs[0][k], outs[1][k]), k
