"""The threaded whole-tensor oracle that the full-size GPU comparison uses gives the same
bytes as one call of the oracle over the whole tensor (several groups, a row count that does
not divide by the thread count, every mode and rule, codes and fake-quant)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from nvfp4_block_scaled_13_b200 import synth
from tests import gpu_util as U


@pytest.mark.parametrize("name,kw,threads", [("c4", dict(rows=64, groups=5), 7), ("c5", dict(rows=40), 16),
                                             ("c3", dict(rows=24, cols=512), 5)])
def test_threaded_oracle_equals_one_call(name, kw, threads):
    x, (g, r, c) = synth.make(name, **kw)
    a = O.amax(x, g, r, c)
    for mode, rule in [(0, 2), (1, 0), (1, 1), (1, 2)]:
        want = O.quantize(x, g, r, c, a, mode, rule)
        got = U.oracle_whole(x, g, r, c, a, mode, rule, threads=threads)
        for k in want:
            assert np.array_equal(want[k], got[k]), (name, mode, rule, k)
        wf = O.fakequant(x, g, r, c, a, mode, rule)
        gf = U.oracle_whole(x, g, r, c, a, mode, rule, fakequant=True, threads=threads)
        for k in wf:
            assert np.array_equal(wf[k], gf[k]), (name, mode, rule, k)
