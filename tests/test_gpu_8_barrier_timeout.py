"""The one-launch amax + quantize kernel's grid-wide wait is bounded and reports.

A test build of the kernel (tests/probe/barrier_probe.cu) is launched with one more expected
arrival than its grid has CTAs, so no CTA can pass the barrier: every CTA's bounded wait runs
out (about two seconds), the kernel sets NVFP4_QUANT_TIMEOUT in the status word, leaves codes,
scales, tensor scale and choice bits untouched (their canaries survive), and the launch
completes, so the host call returns and the context stays usable. With the right count the
same build completes and matches nvfp4_quantize bit for bit. Nothing faults or hangs.
"""
from __future__ import annotations

import ctypes
import time

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth
from tests import gpu_util as U
from tests.probe import build as probe_build

pytestmark = pytest.mark.gpu

NVFP4_QUANT_TIMEOUT = 2


@pytest.fixture(scope="module")
def probe(gpu):
    L = ctypes.CDLL(probe_build.build_barrier())
    vp, i64, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32
    L.probe_amax_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, vp, vp, u32, ctypes.POINTER(u32)]
    L.probe_amax_quantize.restype = ctypes.c_int
    return L


def _launch(probe, xd, r, c, extra):
    n, nb = r * c, r * c // 16
    out = dict(amax=U.Guarded(4), codes=U.Guarded(n // 2), scales=U.Guarded(nb), tscale=U.Guarded(4),
               choice=U.Guarded((nb + 7) // 8))
    arrive = torch.zeros(1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    grid = ctypes.c_uint32(0)
    t0 = time.perf_counter()
    rc = probe.probe_amax_quantize(xd.data_ptr(), r, c, *(out[k].ptr() for k in ("amax", "codes", "scales", "tscale",
                                                                                 "choice")),
                                   arrive.data_ptr(), status.data_ptr(), extra, ctypes.byref(grid))
    torch.cuda.synchronize()
    return rc, time.perf_counter() - t0, out, int(arrive.item()), int(status.item()), grid.value


def test_grid_barrier_wait_runs_out_and_reports(probe):
    x, (g, r, c) = synth.make("c5", rows=512)
    xd = U.to_device_bf16(x)
    rc, dt, out, arrived, status, grid = _launch(probe, xd, r, c, extra=1)
    assert rc == 0, f"cooperative launch refused ({rc})"
    assert grid > 1
    assert status & NVFP4_QUANT_TIMEOUT, "the timed-out wait did not set the status bit"
    assert arrived == grid, (arrived, grid)          # every CTA arrived; the extra one never does
    assert 0.5 < dt < 60, dt                         # the bounded wait (about 2 s) ran out, then returned
    U.assert_same("amax", out["amax"].numpy(np.float32), O.amax(x, 1, r, c))   # phase 1 completed
    for k in ("codes", "scales", "tscale", "choice"):
        assert out[k].guards_intact(), k
        assert bool((out[k].body == U.CANARY).all()), f"{k} written after a timed-out wait"
    # the context is still usable: a library call right after works and is exact
    a = O.amax(x, 1, r, c)
    got = U.gpu_quantize(xd, 1, r, c, a, 1, 2)
    want = O.quantize(x, 1, r, c, a, 1, 2)
    for k in ("codes", "scales", "tscale", "choice"):
        U.assert_same(k, got[k], want[k])


def test_grid_barrier_with_the_grid_count_completes(probe):
    x, (g, r, c) = synth.make("c5", rows=512)
    xd = U.to_device_bf16(x)
    rc, dt, out, arrived, status, grid = _launch(probe, xd, r, c, extra=0)
    assert rc == 0 and status == 0 and arrived == grid
    a = O.amax(x, 1, r, c)
    U.assert_same("amax", out["amax"].numpy(np.float32), a)
    want = O.quantize(x, 1, r, c, a, 1, 2)
    U.assert_same("codes", out["codes"].numpy(), want["codes"])
    U.assert_same("scales", out["scales"].numpy(), want["scales"])
    U.assert_same("tscale", out["tscale"].numpy(np.float32), want["tscale"])
    U.assert_same("choice", out["choice"].numpy(), want["choice"])
