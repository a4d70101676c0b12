"""Helpers for the GPU parity tests: run the library through its C ABI on guarded device
buffers and fetch the results as numpy arrays, and run the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O

GUARD = 4096          # bytes of canary on each side of every output buffer
CANARY = 0xA5


class Guarded:
    """A device buffer of `nbytes` surrounded by canary bytes (alignment kept at 4096)."""

    def __init__(self, nbytes: int, fill: int | None = None):
        self.nbytes = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.body = self.raw[GUARD:GUARD + nbytes]
        if fill is not None:
            self.body.fill_(fill)

    def ptr(self):
        return self.body.data_ptr() if self.nbytes else self.raw.data_ptr() + GUARD

    def numpy(self, dtype=np.uint8):
        return self.body.cpu().numpy().view(dtype)

    def guards_intact(self) -> bool:
        return bool((self.raw[:GUARD] == CANARY).all()) and bool((self.raw[GUARD + self.nbytes:] == CANARY).all())


def to_device_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x.view(np.int16)).cuda()


def gpu_amax(xd, g, r, c):
    out = Guarded(4 * g)
    nv.nvfp4_amax(xd.data_ptr(), g, r, c, out.ptr())
    torch.cuda.synchronize()
    assert out.guards_intact()
    return out.numpy(np.float32)


def gpu_quantize(xd, g, r, c, amax_np, mode, rule, with_choice=True, stream=None):
    n = g * r * c
    nb = n // 16
    amax_d = torch.from_numpy(np.ascontiguousarray(amax_np, np.float32)).cuda()
    codes, scales, tscale = Guarded(n // 2), Guarded(nb), Guarded(4 * g)
    choice = Guarded((nb + 7) // 8) if with_choice else None
    nv.nvfp4_quantize(xd.data_ptr(), g, r, c, amax_d.data_ptr(), mode, rule, codes.ptr(), scales.ptr(),
                      tscale.ptr(), choice.ptr() if choice else None, stream)
    torch.cuda.synchronize()
    bufs = [codes, scales, tscale] + ([choice] if choice else [])
    assert all(b.guards_intact() for b in bufs), "write outside an output buffer"
    out = dict(codes=codes.numpy(), scales=scales.numpy(), tscale=tscale.numpy(np.float32))
    if choice:
        out["choice"] = choice.numpy()
    return out


def gpu_fakequant(xd, g, r, c, amax_np, mode, rule, with_choice=True):
    n = g * r * c
    nb = n // 16
    amax_d = torch.from_numpy(np.ascontiguousarray(amax_np, np.float32)).cuda()
    y = Guarded(2 * n)
    choice = Guarded((nb + 7) // 8) if with_choice else None
    nv.nvfp4_fakequant(xd.data_ptr(), g, r, c, amax_d.data_ptr(), mode, rule, y.ptr(),
                       choice.ptr() if choice else None)
    torch.cuda.synchronize()
    assert y.guards_intact() and (choice is None or choice.guards_intact())
    out = dict(fq=y.numpy(np.uint16))
    if choice:
        out["choice"] = choice.numpy()
    return out


def gpu_dequantize(codes, scales, tscale, g, r, c):
    n = g * r * c
    cd = torch.from_numpy(np.ascontiguousarray(codes)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(scales)).cuda()
    td = torch.from_numpy(np.ascontiguousarray(tscale, np.float32)).cuda()
    y = Guarded(2 * n)
    nv.nvfp4_dequantize(cd.data_ptr(), sd.data_ptr(), td.data_ptr(), g, r, c, y.ptr())
    torch.cuda.synchronize()
    assert y.guards_intact()
    return y.numpy(np.uint16)


def assert_same(name, got, want):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    if got.dtype == np.float32:
        eq = got.view(np.uint32) == want.view(np.uint32)
    else:
        eq = got == want
    if not eq.all():
        bad = np.flatnonzero(~eq)
        raise AssertionError(f"{name}: {bad.size} of {got.size} differ; first at {bad[:8]}: "
                             f"got {got.ravel()[bad[:8]]} want {want.ravel()[bad[:8]]}")


def check_case(x: np.ndarray, g: int, r: int, c: int, mode: int, rule: int, amax_np=None, fakequant=True,
               dequant=True):
    """Bit-exact comparison of every output of the library against the oracle."""
    xd = to_device_bf16(x)
    if amax_np is None:
        amax_np = O.amax(x, g, r, c)
        assert_same("amax", gpu_amax(xd, g, r, c), amax_np)
    want = O.quantize(x, g, r, c, amax_np, mode, rule)
    got = gpu_quantize(xd, g, r, c, amax_np, mode, rule)
    for k in ("tscale", "scales", "codes", "choice"):
        assert_same(k, got[k], want[k])
    if fakequant:
        wfq = O.fakequant(x, g, r, c, amax_np, mode, rule)
        gfq = gpu_fakequant(xd, g, r, c, amax_np, mode, rule)
        assert_same("fakequant", gfq["fq"], wfq["fq"])
        assert_same("fakequant choice", gfq["choice"], wfq["choice"])
    if dequant:
        gy = gpu_dequantize(got["codes"], got["scales"], got["tscale"], g, r, c)
        assert_same("dequantize", gy, O.dequantize(want["codes"], want["scales"], want["tscale"], g, r, c))
    return got


def host_threads() -> int:
    try:
        import os

        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return 1


def oracle_whole(x: np.ndarray, g: int, r: int, c: int, amax_np, mode: int, rule: int, fakequant: bool = False,
                 threads: int | None = None):
    """The oracle's quantization (fakequant=False: codes, scales, tscale, choice; True: fq,
    choice) of the whole [g, r, c] tensor, computed as independent row ranges on host threads.

    Blocks depend only on their group's amax, so a row range quantized alone gives the same
    bytes as the whole tensor (a CPU test pins this); the C oracle releases the interpreter
    lock while it runs, so the ranges run in parallel."""
    from concurrent.futures import ThreadPoolExecutor

    threads = threads or host_threads()
    n, nb, bpr = g * r * c, g * r * c // 16, c // 16
    parts = max(1, -(-threads // g))
    tasks = [(gi, r * k // parts, r * (k + 1) // parts) for gi in range(g) for k in range(parts)]
    tasks = [t for t in tasks if t[2] > t[1]]
    amax_np = np.ascontiguousarray(amax_np, np.float32)

    def run(t):
        gi, lo, hi = t
        xs = x[(gi * r + lo) * c:(gi * r + hi) * c]
        fn = O.fakequant if fakequant else O.quantize
        return t, fn(xs, 1, hi - lo, c, amax_np[gi:gi + 1], mode, rule)

    out = dict(fq=np.empty(n, np.uint16)) if fakequant else dict(
        codes=np.empty(n // 2, np.uint8), scales=np.empty(nb, np.uint8), tscale=np.zeros(g, np.float32))
    bits = np.empty(nb, np.uint8)
    with ThreadPoolExecutor(min(threads, len(tasks))) as ex:
        for (gi, lo, hi), o in ex.map(run, tasks):
            e0, e1 = (gi * r + lo) * c, (gi * r + hi) * c
            if fakequant:
                out["fq"][e0:e1] = o["fq"]
            else:
                out["codes"][e0 // 2:e1 // 2] = o["codes"]
                out["scales"][e0 // 16:e1 // 16] = o["scales"]
                out["tscale"][gi] = o["tscale"][0]
            bits[e0 // 16:e1 // 16] = np.unpackbits(o["choice"], bitorder="little")[:(hi - lo) * bpr]
    out["choice"] = np.packbits(bits, bitorder="little")
    return out
