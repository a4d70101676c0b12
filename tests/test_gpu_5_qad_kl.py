"""QAD distillation loss on the GPU (nvfp4_qad_kl) against the binary64 oracle.

Bounds, derived from the binary32 arithmetic of the kernel: each row's loss is
KL = AT/ZT - lseT + lseS (one online softmax per row); every exponential carries a relative
error below 2^-21 and each thread sums at most vocab/256 terms before a tree reduction, so
the sums ZT, ZS, AT carry a relative error below (vocab/256 + 8) * 2^-23. The loss is then
within that fraction of M = 1 + |lseT| + |lseS| + E_p|t - s| (nats) of the exact value.
Gradients are BF16: within 2^-8 of |g| plus grad_scale * (p + q) times the same fraction."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_13_b200 as nv
import oracle as O
from nvfp4_block_scaled_13_b200 import synth

pytestmark = pytest.mark.gpu


def bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_gpu(t, s, rows, vocab, tau, grad_scale, with_grad, offset=0):
    # offset > 0 places the rows at an address that is only 2-byte aligned (scalar path)
    tt = torch.zeros(rows * vocab + 16, dtype=torch.int16, device="cuda")
    ss = torch.zeros_like(tt)
    tt[offset:offset + rows * vocab] = torch.from_numpy(t.ravel().view(np.int16)).cuda()
    ss[offset:offset + rows * vocab] = torch.from_numpy(s.ravel().view(np.int16)).cuda()
    kl = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
    g = torch.zeros(rows * vocab + 16, dtype=torch.int16, device="cuda") if with_grad else None
    nv.nvfp4_qad_kl(tt.data_ptr() + 2 * offset, ss.data_ptr() + 2 * offset, rows, vocab, tau, grad_scale,
                    kl, (g.data_ptr() + 2 * offset) if with_grad else None)
    torch.cuda.synchronize()
    gout = None
    if with_grad:
        gh = g.cpu().numpy().view(np.uint16)
        assert not gh[:offset].any() and not gh[offset + rows * vocab:].any(), "write outside grad"
        gout = bf16_to_f64(gh[offset:offset + rows * vocab])
    return kl.cpu().numpy().astype(np.float64), gout


def magnitude(t, s, rows, vocab, tau):
    tv = bf16_to_f64(t).reshape(rows, vocab) / tau
    sv = bf16_to_f64(s).reshape(rows, vocab) / tau
    lt = tv.max(1) + np.log(np.exp(tv - tv.max(1, keepdims=True)).sum(1))
    ls = sv.max(1) + np.log(np.exp(sv - sv.max(1, keepdims=True)).sum(1))
    p = np.exp(tv - lt[:, None])
    return 1 + np.abs(lt) + np.abs(ls) + (p * np.abs(tv - sv)).sum(1), p, np.exp(sv - ls[:, None])


# The last three run hundreds of rows at the vocabulary sizes of real models.
CASES = [(64, 1), (16, 5), (64, 8), (33, 1000), (16, 4096), (8, 32000), (4, 131072), (3, 50257),
         (640, 16384), (300, 32000), (96, 131072)]


@pytest.mark.parametrize("rows,vocab", CASES, ids=[f"{r}x{v}" for r, v in CASES])
@pytest.mark.parametrize("tau", [1.0, 2.5])
def test_kl_and_grad_parity(gpu, rows, vocab, tau):
    t, s = synth.qad_logits(rows, vocab, seed=rows * 7 + vocab)
    gs = 1.0 / (tau * rows)
    want_kl, want_g = O.qad_kl(t, s, rows, vocab, tau, gs)
    frac = (vocab / 256 + 8) * 2.0 ** -23
    M, p, q = magnitude(t, s, rows, vocab, tau)
    for offset in ([0, 1] if vocab > 1 else [0]):
        kl, g = run_gpu(t, s, rows, vocab, tau, gs, True, offset)
        assert np.all(np.abs(kl - want_kl) <= frac * M + 1e-7), np.max(np.abs(kl - want_kl) / (frac * M))
        bound = 2.0 ** -8 * np.abs(want_g) + gs * frac * (p + q).ravel() + 1e-30
        assert np.all(np.abs(g - want_g) <= bound), np.max(np.abs(g - want_g) / bound)
        kl2, _ = run_gpu(t, s, rows, vocab, tau, gs, False, offset)
        assert np.array_equal(kl2, kl)


def test_identical_rows_give_exact_zero(gpu):
    t, _ = synth.qad_logits(8, 4096, seed=9)
    kl, g = run_gpu(t, t, 8, 4096, 1.0, 1.0, True)
    assert np.all(kl == 0.0) and np.all(g == 0.0)


def test_extreme_and_confident_logits(gpu):
    rows, vocab = 6, 1024
    t = np.full((rows, vocab), -80.0, np.float32)
    s = np.full((rows, vocab), -80.0, np.float32)
    t[np.arange(rows), np.arange(rows) * 3] = 80.0
    s[np.arange(rows), np.arange(rows) * 3 + (np.arange(rows) % 2)] = 80.0
    tb, sb = synth.to_bf16_bits(t), synth.to_bf16_bits(s)
    want, wg = O.qad_kl(tb, sb, rows, vocab, 1.0, 1.0)
    kl, g = run_gpu(tb, sb, rows, vocab, 1.0, 1.0, True)
    assert np.allclose(kl, want, rtol=1e-5, atol=1e-5)
    assert np.allclose(g, wg, rtol=2.0 ** -8, atol=1e-6)


def test_python_wrappers_and_straight_through_fakequant(gpu):
    t, s = synth.qad_logits(4, 512, seed=11)
    tt = torch.from_numpy(t.view(np.int16)).cuda().view(torch.bfloat16)
    ss = torch.from_numpy(s.view(np.int16)).cuda().view(torch.bfloat16)
    kl, g = nv.qad_kl(tt, ss, tau=1.0)
    want, wg = O.qad_kl(t, s, 4, 512, 1.0, 0.25)
    assert np.allclose(kl.cpu().numpy(), want, rtol=1e-4, atol=1e-6)
    assert np.allclose(g.float().cpu().numpy().ravel(), wg, rtol=2.0 ** -7, atol=1e-7)
    x, _ = synth.make("c1", rows=8, cols=64)
    w = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16).reshape(8, 64).requires_grad_(True)
    y = nv.fakequant_ste(w)
    assert torch.equal(y.detach().view(torch.int16), nv.fakequant(w.detach()).view(torch.int16))
    (y.float() * 3.0).sum().backward()
    assert torch.equal(w.grad.float(), torch.full_like(w.grad.float(), 3.0))
