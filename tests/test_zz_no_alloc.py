"""The allocation-free decode step (saga_decode_step_noalloc), for callers
that cannot allocate device memory: it runs the same plan and kernels as the
ordinary saga_decode_step, so its output and counts must equal that call's
bit for bit, on two calls in a row (the second call finds the first call's
leftovers in the shared scratch array), and pass the oracle's row checks.
Shapes whose scratch just fits the fixed array run; one sequence more is
refused. This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_decode_attention_step_b200 as saga
import synth

from gpu_harness import Chain, HostRows, check_row

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def planned_scratch_bytes(B, h_q, h_k, h_v, d, L):
    """Scratch of a plain step on the tensor-core path, as the library plans
    it: the 256-byte error and abort words; one (m, l, count, pad, acc[d])
    float record per (b, j, gather split); and, per (b, j) and 32-position
    block, a 4-byte kept mask and 32 4-byte kept scores. Each part is rounded
    up to 256 bytes. The gather splits each (b, j) row so that all rows take
    at most 4736 CTAs (more only when there are more rows), each at least 64
    blocks long."""
    up = lambda x: -(-x // 256) * 256
    cdiv = lambda a, b: -(-a // b)
    nblk = cdiv(L, 32)
    sb = min(max(1, nblk // 64), max(1, 4736 // (B * h_q)))
    bps = cdiv(nblk, sb)
    SB = cdiv(nblk, bps)
    lists = B * h_q * nblk
    off = up(256 + B * h_q * SB * (d + 4) * 4)
    off = up(off + lists * 4)
    return up(off + lists * 32 * 4)


def test_noalloc_matches_workspace_step_twice():
    assert torch.cuda.is_available()
    saga.load()
    w = synth.Workload("noalloc", synth.BF16, B=2, h_q=16, h_k=2, h_v=4, d=64, l_kv=3000,
                       N=64, R=1, steps=3, seed=9090)
    lens = np.array([3000, 1777], dtype=np.int32)
    Kh = synth.cache(w, 0, "K", w.h_k, 3000, lens)
    Vh = synth.cache(w, 0, "V", w.h_v, 3000, lens)
    qs = synth.queries(w, 0, 3)
    q64 = synth.widen(qs)
    rows = HostRows(synth.widen(Kh), synth.widen(Vh))
    K, V = dev(Kh), dev(Vh)
    shp = saga.shape(w.B, w.h_q, w.h_k, w.h_v, w.d, w.dtype, 3000)
    ch = Chain(shp, K, V, lens, w.N)             # checked calls: mask, counts, score rows
    rec0 = ch.step(dev(qs[0]), refresh=True)
    tau_o = {}
    for b in range(w.B):
        for j in range(w.h_q):
            kh = j // (w.h_q // w.h_k)
            tau_o[(b, j)] = check_row(rec0, q64[0, b, j], rows.k_row(b, kh, int(lens[b])), rows,
                                      b, j, w.h_q, w.h_v, int(lens[b]), w.d, w.N, True, w.dtype,
                                      None)
    for t in (1, 2):                       # two calls in a row
        q = dev(qs[t])
        rec = ch.step(q, refresh=False)    # saga_decode_step on the same tau
        out = torch.full((w.B, w.h_q, w.d), float("nan"), device="cuda")
        cnt = torch.full((w.B, w.h_q), -1, dtype=torch.int32, device="cuda")
        saga.decode_step_noalloc(shp, q, K, V, ch.l, ch.tau, out, sel_count=cnt)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), rec.out.view(np.uint32))
        np.testing.assert_array_equal(cnt.cpu().numpy(), rec.cnt)
        for b in range(w.B):
            for j in range(w.h_q):
                kh = j // (w.h_q // w.h_k)
                tau_o[(b, j)] = check_row(rec, q64[t, b, j], rows.k_row(b, kh, int(lens[b])),
                                          rows, b, j, w.h_q, w.h_v, int(lens[b]), w.d, w.N,
                                          False, w.dtype, tau_o[(b, j)])


def test_noalloc_scratch_limit_both_sides():
    """The largest batch of 128K-position sequences (h_q=16, h_k=2, h_v=4,
    d=64) whose scratch fits the fixed array runs and matches
    saga_decode_step; one sequence more is refused before anything runs."""
    lib = saga.load()
    limit = saga.NOALLOC_SCRATCH_BYTES
    L, h_q, h_k, h_v, d = 131072, 16, 2, 4, 64
    under = max(B for B in range(1, 256) if planned_scratch_bytes(B, h_q, h_k, h_v, d, L) <= limit)
    over = under + 1
    assert planned_scratch_bytes(over, h_q, h_k, h_v, d, L) > limit

    big = saga.shape(over, h_q, h_k, h_v, d, synth.BF16, L)
    fake = 1 << 40          # never dereferenced: the call is refused first
    rc = lib.saga_decode_step_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake, fake,
                                      None, None)
    assert rc == saga.SAGA_ERR_WORKSPACE

    w = synth.Workload("noalloc_edge", synth.BF16, B=under, h_q=h_q, h_k=h_k, h_v=h_v, d=d,
                       l_kv=L, N=16, R=1, steps=2, seed=777)
    from synth import device as sdev
    K = torch.empty(under, h_k, L, d, dtype=torch.int16, device="cuda")
    V = torch.empty(under, h_v, L, d, dtype=torch.int16, device="cuda")
    sdev.fill(K, w, 0, "K")
    sdev.fill(V, w, 0, "V")
    lens = np.full(under, L, dtype=np.int32)
    lens[::7] = 77                                # ragged tails too
    lens[1::5] = L - 45
    shp = saga.shape(under, h_q, h_k, h_v, d, synth.BF16, L)
    ch = Chain(shp, K, V, lens, w.N, dump=False)
    qs = synth.queries(w, 0, 2)
    ch.step(dev(qs[0]), refresh=True)
    q = dev(qs[1])
    rec = ch.step(q, refresh=False)
    out = torch.full((under, h_q, d), float("nan"), device="cuda")
    cnt = torch.full((under, h_q), -1, dtype=torch.int32, device="cuda")
    saga.decode_step_noalloc(shp, q, K, V, ch.l, ch.tau, out, sel_count=cnt)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), rec.out.view(np.uint32))
    np.testing.assert_array_equal(cnt.cpu().numpy(), rec.cnt)
