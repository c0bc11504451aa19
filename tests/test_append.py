"""KV-cache append and the growing-context decode loop (GPU): the appended
rows land bit-exact at position l_kv[b], lengths grow on the device, and
Atop-N steps over the grown caches pass the same per-row parity checks as
the fixed-length chains."""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_decode_attention_step_b200 as saga
import synth
from synth import device as sdev

from gpu_harness import Chain, SynthRows, check_row, dev_dtype, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(gpu_lib):
    import os
    if not os.path.exists(sdev.LIB_PATH):
        sdev.build()
    return gpu_lib


def new_rows(w, kind, heads, pos):
    """Storage-dtype rows [B][heads][d] of the generator's cache at position pos[b]."""
    out = np.stack([np.stack([synth.cache_rows(w, 0, kind, b, hh, int(pos[b]), int(pos[b]) + 1)[0]
                              for hh in range(heads)]) for b in range(w.B)])
    return np.ascontiguousarray(out)


def workload(dtype, B, cap, N, R):
    return synth.Workload("grow", dtype, B=B, h_q=16, h_k=2, h_v=4, d=64, l_kv=cap, N=N, R=R,
                          steps=1, seed=20261210)


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
def test_append_writes_rows_and_grows_lengths(dtype):
    w = workload(dtype, 3, 1024, 64, 4)
    shp = saga.shape(w.B, w.h_q, w.h_k, w.h_v, w.d, w.dtype, w.l_kv, w.l_kv)
    K = torch.zeros(w.B, w.h_k, w.l_kv, w.d, dtype=dev_dtype(w), device="cuda")
    V = torch.zeros(w.B, w.h_v, w.l_kv, w.d, dtype=dev_dtype(w), device="cuda")
    l0 = np.array([0, 517, 1020], dtype=np.int32)
    l = torch.from_numpy(l0).cuda()
    ws = saga.Workspace(shp, w.N)
    for s in range(4):
        pos = l0 + s
        saga.append_kv(shp, to_dev(new_rows(w, "K", w.h_k, pos)), to_dev(new_rows(w, "V", w.h_v, pos)),
                       K, V, l, ws)
    torch.cuda.synchronize()
    assert np.array_equal(l.cpu().numpy(), l0 + 4)
    assert saga.read_device_error(ws) == 0
    Kh, Vh = K.cpu().numpy(), V.cpu().numpy()
    for b in range(w.B):
        for kind, arr, heads in (("K", Kh, w.h_k), ("V", Vh, w.h_v)):
            for hh in range(heads):
                want = synth.cache_rows(w, 0, kind, b, hh, int(l0[b]), int(l0[b]) + 4)
                got = arr[b, hh, l0[b]:l0[b] + 4]
                assert np.array_equal(got.view(want.dtype), want), (kind, b, hh)
                assert not np.any(arr[b, hh, :l0[b]]) and not np.any(arr[b, hh, l0[b] + 4:])


def test_append_to_a_full_cache_sets_the_error_word():
    w = workload(synth.BF16, 2, 256, 8, 4)
    shp = saga.shape(w.B, w.h_q, w.h_k, w.h_v, w.d, w.dtype, w.l_kv, w.l_kv)
    K = torch.zeros(w.B, w.h_k, w.l_kv, w.d, dtype=torch.int16, device="cuda")
    V = torch.zeros(w.B, w.h_v, w.l_kv, w.d, dtype=torch.int16, device="cuda")
    l = torch.tensor([256, 100], dtype=torch.int32, device="cuda")
    ws = saga.Workspace(shp, w.N)
    ones_k = torch.ones(w.B, w.h_k, w.d, dtype=torch.int16, device="cuda")
    ones_v = torch.ones(w.B, w.h_v, w.d, dtype=torch.int16, device="cuda")
    saga.append_kv(shp, ones_k, ones_v, K, V, l, ws)
    torch.cuda.synchronize()
    assert l.cpu().tolist() == [256, 101]
    assert saga.read_device_error(ws) == saga.DEVERR_LKV_TOO_LONG
    assert not torch.any(K[0]) and torch.all(K[1, :, 100] == 1)


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
def test_growing_context_decode_loop(dtype):
    """Append then attend, step after step, refreshing every R steps: every
    row of every step against the oracle over the grown cache."""
    T, R = 7, 3
    w = workload(dtype, 3, 4096, 96, R)
    l0 = np.array([4096 - T, 1500, 37], dtype=np.int32)
    K = torch.empty(w.B, w.h_k, w.l_kv, w.d, dtype=dev_dtype(w), device="cuda")
    V = torch.empty(w.B, w.h_v, w.l_kv, w.d, dtype=dev_dtype(w), device="cuda")
    sdev.fill(K, w, 0, "K")
    sdev.fill(V, w, 0, "V")
    for b in range(w.B):           # positions from l0 on are not in the cache yet
        K[b, :, l0[b]:] = 0
        V[b, :, l0[b]:] = 0
    shp = saga.shape(w.B, w.h_q, w.h_k, w.h_v, w.d, w.dtype, w.l_kv, w.l_kv)
    ch = Chain(shp, K, V, l0, w.N)
    rows = SynthRows(w, 0)
    qs = synth.queries(w, 0, T)
    q64 = synth.widen(qs)
    tau_o = {}
    G = w.h_q // w.h_k
    for t in range(T):
        pos = l0 + t
        saga.append_kv(shp, to_dev(new_rows(w, "K", w.h_k, pos)), to_dev(new_rows(w, "V", w.h_v, pos)),
                       K, V, ch.l, ch.ws)
        rec = ch.step(to_dev(qs[t]), t % R == 0)
        for b in range(w.B):
            L = int(pos[b]) + 1
            for kh in range(w.h_k):
                krow = rows.k_row(b, kh, L)
                for j in range(kh * G, (kh + 1) * G):
                    tau_o[(b, j)] = check_row(rec, q64[t, b, j], krow, rows, b, j, w.h_q, w.h_v,
                                              L, w.d, w.N, t % R == 0, w.dtype, tau_o.get((b, j)))
    assert np.array_equal(ch.l.cpu().numpy(), l0 + T)
