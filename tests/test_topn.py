"""Exact top-N attention (Eq. 6 with ties to the lower position) on the GPU:
the kept set equals the N largest of the GPU's own dumped fp32 score row
under totalOrder (checked exactly, as integers), the count is exactly
min(N, l_kv), and the output matches the oracle's Eq. (7) on that set."""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_decode_attention_step_b200 as saga
import synth
from synth import device as sdev

from gpu_harness import OUT_TOL, SCORE_TOL, HostRows, SynthRows, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(gpu_lib):
    import os
    if not os.path.exists(sdev.LIB_PATH):
        sdev.build()
    return gpu_lib


def run_topn(w, Kh, Vh, lens, N):
    rows = HostRows(synth.widen(Kh), synth.widen(Vh))
    check_topn(w, to_dev(Kh), to_dev(Vh), Kh.shape[2], lens, N, rows)


def check_topn(w, K, V, cap, lens, N, rows, heads=None):
    B, h_q, d = w.B, w.h_q, w.d
    shp = saga.shape(B, h_q, w.h_k, w.h_v, d, w.dtype, cap)
    ws = saga.Workspace(shp, N)
    qs = synth.queries(w, 0, 1, B=B, h_q=h_q)
    l = torch.from_numpy(lens).cuda()
    out = torch.zeros(B, h_q, d, dtype=torch.float32, device="cuda")
    cnt = torch.zeros(B, h_q, dtype=torch.int32, device="cuda")
    mask = torch.full((B, h_q, cap), 2, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(B, h_q, cap, dtype=torch.float32, device="cuda")
    saga.topn_step(shp, to_dev(qs[0]), K, V, l, N, out, ws, sel_count=cnt,
                   sel_mask=mask, scores=sc)
    torch.cuda.synchronize()
    assert saga.read_device_error(ws) == 0
    q64 = synth.widen(qs[0])
    o, c, m, s = out.cpu().numpy(), cnt.cpu().numpy(), mask.cpu().numpy(), sc.cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        for j in (range(h_q) if heads is None else heads):
            kh, vh = orc.key_head(j, h_q, w.h_k), orc.value_head(j, h_q, w.h_v)
            assert np.all(m[b, j, L:] == 2)
            kept = np.nonzero(m[b, j, :L] == 1)[0]
            assert c[b, j] == kept.size == min(N, L)
            keys = orc.f32_order_key(s[b, j, :L]).astype(np.float64)   # exact integers
            assert np.array_equal(kept, orc.top_n_exact(keys, N)), (b, j)
            A = rows.k_row(b, kh, L) @ q64[b, j] / np.sqrt(d)
            if L:
                assert np.max(np.abs(s[b, j, :L] - A)) <= SCORE_TOL * max(1.0, np.max(np.abs(A)))
            ref = orc.sparse_attend(A[kept], rows.v_rows(b, vh, kept), np.arange(kept.size))
            assert rel_err(o[b, j].astype(np.float64), ref) <= OUT_TOL[w.dtype], (b, j)


@pytest.mark.parametrize("dtype,d,h_q,h_k,h_v", [
    (synth.BF16, 64, 16, 2, 4), (synth.BF16, 128, 12, 1, 4), (synth.F32, 64, 4, 1, 2)])
@pytest.mark.parametrize("N", [1, 7, 45, 100, 1500, 2999, 5000])
def test_topn_with_heavy_ties(dtype, d, h_q, h_k, h_v, N):
    """Caches made of one 100-position block repeated: every score value
    occurs 30 times, so the N-th largest is almost always tied."""
    cap = 3000
    w = synth.Workload("ties", dtype, B=2, h_q=h_q, h_k=h_k, h_v=h_v, d=d, l_kv=cap, N=N, R=1,
                       steps=1, seed=321 + d)
    lens = np.array([cap, 1234], dtype=np.int32)
    Kh = synth.cache(w, 0, "K", h_k, cap, lens)
    Vh = synth.cache(w, 0, "V", h_v, cap, lens)
    Kh = np.ascontiguousarray(np.tile(Kh[:, :, :100], (1, 1, cap // 100, 1)))
    run_topn(w, Kh, Vh, lens, N)


@pytest.mark.parametrize("N", [1, 777, 32999])
def test_topn_rows_of_one_score(N):
    """Every key of a sequence the same row, so every score of a head is the
    same value: the radix select's top-byte bucket is the whole row (more
    than its bucket list holds) and so is the 16-bit bucket (more than the
    on-chip candidates), which takes the select through its passes over the
    row; the kept set is the first N positions."""
    cap = 40000
    w = synth.Workload("one_score", synth.BF16, B=2, h_q=4, h_k=1, h_v=2, d=64, l_kv=cap, N=N,
                       R=1, steps=1, seed=97)
    lens = np.array([cap, 33000], dtype=np.int32)
    Kh = synth.cache(w, 0, "K", 1, cap, lens)
    Vh = synth.cache(w, 0, "V", 2, cap, lens)
    Kh = np.ascontiguousarray(np.repeat(Kh[:, :, :1], cap, axis=2))
    run_topn(w, Kh, Vh, lens, N)


@pytest.mark.parametrize("name,N", [("llama1b_32k", 1024), ("tiny_f32", 64), ("qwen1p5b_128k", 2048)])
def test_topn_on_the_workloads(name, N):
    """At the workloads' full sizes: caches filled on the device by the
    generator's twin, rows regenerated on the host for the checks."""
    w = synth.WORKLOADS[name]
    lens = synth.seq_lens(w)
    dt = torch.float32 if w.dtype == synth.F32 else torch.int16
    K = torch.empty(w.B, w.h_k, w.l_kv, w.d, dtype=dt, device="cuda")
    V = torch.empty(w.B, w.h_v, w.l_kv, w.d, dtype=dt, device="cuda")
    sdev.fill(K, w, 0, "K")
    sdev.fill(V, w, 0, "V")
    check_topn(w, K, V, w.l_kv, lens, N, SynthRows(w, 0))
    del K, V
    torch.cuda.empty_cache()
