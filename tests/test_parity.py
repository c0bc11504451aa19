"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

The five workloads run at their full sizes in the launch configuration the
benchmark times (one call per layer, the same shape); outputs are checked on
every row for the single-layer workloads and on sampled (sequence, key-head
group) rows for the 16-layer stack and the ragged batch. Small cases cover the
edges: ragged tails, empty sequences, empty selections, N >= l_kv, ties,
strided caches, every kernel instantiation and the device error word.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_decode_attention_step_b200 as saga
import synth
from synth import device as sdev

from gpu_harness import (Chain, HostRows, SynthRows, check_row, dev_dtype, rel_err, to_dev,
                         OUT_TOL)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(gpu_lib):
    import os
    if not os.path.exists(sdev.LIB_PATH):
        sdev.build()
    return gpu_lib


def saga_shape(w, cap=None, max_l=None, h_k=None, h_v=None):
    cap = w.l_kv if cap is None else cap
    return saga.shape(w.B, w.h_q, w.h_k if h_k is None else h_k, w.h_v if h_v is None else h_v,
                      w.d, w.dtype, cap, cap if max_l is None else max_l)


def dev_cache(w, layer, kind, heads, cap):
    t = torch.empty(w.B, heads, cap, w.d, dtype=dev_dtype(w), device="cuda")
    sdev.fill(t, w, layer, kind)
    return t


def run_chain(w, shp, K, V, lens, rows, steps, groups, layer=0, N=None, R=None):
    """Run `steps` steps and check the rows of the (b, kh) groups given."""
    N = w.N if N is None else N
    R = w.R if R is None else R
    qs = synth.queries(w, layer, steps)
    q64 = synth.widen(qs)
    ch = Chain(shp, K, V, lens, N)
    G = w.h_q // w.h_k
    tau_o = {}
    for t in range(steps):
        refresh = t % R == 0
        rec = ch.step(to_dev(qs[t]), refresh)
        for (b, kh) in groups:
            L = int(lens[b])
            krow = rows.k_row(b, kh, L)
            for j in range(kh * G, (kh + 1) * G):
                tau_o[(b, j)] = check_row(rec, q64[t, b, j], krow, rows, b, j, w.h_q, w.h_v, L,
                                          w.d, N, refresh, w.dtype, tau_o.get((b, j)))
    return ch


# ---------------------------------------------------------------------------
# single-layer workloads, every row, every step
# ---------------------------------------------------------------------------
def test_tiny_f32_chain():
    w = synth.WORKLOADS["tiny_f32"]
    lens = synth.seq_lens(w)
    Kh = synth.cache(w, 0, "K", w.h_k)
    Vh = synth.cache(w, 0, "V", w.h_v)
    rows = HostRows(synth.widen(Kh), synth.widen(Vh))
    groups = [(b, kh) for b in range(w.B) for kh in range(w.h_k)]
    run_chain(w, saga_shape(w), to_dev(Kh), to_dev(Vh), lens, rows, w.steps, groups)


def test_llama1b_32k_chain():
    w = synth.WORKLOADS["llama1b_32k"]
    lens = synth.seq_lens(w)
    K = dev_cache(w, 0, "K", w.h_k, w.l_kv)
    V = dev_cache(w, 0, "V", w.h_v, w.l_kv)
    groups = [(0, 0), (0, 1)]
    run_chain(w, saga_shape(w), K, V, lens, SynthRows(w, 0), w.steps, groups)


def test_qwen1p5b_128k_chain():
    w = synth.WORKLOADS["qwen1p5b_128k"]
    lens = synth.seq_lens(w)
    K = dev_cache(w, 0, "K", w.h_k, w.l_kv)
    V = dev_cache(w, 0, "V", w.h_v, w.l_kv)
    run_chain(w, saga_shape(w), K, V, lens, SynthRows(w, 0), w.steps, [(0, 0)])


# ---------------------------------------------------------------------------
# the 16-layer batch-8 stack at 128K, as the benchmark launches it
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("layer", [0, 15])
def test_stack_layer_full_size(layer):
    w = synth.WORKLOADS["llama1b_stack16_b8_128k"]
    lens = synth.seq_lens(w)
    K = dev_cache(w, layer, "K", w.h_k, w.l_kv)
    V = dev_cache(w, layer, "V", w.h_v, w.l_kv)
    # three steps at R = 2: refresh, plain step, refresh again
    groups = [(0, 0), (5, 1), (7, 0)]
    run_chain(w, saga_shape(w), K, V, lens, SynthRows(w, layer), 3, groups, layer=layer, R=2)
    del K, V
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# the calls the benchmark times (no selection mask, no count, scores kept in
# the workspace) against the checked calls, bit for bit
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,layer,groups", [
    ("llama1b_stack16_b8_128k", 3, [(2, 1), (6, 0)]),
    ("qwen1p5b_128k", 0, [(0, 0)]),
    ("llama1b_32k", 0, [(0, 1)])])
def test_timed_calls_equal_checked_calls_bitwise(name, layer, groups):
    """One refresh and the plain steps after it, called exactly as the
    benchmark calls them (sel_mask, sel_count and scores all NULL), must give
    the same thresholds and outputs, bit for bit, as the same calls with the
    selection mask, count and score dump the parity checks read; the checked
    run is then compared with the oracle row by row."""
    w = synth.WORKLOADS[name]
    lens = synth.seq_lens(w)
    K = dev_cache(w, layer, "K", w.h_k, w.l_kv)
    V = dev_cache(w, layer, "V", w.h_v, w.l_kv)
    shp = saga_shape(w)
    steps = 3
    qs = synth.queries(w, layer, steps)
    q64 = synth.widen(qs)
    l = torch.from_numpy(lens).cuda()
    ws = saga.Workspace(shp, w.N)
    tau = torch.zeros(w.B, w.h_q, dtype=torch.float32, device="cuda")
    out = torch.zeros(w.B, w.h_q, w.d, dtype=torch.float32, device="cuda")
    ch = Chain(shp, K, V, lens, w.N)
    rows = SynthRows(w, layer)
    G = w.h_q // w.h_k
    tau_o = {}
    for t in range(steps):
        q = to_dev(qs[t])
        refresh = t == 0
        if refresh:
            saga.refresh_threshold(shp, q, K, l, w.N, tau, ws, V=V, out=out)
        else:
            saga.decode_step(shp, q, K, V, l, tau, out, ws)
        rec = ch.step(q, refresh)
        assert saga.read_device_error(ws) == 0
        np.testing.assert_array_equal(tau.cpu().numpy().view(np.uint32), rec.tau.view(np.uint32))
        np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), rec.out.view(np.uint32))
        for (b, kh) in groups:
            L = int(lens[b])
            krow = rows.k_row(b, kh, L)
            for j in range(kh * G, (kh + 1) * G):
                tau_o[(b, j)] = check_row(rec, q64[t, b, j], krow, rows, b, j, w.h_q, w.h_v, L,
                                          w.d, w.N, refresh, w.dtype, tau_o.get((b, j)))
    del K, V
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# ragged batch, refresh every step, N swept
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def ragged_caches():
    w = synth.WORKLOADS["ragged_refresh_b16"]
    K = dev_cache(w, 0, "K", w.h_k, w.l_kv)
    V = dev_cache(w, 0, "V", w.h_v, w.l_kv)
    yield w, K, V, SynthRows(w, 0)
    del K, V
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N", [256, 1024, 4096, 8192])
def test_ragged_refresh_full_size(ragged_caches, N):
    w, K, V, rows = ragged_caches
    lens = synth.seq_lens(w)
    b_short, b_long = int(np.argmin(lens)), int(np.argmax(lens))
    groups = [(b_short, 0), (b_short, 1), (b_long, 1)]
    run_chain(w, saga_shape(w), K, V, lens, rows, 2, groups, N=N)


# ---------------------------------------------------------------------------
# dense GQA baseline
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,samples", [("llama1b_32k", [(0, 0), (0, 5)]),
                                          ("qwen1p5b_128k", [(0, 1)]),
                                          ("llama1b_stack16_b8_128k", [(3, 2)])])
def test_dense_gqa_matches_oracle(name, samples):
    w = synth.WORKLOADS[name]
    h = w.dense_hkv
    lens = synth.seq_lens(w)
    K = dev_cache(w, 0, "KD", h, w.l_kv)
    V = dev_cache(w, 0, "VD", h, w.l_kv)
    shp = saga_shape(w, h_k=h, h_v=h)
    ws = saga.Workspace(shp)
    qs = synth.queries(w, 0, 1)
    out = torch.zeros(w.B, w.h_q, w.d, dtype=torch.float32, device="cuda")
    l = torch.from_numpy(lens).cuda()
    saga.gqa_dense_decode(shp, to_dev(qs[0]), K, V, l, out, ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    q64 = synth.widen(qs[0])
    G = w.h_q // h
    for (b, kvh) in samples:
        L = int(lens[b])
        Kr = synth.widen(synth.cache_rows(w, 0, "KD", b, kvh, 0, L))
        Vr = synth.widen(synth.cache_rows(w, 0, "VD", b, kvh, 0, L))
        for j in range(kvh * G, (kvh + 1) * G):
            A = Kr @ q64[b, j] / np.sqrt(w.d)
            ref = orc.sparse_attend(A, Vr, np.arange(L))
            assert rel_err(o[b, j].astype(np.float64), ref) <= OUT_TOL[w.dtype]
    del K, V
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# SAGA full attention (asymmetric heads, every position): the ablation arm
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,samples", [("tiny_f32", [(0, 0), (0, 3)]),
                                          ("llama1b_32k", [(0, 0), (0, 13), (0, 31)]),
                                          ("qwen1p5b_128k", [(0, 2), (0, 11)]),
                                          ("llama1b_stack16_b8_128k", [(5, 6), (7, 29)])])
def test_saga_full_matches_oracle(name, samples):
    w = synth.WORKLOADS[name]
    lens = synth.seq_lens(w)
    K = dev_cache(w, 0, "K", w.h_k, w.l_kv)
    V = dev_cache(w, 0, "V", w.h_v, w.l_kv)
    shp = saga_shape(w)
    ws = saga.Workspace(shp)
    qs = synth.queries(w, 0, 1)
    out = torch.zeros(w.B, w.h_q, w.d, dtype=torch.float32, device="cuda")
    l = torch.from_numpy(lens).cuda()
    saga.dense_decode(shp, to_dev(qs[0]), K, V, l, out, ws)
    torch.cuda.synchronize()
    assert saga.read_device_error(ws) == 0
    o = out.cpu().numpy()
    q64 = synth.widen(qs[0])
    for (b, j) in samples:
        L = int(lens[b])
        kh = orc.key_head(j, w.h_q, w.h_k)
        vh = orc.value_head(j, w.h_q, w.h_v)
        Kr = synth.widen(synth.cache_rows(w, 0, "K", b, kh, 0, L))
        Vr = synth.widen(synth.cache_rows(w, 0, "V", b, vh, 0, L))
        A = Kr @ q64[b, j] / np.sqrt(w.d)
        ref = orc.sparse_attend(A, Vr, np.arange(L))
        assert rel_err(o[b, j].astype(np.float64), ref) <= OUT_TOL[w.dtype]
    del K, V
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# edge cases on small host-generated inputs
# ---------------------------------------------------------------------------
def small_case(dtype, B, h_q, h_k, h_v, d, cap, seed):
    w = synth.Workload("edge", dtype, B=B, h_q=h_q, h_k=h_k, h_v=h_v, d=d, l_kv=cap, N=1,
                       R=1, steps=1, seed=seed)
    lens = np.full(B, cap, dtype=np.int32)
    Kh = synth.cache(w, 0, "K", h_k, cap, lens)
    Vh = synth.cache(w, 0, "V", h_v, cap, lens)
    return w, Kh, Vh


@pytest.mark.parametrize("dtype,d,h_q,h_k,h_v", [
    (synth.F32, 64, 4, 1, 2), (synth.F32, 128, 16, 1, 4), (synth.F32, 64, 8, 1, 8),
    (synth.BF16, 64, 32, 2, 8), (synth.BF16, 128, 12, 1, 4), (synth.BF16, 128, 8, 2, 4),
    (synth.BF16, 64, 16, 4, 4), (synth.BF16, 64, 4, 4, 4), (synth.BF16, 128, 16, 1, 16)])
def test_ragged_lengths_every_instantiation(dtype, d, h_q, h_k, h_v):
    cap = 1300
    w, Kh, Vh = small_case(dtype, 5, h_q, h_k, h_v, d, cap, seed=77 + d + h_q)
    lens = np.array([0, 1, 255, 1027, 1300], dtype=np.int32)
    rows = HostRows(synth.widen(Kh), synth.widen(Vh))
    shp = saga.shape(5, h_q, h_k, h_v, d, dtype, cap)
    groups = [(b, kh) for b in range(5) for kh in range(h_k)]
    for N in (1, 7, 256):
        run_chain(w, shp, to_dev(Kh), to_dev(Vh), lens, rows, 3, groups, N=N, R=2)


def test_n_at_least_length_is_dense():
    w, Kh, Vh = small_case(synth.BF16, 2, 16, 2, 4, 64, 700, seed=5)
    lens = np.array([700, 333], dtype=np.int32)
    shp = saga.shape(2, 16, 2, 4, 64, synth.BF16, 700)
    ch = Chain(shp, to_dev(Kh), to_dev(Vh), lens, N=700)
    qs = synth.queries(w, 0, 1, B=2, h_q=16)
    rec = ch.step(to_dev(qs[0]), refresh=True)
    assert np.all(np.isneginf(rec.tau))
    ref = orc.dense_attend(synth.widen(qs[0]), synth.widen(Kh), synth.widen(Vh), lens)
    for b in range(2):
        for j in range(16):
            assert rec.cnt[b, j] == lens[b]
            assert rel_err(rec.out[b, j].astype(np.float64), ref[b, j]) <= 2e-3


def test_stale_threshold_gives_empty_selection():
    w, Kh, Vh = small_case(synth.F32, 1, 4, 1, 2, 64, 512, seed=6)
    shp = saga.shape(1, 4, 1, 2, 64, synth.F32, 512)
    ch = Chain(shp, to_dev(Kh), to_dev(Vh), [512], N=8)
    ch.tau.fill_(1e30)
    qs = synth.queries(w, 0, 1, B=1, h_q=4)
    rec = ch.step(to_dev(qs[0]), refresh=False)
    assert np.all(rec.cnt == 0) and np.all(rec.out == 0) and np.all(rec.mask[..., :512] == 0)


def test_ties_keep_every_tied_entry():
    # duplicate key rows: tied scores at the threshold are all kept
    w, Kh, Vh = small_case(synth.BF16, 1, 16, 2, 4, 64, 600, seed=7)
    Kh[:, :, 300:400] = Kh[:, :, 100:200]
    Kh[:, :, 500:600] = Kh[:, :, 100:200]
    rows = HostRows(synth.widen(Kh), synth.widen(Vh))
    shp = saga.shape(1, 16, 2, 4, 64, synth.BF16, 600)
    groups = [(0, 0), (0, 1)]
    lens = np.array([600], dtype=np.int32)
    for N in (1, 2, 3, 50, 299):
        ch = run_chain(w, shp, to_dev(Kh), to_dev(Vh), lens, rows, 2, groups, N=N, R=1)


def test_strided_caches_and_debug_scores():
    # heads padded to a larger capacity, max_l_kv below cap
    w, Kh, Vh = small_case(synth.BF16, 2, 32, 2, 8, 64, 1500, seed=8)
    capx = 2048
    Kx = np.zeros((2, 2, capx, 64), np.uint16); Kx[:, :, :1500] = Kh
    Vx = np.zeros((2, 8, capx, 64), np.uint16); Vx[:, :, :1500] = Vh
    shp = saga.shape(2, 32, 2, 8, 64, synth.BF16, capx, 1500)
    lens = np.array([1500, 999], dtype=np.int32)
    rows = HostRows(synth.widen(Kh), synth.widen(Vh))
    ch = run_chain(w, shp, to_dev(Kx), to_dev(Vx), lens, rows, 3, [(0, 0), (1, 1)], N=33, R=2)
    # the score dump entry point reproduces the refresh's own rows bit for bit
    qs = synth.queries(w, 0, 1)
    q = to_dev(qs[0])
    rec = ch.step(q, refresh=True)
    dump = torch.zeros(2, 32, 1500, dtype=torch.float32, device="cuda")
    saga.debug_scores(shp, q, ch.K, ch.l, dump, ch.ws)
    torch.cuda.synchronize()
    dmp = dump.cpu().numpy()
    for b in range(2):
        L = lens[b]
        np.testing.assert_array_equal(dmp[b, :, :L].view(np.uint32),
                                      rec.scores[b, :, :L].view(np.uint32))


def test_device_error_word_on_bad_lengths():
    w, Kh, Vh = small_case(synth.F32, 3, 4, 1, 2, 64, 256, seed=9)
    shp = saga.shape(3, 4, 1, 2, 64, synth.F32, 256)
    ws = saga.Workspace(shp, 4)
    q = to_dev(synth.queries(w, 0, 1, B=3, h_q=4)[0])
    l = torch.tensor([-5, 1000, 100], dtype=torch.int32, device="cuda")
    tau = torch.zeros(3, 4, device="cuda")
    out = torch.zeros(3, 4, 64, device="cuda")
    cnt = torch.zeros(3, 4, dtype=torch.int32, device="cuda")
    saga.refresh_threshold(shp, q, to_dev(Kh), l, 4, tau, ws, V=to_dev(Vh), out=out,
                           sel_count=cnt)
    flags = saga.read_device_error(ws)
    assert flags == saga.DEVERR_LKV_NEGATIVE | saga.DEVERR_LKV_TOO_LONG
    assert saga.read_device_error(ws) == 0          # reading clears it
    c = cnt.cpu().numpy()
    assert np.all(c[0] == 0) and np.all(c[1] == 4) and np.all(c[2] == 4)
    assert np.all(out.cpu().numpy()[0] == 0)
