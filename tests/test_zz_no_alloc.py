"""The allocation-free decode step (saga_decode_step_noalloc), for callers
that cannot allocate device memory: its output must equal the ordinary
saga_decode_step's on the same inputs, on two calls in a row (the second call
finds the first call's leftovers in the shared scratch array). This file is
named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_decode_attention_step_b200 as saga
import synth

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_step_twice():
    assert torch.cuda.is_available()
    saga.load()
    w = synth.Workload("noalloc", synth.BF16, B=2, h_q=16, h_k=2, h_v=4, d=64, l_kv=3000,
                       N=64, R=1, steps=3, seed=9090)
    lens = np.array([3000, 1777], dtype=np.int32)
    Kh = synth.cache(w, 0, "K", w.h_k, 3000, lens)
    Vh = synth.cache(w, 0, "V", w.h_v, 3000, lens)
    qs = synth.queries(w, 0, 3)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    K, V, l = dev(Kh), dev(Vh), torch.from_numpy(lens).cuda()
    shp = saga.shape(w.B, w.h_q, w.h_k, w.h_v, w.d, w.dtype, 3000)
    ws = saga.Workspace(shp, w.N)
    tau = torch.zeros(w.B, w.h_q, device="cuda")
    saga.refresh_threshold(shp, dev(qs[0]), K, l, w.N, tau, ws)
    for t in (1, 2):                       # two calls in a row
        q = dev(qs[t])
        ref = torch.zeros(w.B, w.h_q, w.d, device="cuda")
        ref_cnt = torch.zeros(w.B, w.h_q, dtype=torch.int32, device="cuda")
        saga.decode_step(shp, q, K, V, l, tau, ref, ws, sel_count=ref_cnt)
        out = torch.full((w.B, w.h_q, w.d), float("nan"), device="cuda")
        cnt = torch.full((w.B, w.h_q), -1, dtype=torch.int32, device="cuda")
        saga.decode_step_noalloc(shp, q, K, V, l, tau, out, sel_count=cnt)
        torch.cuda.synchronize()
        o, r = out.cpu().numpy(), ref.cpu().numpy()
        assert np.all(np.isfinite(o))
        err = np.max(np.abs(o - r), axis=-1) / np.maximum(np.max(np.abs(r), axis=-1), 1e-30)
        assert np.max(err) <= 2e-3, (t, np.max(err))
        np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt.cpu().numpy())


def test_noalloc_rejects_shapes_beyond_its_scratch():
    saga.load()
    # 64 sequences x 32 heads x 5 splits x 132 floats of split state: 5.4 MB
    big = saga.shape(64, 32, 2, 8, 128, synth.BF16, 1 << 20)
    fake = 1 << 40          # never dereferenced: the call is rejected first
    rc = saga.load().saga_decode_step_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake,
                                              fake, None, None)
    assert rc == saga.SAGA_ERR_WORKSPACE
