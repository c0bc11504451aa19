"""Pins for the float64 oracle, each against something other than the oracle.

  * torch's scaled_dot_product_attention (float64, CPU) for Eq. (2-4) and the
    GQA head grouping;
  * the counting definition of the N-th largest, by brute force;
  * torch.topk + torch.softmax for exact top-N attention, Eq. (6)+(7);
  * a hand-derived worked example (tests/golden/hand_example.json);
  * invariants: exactly N kept on a refresh without ties, joint permutation
    of positions, N = 1, convex hull, monotone threshold in N, empty cases.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(rng, B=2, h_q=8, h_k=2, h_v=4, d=16, L=40, distinct=True):
    q = rng.standard_normal((B, h_q, d))
    K = rng.standard_normal((B, h_k, L, d))
    V = rng.standard_normal((B, h_v, L, d))
    return q, K, V


def sdpa_dense(q, K, V, l):
    """torch float64 SDPA on positions < l, with K expanded to V's head count
    by repeat_interleave and the query groups handled by enable_gqa."""
    h_k, h_v = K.shape[1], V.shape[1]
    Kx = torch.from_numpy(K[:, :, :l]).repeat_interleave(h_v // h_k, dim=1)
    Vx = torch.from_numpy(V[:, :, :l])
    qx = torch.from_numpy(q)[:, :, None, :]
    o = F.scaled_dot_product_attention(qx, Kx, Vx, enable_gqa=True)
    return o[:, :, 0, :].numpy()


def test_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    q = np.array(g["q"], float)[None]
    K = np.array(g["K"], float)[None]
    V = np.array(g["V"], float)[None]
    l = np.array([g["l_kv"]])
    A = orc.scores(q, K, l)[0]
    np.testing.assert_array_equal(A, np.array(g["expect_scores"], float))
    tau = orc.refresh(q, K, l, g["N"])
    np.testing.assert_array_equal(tau[0], g["expect_tau"])
    sel, out = orc.decode_step(q, K, V, l, tau)
    for j in range(2):
        assert list(sel[0][j]) == g["expect_sel"][j]
    np.testing.assert_allclose(out[0], np.array(g["expect_out"]), rtol=0, atol=1e-15)
    tc = g["tie_case"]
    t3 = orc.nth_largest(A[tc["head"]], tc["N"])
    assert t3 == tc["expect_tau"]
    assert list(orc.select(A[tc["head"]], t3)) == tc["expect_sel"]
    dense = orc.dense_attend(q, K, V, l)
    np.testing.assert_allclose(dense[0, 0], g["dense_head0_expect_out"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("h_q,h_kv", [(4, 4), (8, 2), (12, 2), (32, 8), (4, 1)])
def test_dense_matches_sdpa(h_q, h_kv):
    rng = np.random.default_rng(h_q * 100 + h_kv)
    q, K, V = rand_case(rng, B=2, h_q=h_q, h_k=h_kv, h_v=h_kv, d=16, L=37)
    l = np.array([37, 37])
    ours = orc.dense_attend(q, K, V, l)
    ref = sdpa_dense(q, K, V, 37)
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("h_q,h_k,h_v", [(4, 1, 2), (32, 2, 8), (12, 1, 4), (8, 2, 2)])
def test_saga_all_selected_is_dense(h_q, h_k, h_v):
    """N >= l_kv keeps everything (tau = -inf): the step is dense attention,
    checked against SDPA with K broadcast to the value heads."""
    rng = np.random.default_rng(7 + h_q)
    L = 29
    q, K, V = rand_case(rng, B=2, h_q=h_q, h_k=h_k, h_v=h_v, d=8, L=L)
    l = np.array([L, L])
    tau = orc.refresh(q, K, l, N=L)
    assert np.all(tau == -np.inf)
    _, out = orc.decode_step(q, K, V, l, tau)
    np.testing.assert_allclose(out, sdpa_dense(q, K, V, L), rtol=1e-12, atol=1e-13)


def brute_nth(row, N):
    """The value v of the row with #{x > v} < N <= #{x >= v} (counting only)."""
    for v in row:
        gt = sum(1 for x in row if x > v)
        ge = sum(1 for x in row if x >= v)
        if gt < N <= ge:
            return v
    raise AssertionError("no such value")


def test_nth_largest_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(300):
        L = int(rng.integers(1, 40))
        # small integer values force many ties
        row = rng.integers(-4, 5, size=L).astype(float) * 0.5
        N = int(rng.integers(1, L + 3))
        t = orc.nth_largest(row, N)
        if N >= L:
            assert t == -np.inf
        else:
            assert t == brute_nth(list(row), N)


def test_nth_largest_f32_total_order():
    rng = np.random.default_rng(4)
    for trial in range(300):
        L = int(rng.integers(1, 50))
        row = (rng.integers(-3, 4, size=L) * 0.25).astype(np.float32)
        # sprinkle signed zeros
        z = rng.random(L) < 0.3
        row[z] = np.where(rng.random(z.sum()) < 0.5, np.float32(-0.0), np.float32(0.0))
        N = int(rng.integers(1, L + 2))
        t = orc.nth_largest_f32(row, N)
        if N >= L:
            assert np.isneginf(t)
            continue
        # brute force under totalOrder: compare (value, sign-of-zero) pairs
        def tot(x):
            return (float(x), 0 if np.signbit(x) else 1)
        v = brute_nth([tot(x) for x in row], N)
        assert tot(t) == v
        assert t.view(np.uint32) in row.view(np.uint32)


def test_exactly_n_on_refresh_without_ties():
    rng = np.random.default_rng(5)
    q, K, V = rand_case(rng, B=3, h_q=8, h_k=2, h_v=4, d=16, L=200)
    l = np.array([200, 150, 77])
    for N in (1, 5, 64, 76):
        tau = orc.refresh(q, K, l, N)
        sel, _ = orc.decode_step(q, K, V, l, tau)
        for b in range(3):
            for j in range(8):
                assert len(sel[b][j]) == (N if N < l[b] else l[b])


def test_gqa_top_n_matches_torch_topk():
    """h_k = h_v and a fresh threshold: the step is exact top-N attention,
    Eq. (6) + (7), computed here with torch.topk and torch.softmax."""
    rng = np.random.default_rng(6)
    h_q, h, d, L, N = 8, 2, 16, 300, 17
    q, K, V = rand_case(rng, B=2, h_q=h_q, h_k=h, h_v=h, d=d, L=L)
    l = np.array([L, L])
    tau = orc.refresh(q, K, l, N)
    sel, out = orc.decode_step(q, K, V, l, tau)
    Kt, Vt, qt = torch.from_numpy(K), torch.from_numpy(V), torch.from_numpy(q)
    G = h_q // h
    for b in range(2):
        for j in range(h_q):
            a = (Kt[b, j // G] @ qt[b, j]) / d ** 0.5
            vals, idx = torch.topk(a, N)
            assert sorted(idx.tolist()) == list(sel[b][j])
            ref = torch.softmax(vals, 0) @ Vt[b, j // G, idx]
            np.testing.assert_allclose(out[b, j], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_n_equals_one_is_argmax_row():
    rng = np.random.default_rng(8)
    q, K, V = rand_case(rng, B=2, h_q=4, h_k=1, h_v=2, d=8, L=50)
    l = np.array([50, 31])
    tau = orc.refresh(q, K, l, 1)
    sel, out = orc.decode_step(q, K, V, l, tau)
    for b in range(2):
        for j in range(4):
            a = K[b, 0, :l[b]] @ q[b, j]
            t = int(np.argmax(a))
            assert list(sel[b][j]) == [t]
            np.testing.assert_array_equal(out[b, j], V[b, (j * 2) // 4, t])


def test_joint_permutation_invariance():
    rng = np.random.default_rng(9)
    q, K, V = rand_case(rng, B=1, h_q=8, h_k=2, h_v=4, d=16, L=120)
    l = np.array([120])
    tau = orc.refresh(q, K, l, 11)
    sel, out = orc.decode_step(q, K, V, l, tau)
    perm = rng.permutation(120)
    sel2, out2 = orc.decode_step(q, K[:, :, perm], V[:, :, perm], l, tau)
    np.testing.assert_allclose(out, out2, rtol=1e-12, atol=1e-14)
    for j in range(8):
        assert sorted(perm[sel2[0][j]].tolist()) == list(sel[0][j])


def test_convex_hull_and_monotone_tau():
    rng = np.random.default_rng(10)
    q, K, V = rand_case(rng, B=2, h_q=8, h_k=2, h_v=8, d=16, L=90)
    l = np.array([90, 60])
    prev = None
    for N in (1, 3, 10, 30, 59, 80):
        tau = orc.refresh(q, K, l, N)
        if prev is not None:
            assert np.all(tau <= prev)
        prev = tau
        sel, out = orc.decode_step(q, K, V, l, tau)
        for b in range(2):
            for j in range(8):
                rows = V[b, j, sel[b][j]]
                assert np.all(out[b, j] <= rows.max(0) + 1e-12)
                assert np.all(out[b, j] >= rows.min(0) - 1e-12)


def test_empty_selection_and_empty_sequence():
    rng = np.random.default_rng(11)
    q, K, V = rand_case(rng, B=2, h_q=4, h_k=1, h_v=2, d=8, L=20)
    l = np.array([20, 0])
    tau = np.full((2, 4), 1e9)           # a stale threshold above every score
    sel, out = orc.decode_step(q, K, V, l, tau)
    assert all(len(s) == 0 for sb in sel for s in sb)
    assert np.all(out == 0)
    tau = orc.refresh(q, K, l, 5)
    assert np.all(tau[1] == -np.inf)
    sel, out = orc.decode_step(q, K, V, l, tau)
    assert np.all(out[1] == 0) and all(len(s) == 0 for s in sel[1])


def test_chain_refreshes_on_schedule():
    rng = np.random.default_rng(12)
    q, K, V = rand_case(rng, B=1, h_q=4, h_k=1, h_v=2, d=8, L=64)
    qs = [q + 0.1 * t * rng.standard_normal(q.shape) for t in range(7)]
    l = np.array([64])
    taus, sels, outs = orc.decode_chain(qs, K, V, l, N=9, R=3)
    for t in range(7):
        r = t - t % 3
        np.testing.assert_array_equal(taus[t], orc.refresh(qs[r], K, l, 9))
        s, o = orc.decode_step(qs[t], K, V, l, taus[t])
        np.testing.assert_array_equal(outs[t], o)


# ---------------------------------------------------------------------------
# exact top-N (Eq. 6) with ties broken towards the lower position
# ---------------------------------------------------------------------------
def test_top_n_exact_brute_force_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(300):
        L = int(rng.integers(1, 40))
        row = rng.integers(-3, 4, size=L).astype(np.float64)   # many ties
        N = int(rng.integers(1, 50))
        ranked = sorted(range(L), key=lambda t: (-row[t], t))
        want = sorted(ranked[:min(N, L)])
        assert list(orc.top_n_exact(row, N)) == want


def test_top_n_exact_keeps_exactly_n():
    rng = np.random.default_rng(12)
    for trial in range(50):
        L = int(rng.integers(1, 200))
        row = np.round(rng.standard_normal(L), 1)            # ties at every threshold
        N = int(rng.integers(1, 250))
        assert orc.top_n_exact(row, N).size == min(N, L)


def test_top_n_exact_without_ties_is_the_refresh_selection():
    rng = np.random.default_rng(13)
    for trial in range(50):
        L = int(rng.integers(2, 500))
        row = rng.standard_normal(L)
        N = int(rng.integers(1, L))
        tau = orc.nth_largest(row, N)
        assert np.array_equal(orc.top_n_exact(row, N), orc.select(row, tau))


def test_topn_step_matches_atop_n_refresh_without_ties():
    rng = np.random.default_rng(14)
    B, h_q, h_k, h_v, d, L, N = 2, 8, 2, 4, 16, 90, 11
    q = rng.standard_normal((B, h_q, d))
    K = rng.standard_normal((B, h_k, L, d))
    V = rng.standard_normal((B, h_v, L, d))
    l = np.array([L, 57])
    sel_t, out_t = orc.topn_step(q, K, V, l, N)
    tau = orc.refresh(q, K, l, N)
    sel_a, out_a = orc.decode_step(q, K, V, l, tau)
    np.testing.assert_allclose(out_t, out_a, rtol=0, atol=1e-12)
    for b in range(B):
        for j in range(h_q):
            assert np.array_equal(sel_t[b][j], sel_a[b][j])


# ---------------------------------------------------------------------------
# KV-cache append and the growing-context decode loop
# ---------------------------------------------------------------------------
def test_append_then_attend_equals_concatenated_cache():
    rng = np.random.default_rng(15)
    B, h_q, h_k, h_v, d, cap = 2, 8, 2, 4, 16, 64
    l0 = np.array([20, 33])
    K = rng.standard_normal((B, h_k, cap, d))
    V = rng.standard_normal((B, h_v, cap, d))
    K2, V2, l = K, V, l0.copy()
    steps = 5
    kn = rng.standard_normal((steps, B, h_k, d))
    vn = rng.standard_normal((steps, B, h_v, d))
    for s_ in range(steps):
        K2, V2, l = orc.append(K2, V2, l, kn[s_], vn[s_])
    assert np.array_equal(l, l0 + steps)
    q = rng.standard_normal((B, h_q, d))
    got = orc.dense_attend(q, K2, V2, l)
    for b in range(B):
        Kc = np.concatenate([K[b, :, :l0[b]], np.transpose(kn[:, b], (1, 0, 2))], axis=1)
        Vc = np.concatenate([V[b, :, :l0[b]], np.transpose(vn[:, b], (1, 0, 2))], axis=1)
        for j in range(h_q):
            kh, vh = orc.key_head(j, h_q, h_k), orc.value_head(j, h_q, h_v)
            A = Kc[kh] @ q[b, j] / np.sqrt(d)
            w = np.exp(A - A.max())
            np.testing.assert_allclose(got[b, j], (w @ Vc[vh]) / w.sum(), rtol=1e-12, atol=1e-12)
    # positions before the append point and after it stay as they were
    for b in range(B):
        assert np.array_equal(K2[b, :, :l0[b]], K[b, :, :l0[b]])
        assert np.array_equal(K2[b, :, l0[b] + steps:], K[b, :, l0[b] + steps:])


def test_append_refuses_a_full_cache():
    K = np.zeros((1, 1, 4, 2)); V = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        orc.append(K, V, np.array([4]), np.ones((1, 1, 2)), np.ones((1, 1, 2)))
