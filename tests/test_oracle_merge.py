"""Pins for the float64 key-merge oracle, each against something other than
the oracle's own formulas.

  * a hand-worked two-head example and a four-node matching
    (tests/golden/merge_hand_example.json);
  * Lemma 4.1 against numpy's least-squares solver on the vectorised Eq. (13)
    problem (the minimum loss, and the minimum-norm minimiser when S is
    singular);
  * convexity: no perturbation of the Eq. (15) optimum lowers Eq. (13);
  * special cases: identical heads, identical query statistics, absent
    queries;
  * Theorem 4.2's matching against networkx's minimum-weight matching and
    against enumeration over all node orders;
  * the planted pairing of the synthetic calibration inputs is recovered.
"""
import itertools
import json
import os

import networkx as nx
import numpy as np
import pytest

import synth
from oracle import key_merge as km
from synth import merge_workload as mw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(rng, T=7, d_model=5, h_q=4, h_k=2, d=3):
    X = rng.standard_normal((T, d_model))
    W = rng.standard_normal((h_k * d, d_model))
    Q = rng.standard_normal((T, h_q * d))
    return X, W, Q


def lstsq_pair(X, W, Q, h_q, h_k, d, a, b):
    """Eq. (13) as one linear least-squares problem in the entries of M:
    residual (j, s, t) = sum_{i,c} Q^j[s,c] X[t,i] M[i,c] - (Q^j W_r^T X^T)[s,t]."""
    G = h_q // h_k
    rows, rhs = [], []
    for r in (a, b):
        W_r = W[r * d:(r + 1) * d].T
        for j in range(r * G, (r + 1) * G):
            Qj = Q[:, j * d:(j + 1) * d]
            A = np.einsum("sc,ti->stic", Qj, X).reshape(-1, X.shape[1] * d)
            rows.append(A)
            rhs.append((Qj @ W_r.T @ X.T).reshape(-1))
    A = np.concatenate(rows)
    y = np.concatenate(rhs)
    m, _, _, _ = np.linalg.lstsq(A, y, rcond=None)
    res = A @ m - y
    return m.reshape(X.shape[1], d), float(res @ res)


def test_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "merge_hand_example.json")))
    X, W, Q = (np.array(g[k], float) for k in ("X", "W_lin", "Q"))
    h_q, h_k, d = g["h_q"], g["h_k"], g["d"]
    S = km.query_gram(Q, h_q, h_k, d)
    np.testing.assert_array_equal(S[:, 0, 0], g["expect_S"])
    w, Ms = km.pair_weights(X, W, Q, h_q, h_k, d, rcond=1e-12)
    np.testing.assert_allclose(Ms[(0, 1)][:, 0], g["expect_M"], rtol=1e-15)
    assert w[0, 1] == pytest.approx(g["expect_loss_num"] / g["expect_loss_den"], rel=1e-14)
    pairs, total = km.min_weight_perfect_matching(np.array(g["matching_w"], float))
    assert [list(p) for p in pairs] == g["expect_pairs"]
    assert total == g["expect_total"]


@pytest.mark.parametrize("seed", range(6))
def test_lemma_matches_least_squares(seed):
    rng = np.random.default_rng(seed)
    h_q, h_k, d = 4, 2, 3
    X, W, Q = rand_problem(rng, h_q=h_q, h_k=h_k, d=d)
    w, Ms = km.pair_weights(X, W, Q, h_q, h_k, d, rcond=1e-12)
    M_ls, loss_ls = lstsq_pair(X, W, Q, h_q, h_k, d, 0, 1)
    assert w[0, 1] == pytest.approx(loss_ls, rel=1e-9)
    np.testing.assert_allclose(Ms[(0, 1)], M_ls, rtol=1e-9, atol=1e-12)


def test_lemma_rank_deficient_is_minimum_norm():
    """Only two calibration tokens per head group: S = S_a + S_b has rank 2 < d.
    With X of full column rank, Eq. (15) with the pseudoinverse is the
    minimum-norm minimiser, which is what lstsq returns."""
    rng = np.random.default_rng(11)
    h_q, h_k, d = 2, 2, 4
    X, W, Q = rand_problem(rng, T=6, d_model=5, h_q=h_q, h_k=h_k, d=d)
    Q[:, 0 * d + 2:0 * d + 4] = 0.0        # head 0 spans e0, e1 only
    Q[:, 1 * d + 2:1 * d + 4] = 0.0        # so does head 1
    w, Ms = km.pair_weights(X, W, Q, h_q, h_k, d, rcond=1e-12)
    M_ls, loss_ls = lstsq_pair(X, W, Q, h_q, h_k, d, 0, 1)
    assert w[0, 1] == pytest.approx(loss_ls, rel=1e-9)
    np.testing.assert_allclose(Ms[(0, 1)], M_ls, rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(Ms[(0, 1)][:, 2:], 0.0)


def test_optimum_is_not_improved_by_perturbation():
    rng = np.random.default_rng(5)
    h_q, h_k, d = 8, 4, 6
    X, W, Q = rand_problem(rng, T=40, d_model=12, h_q=h_q, h_k=h_k, d=d)
    w, Ms = km.pair_weights(X, W, Q, h_q, h_k, d, rcond=1e-12)
    for (a, b), M in Ms.items():
        for _ in range(5):
            E = rng.standard_normal(M.shape)
            for eps in (1e-3, 1e-1):
                assert km.pair_loss(X, W, Q, h_q, h_k, d, a, b, M + eps * E) >= w[a, b]


def test_special_cases():
    rng = np.random.default_rng(8)
    h_q, h_k, d = 4, 2, 3
    X, W, Q = rand_problem(rng, T=9, d_model=5, h_q=h_q, h_k=h_k, d=d)
    # identical key heads: nothing to lose
    Wi = W.copy()
    Wi[d:2 * d] = Wi[:d]
    w, Ms = km.pair_weights(X, Wi, Q, h_q, h_k, d, rcond=1e-12)
    np.testing.assert_allclose(Ms[(0, 1)], Wi[:d].T, rtol=1e-12, atol=1e-13)
    assert w[0, 1] == pytest.approx(0.0, abs=1e-18 + 1e-12 * np.sum(Q * Q))
    # both heads see the same query statistics: the plain average
    Qs = Q.copy()
    Qs[:, 2 * d:] = Q[:, :2 * d]           # heads 2, 3 (key head 1) copy heads 0, 1
    _, Ms = km.pair_weights(X, W, Qs, h_q, h_k, d, rcond=1e-12)
    np.testing.assert_allclose(Ms[(0, 1)], 0.5 * (W[:d].T + W[d:].T), rtol=1e-12)
    # head b has no queries: keep head a's projection, lose nothing
    Qz = Q.copy()
    Qz[:, 2 * d:] = 0.0
    w, Ms = km.pair_weights(X, W, Qz, h_q, h_k, d, rcond=1e-12)
    np.testing.assert_allclose(Ms[(0, 1)], W[:d].T, rtol=1e-12, atol=1e-13)
    assert abs(w[0, 1]) <= 1e-20 + 1e-24 * np.sum(Q * Q)


def test_perfect_matchings_enumeration():
    for n in (2, 4, 6, 8):
        ms = list(km.perfect_matchings(list(range(n))))
        assert len(ms) == int(np.prod(np.arange(n - 1, 0, -2)))      # (n-1)!!
        seen = set()
        for m in ms:
            flat = sorted(x for p in m for x in p)
            assert flat == list(range(n))
            assert all(a < b for a, b in m) and [p[0] for p in m] == sorted(p[0] for p in m)
            seen.add(tuple(m))
        assert len(seen) == len(ms)


def sym_weights(rng, n):
    w = rng.random((n, n))
    w = w + w.T
    np.fill_diagonal(w, 0.0)
    return w


@pytest.mark.parametrize("n", [2, 4, 6, 8, 10])
def test_matching_against_networkx(n):
    rng = np.random.default_rng(100 + n)
    for _ in range(4):
        w = sym_weights(rng, n)
        pairs, total = km.min_weight_perfect_matching(w)
        G = nx.Graph()
        for a in range(n):
            for b in range(a + 1, n):
                G.add_edge(a, b, weight=float(w[a, b]))
        ref = nx.min_weight_matching(G)
        ref_pairs = sorted(tuple(sorted(e)) for e in ref)
        assert pairs == ref_pairs
        assert total == pytest.approx(sum(w[a, b] for a, b in ref_pairs), rel=1e-12)


def test_matching_against_all_orders():
    """Every node order read two by two is a perfect matching; the best of
    them all is the minimum."""
    rng = np.random.default_rng(7)
    n = 8
    w = sym_weights(rng, n)
    best = min(sum(w[p[i], p[i + 1]] for i in range(0, n, 2))
               for p in itertools.permutations(range(n)))
    _, total = km.min_weight_perfect_matching(w)
    assert total == pytest.approx(best, rel=1e-12)


def test_odd_node_count_refused():
    with pytest.raises(ValueError):
        km.min_weight_perfect_matching(np.zeros((3, 3)))


@pytest.mark.parametrize("name", ["merge_tiny", "merge_tail_g1", "merge_tiny_d128",
                                  "merge_rank_deficient"])
def test_planted_pairs_recovered(name):
    w = mw.MERGE_WORKLOADS[name]
    X, W, Q = (synth.widen(a) for a in mw.merge_inputs(w))
    r = km.merge_keys(X, W, Q, w.h_q, w.h_k, w.d, rcond=1e-6)
    assert r["pairs"] == mw.planted_pairs(w)
    assert r["W_S"].shape == (w.h_k // 2 * w.d, w.d_model)
    # every planted pair loses less than any pairing across planted pairs
    planted = set(mw.planted_pairs(w))
    inside = max(r["w"][a, b] for a, b in planted)
    across = min(r["w"][a, b] for a in range(w.h_k) for b in range(a + 1, w.h_k)
                 if (a, b) not in planted)
    assert inside < across


def test_identical_pairs_keep_their_rows():
    """Teacher heads 0 = 2 and 1 = 3 exactly: the pairing is {(0, 2), (1, 3)}
    at zero loss, and the student's key projection is the teacher's rows of
    heads 0 and 1 in the linear layer's layout."""
    rng = np.random.default_rng(21)
    h_q, h_k, d = 8, 4, 3
    X, W, Q = rand_problem(rng, T=30, d_model=7, h_q=h_q, h_k=h_k, d=d)
    W[2 * d:3 * d] = W[0:d]
    W[3 * d:4 * d] = W[d:2 * d]
    r = km.merge_keys(X, W, Q, h_q, h_k, d, rcond=1e-12)
    assert r["pairs"] == [(0, 2), (1, 3)]
    np.testing.assert_allclose(r["W_S"], W[:2 * d], rtol=1e-11, atol=1e-12)
    assert r["total"] == pytest.approx(0.0, abs=1e-12 * np.sum(Q * Q) * np.sum(X * X))


def test_student_head_order():
    assert km.student_head_order([(0, 3), (1, 2)]) == [0, 3, 1, 2]
