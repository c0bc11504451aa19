"""GPU parity of the closed-form key merge (saga_merge_keys) against the
float64 oracle (oracle/key_merge.py: Eq. 13 from explicit logits, Eq. 15 with
numpy's pseudoinverse, Theorem 4.2 by enumeration).

Tolerance. The inputs are exact bf16 values. The GPU forms the query Gram
matrices S_r from exact bf16 products accumulated in fp32, and the key Gram
matrix C = K^T K from K = X W^T (fp32 accumulation) split into bf16 hi + lo
parts, with the lo.lo product dropped (at most 2^-18 of |K_a K_b|); the
per-pair algebra then runs in float64. The resulting error of w(a, b) scales
with E_ab = sum over r in {a, b} of trace(S_r K_r^T K_r), the Eq. (13) loss of
M = 0, and a float64 emulation of these roundings on the host gives
|dw| / E_ab near 2e-6 on every workload here: the bound below is 2e-5 E_ab.
The merged projection W_S is compared in relative Frobenius norm, also at
2e-5 (the emulation: 1e-7 with float64 eigenvectors at d = 64, 2e-6 with the
float32 eigenvectors of the d = 128 kernel). The pairing is an argmin over
the weights, so it is checked in the GPU's own precision: it is a perfect
matching of minimal total under the GPU's weights (the oracle's enumeration
run on them), and it equals the oracle's pairing, whose margin over the next
best pairing is far above the weight tolerance on these inputs.
"""
import networkx as nx
import numpy as np
import pytest
import torch

import synth
from oracle import key_merge as km
from synth import merge_workload as mw

pytestmark = pytest.mark.gpu

TOL = 2e-5
RCOND = 1e-6


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def run_gpu(saga, w, stored=None):
    Xb, Wb, Qb = stored if stored is not None else mw.merge_inputs(w)
    ms = saga.merge_shape(w.T, w.d_model, w.h_q, w.h_k, w.d)
    ws = saga.MergeWorkspace(ms)
    X, W, Q = to_dev(Xb), to_dev(Wb), to_dev(Qb)
    wout = torch.full((w.h_k, w.h_k), float("nan"), dtype=torch.float64, device="cuda")
    pairs = torch.full((w.h_k // 2, 2), -1, dtype=torch.int32, device="cuda")
    total = torch.zeros(1, dtype=torch.float64, device="cuda")
    W_S = torch.full((w.h_k // 2 * w.d, w.d_model), float("nan"), dtype=torch.float32,
                     device="cuda")
    saga.merge_keys(ms, X, W, Q, RCOND, wout, pairs, W_S, ws, total=total)
    assert saga.read_device_error(ws) == 0
    return ((Xb, Wb, Qb), wout.cpu().numpy(), [tuple(p) for p in pairs.cpu().tolist()],
            float(total.item()), W_S.cpu().numpy())


def energies(X, W, Q, w):
    """E_ab scale: per key head r, sum over its query heads of ||Q^j K_r^T||_F^2."""
    d, G = w.d, w.h_q // w.h_k
    e = np.zeros(w.h_k)
    for r in range(w.h_k):
        K = X @ W[r * d:(r + 1) * d].T
        Cr = K.T @ K
        for j in range(r * G, (r + 1) * G):
            Qj = Q[:, j * d:(j + 1) * d]
            e[r] += float(np.sum((Qj.T @ Qj) * Cr))
    return e


def check_pairing(w_gpu, pairs, total, n):
    assert sorted(x for p in pairs for x in p) == list(range(n))
    assert all(a < b for a, b in pairs) and pairs == sorted(pairs)
    assert total == km.matching_total(w_gpu, pairs)          # the DP's summation order
    if n <= 10:
        _, best = km.min_weight_perfect_matching(w_gpu)      # the decision, in the GPU's weights
        assert total == best


def check_w_s(W_S, X, W, Q, w, pairs):
    S = km.query_gram(Q, w.h_q, w.h_k, w.d)
    d = w.d
    for i, (a, b) in enumerate(pairs):
        M = km.merged_projection(km.key_block(W, a, d), km.key_block(W, b, d), S[a], S[b], RCOND)
        got = W_S[i * d:(i + 1) * d].astype(np.float64)
        err = np.linalg.norm(got - M.T) / np.linalg.norm(M)
        assert err <= TOL, (i, a, b, err)


@pytest.mark.parametrize("name", ["merge_tiny", "merge_tail_g1", "merge_tiny_d128",
                                  "merge_rank_deficient", "merge_wide16"])
def test_merge_matches_oracle(gpu_lib, name):
    w = mw.MERGE_WORKLOADS[name]
    stored, w_gpu, pairs, total, W_S = run_gpu(gpu_lib, w)
    X, W, Q = (synth.widen(a) for a in stored)
    n = w.h_k
    assert np.array_equal(w_gpu, w_gpu.T) and np.all(np.diag(w_gpu) == 0.0)
    ref_w, _ = km.pair_weights(X, W, Q, w.h_q, n, w.d, RCOND)
    if n <= 10:
        ref_pairs, _ = km.min_weight_perfect_matching(ref_w)
    else:                       # 15!! matchings at n = 16: networkx's blossom instead
        G = nx.Graph()
        for a in range(n):
            for b in range(a + 1, n):
                G.add_edge(a, b, weight=float(ref_w[a, b]))
        ref_pairs = sorted(tuple(sorted(e)) for e in nx.min_weight_matching(G))
    e = energies(X, W, Q, w)
    for a in range(n):
        for b in range(a + 1, n):
            assert abs(w_gpu[a, b] - ref_w[a, b]) <= TOL * (e[a] + e[b]), (a, b)
    check_pairing(w_gpu, pairs, total, n)
    assert pairs == ref_pairs == mw.planted_pairs(w)
    check_w_s(W_S, X, W, Q, w, pairs)
    if w.d_eff is not None:
        # query columns >= d_eff are zero: the pseudoinverse leaves those
        # output columns of every merged head exactly zero
        for i in range(n // 2):
            assert np.all(W_S[i * w.d + w.d_eff:(i + 1) * w.d] == 0.0)


@pytest.mark.parametrize("name", ["llama1b_merge_8k", "qwen1p5b_merge_8k"])
def test_merge_full_size_sampled(gpu_lib, name):
    """Model-sized calibration sets: every weight the GPU reports for the
    planted pairs and two others (Eq. 13 from explicit 8192 x 8192 logit
    blocks in the oracle), the pairing, and every merged head."""
    w = mw.MERGE_WORKLOADS[name]
    stored, w_gpu, pairs, total, W_S = run_gpu(gpu_lib, w)
    X, W, Q = (synth.widen(a) for a in stored)
    n = w.h_k
    planted = mw.planted_pairs(w)
    sample = planted[:2] + [p for p in [(0, 1), (0, 2), (1, 2)] if p not in planted and p[1] < n][:2]
    ref_w, _ = km.pair_weights(X, W, Q, w.h_q, n, w.d, RCOND, pairs=sample)
    e = energies(X, W, Q, w)
    for a, b in sample:
        assert abs(w_gpu[a, b] - ref_w[a, b]) <= TOL * (e[a] + e[b]), (a, b)
    check_pairing(w_gpu, pairs, total, n)
    assert pairs == planted
    check_w_s(W_S, X, W, Q, w, pairs)


def test_merge_is_deterministic(gpu_lib):
    w = mw.MERGE_WORKLOADS["merge_tail_g1"]
    stored = mw.merge_inputs(w)
    _, w1, p1, t1, s1 = run_gpu(gpu_lib, w, stored)
    _, w2, p2, t2, s2 = run_gpu(gpu_lib, w, stored)
    assert np.array_equal(w1, w2) and p1 == p2 and t1 == t2 and np.array_equal(s1, s2)
