"""The key-merge routines the CUDA kernels run (csrc/merge_math.cuh), built for
the host with g++ and checked on the CPU:

  * the Jacobi ordering meets every index pair once per sweep;
  * the eigen-decomposition against numpy's eigvalsh, orthonormality and
    reconstruction (full rank, repeated and zero eigenvalues);
  * the per-pair stage (pseudoinverse, A_a and A_b, w = trace(D A_a S_b)) fed
    with float64 Gram matrices of the synthetic calibration inputs, against
    the oracle's Eq. (13) loss at the Eq. (15) optimum and its merged
    projection;
  * the subset programme of the matching against the oracle's enumeration
    (pairs and bit-identical totals, ties included) and networkx at n = 16.

The host build runs the device's loops on one thread in the same order, so
these are the device's results on exact inputs; the GPU tests then cover the
tensor-core Gram matrices that feed them.
"""
import ctypes
import os
import subprocess

import networkx as nx
import numpy as np
import pytest

import synth
from oracle import key_merge as km
from synth import merge_workload as mw

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "sparse_decode_attention_step_b200", "csrc")

D_P = ctypes.POINTER(ctypes.c_double)
I_P = ctypes.POINTER(ctypes.c_int32)


def dptr(a):
    return a.ctypes.data_as(D_P)


def iptr(a):
    return a.ctypes.data_as(I_P)


@pytest.fixture(scope="module")
def host(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("kmhost") / "libkmhost.so")
    subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-I", CSRC, "-o", out,
                    os.path.join(HERE, "merge_host_harness.cpp")], check=True)
    lib = ctypes.CDLL(out)
    lib.km_host_jacobi.argtypes = [ctypes.c_int, D_P, D_P]
    lib.km_host_jacobi.restype = ctypes.c_int
    lib.km_host_rounds.argtypes = [ctypes.c_int, I_P]
    lib.km_host_pair.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, D_P, D_P, D_P,
                                 ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                 D_P, I_P]
    lib.km_host_pair.restype = ctypes.c_double
    lib.km_host_match.argtypes = [ctypes.c_int, D_P, I_P, D_P]
    lib.km_host_merged.argtypes = [ctypes.c_int, ctypes.c_int, D_P, D_P, D_P, D_P, D_P]
    lib.km_host_pair_index.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.km_host_pair_index.restype = ctypes.c_int
    lib.km_host_pair_of.argtypes = [ctypes.c_int, ctypes.c_int, I_P]
    return lib


@pytest.mark.parametrize("d", [4, 8, 64, 128])
def test_rounds_meet_every_pair_once(host, d):
    out = np.zeros((d - 1, d // 2, 2), np.int32)
    host.km_host_rounds(d, iptr(out))
    seen = set()
    for r in range(d - 1):
        idx = sorted(out[r].reshape(-1).tolist())
        assert idx == list(range(d))                       # a round touches each index once
        for p, q in out[r]:
            assert p < q
            seen.add((int(p), int(q)))
    assert len(seen) == d * (d - 1) // 2


def psd(rng, d, rank=None, scale=None):
    G = rng.standard_normal((d, d if rank is None else rank))
    if scale is not None:
        G = G * scale
    return G @ G.T


@pytest.mark.parametrize("case", ["full64", "full128", "rank20", "repeated"])
def test_jacobi_against_eigvalsh(host, case):
    rng = np.random.default_rng({"full64": 1, "full128": 2, "rank20": 3, "repeated": 4}[case])
    if case == "full64":
        S = psd(rng, 64, scale=np.exp(rng.standard_normal(64)))
    elif case == "full128":
        S = psd(rng, 128)
    elif case == "rank20":
        S = psd(rng, 64, rank=20)
    else:
        Q, _ = np.linalg.qr(rng.standard_normal((64, 64)))
        lam = np.repeat([5.0, 2.0, 1.0, 0.5], 16)
        S = (Q * lam) @ Q.T
        S = 0.5 * (S + S.T)
    d = S.shape[0]
    A = S.copy()
    E = np.zeros_like(S)
    sweeps = host.km_host_jacobi(d, dptr(A), dptr(E))
    assert 1 <= sweeps < 40
    lam = np.diag(A).copy()
    ref = np.linalg.eigvalsh(S)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(np.sort(lam), ref, rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(E @ E.T, np.eye(d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(E.T @ np.diag(lam) @ E, S, rtol=0, atol=1e-12 * scale)


def gram_inputs(w):
    """Float64 Gram matrices of the calibration inputs, as the tensor-core
    stages would give them without rounding: S_r and C = K^T K, K = X W^T."""
    X, W, Q = (synth.widen(a) for a in mw.merge_inputs(w))
    d, G = w.d, w.h_q // w.h_k
    S = np.zeros((w.h_k, d, d))
    for r in range(w.h_k):
        for j in range(r * G, (r + 1) * G):
            Qj = Q[:, j * d:(j + 1) * d]
            S[r] += Qj.T @ Qj
    K = X @ W.T
    C = K.T @ K
    return X, W, Q, S, np.ascontiguousarray(C)


@pytest.mark.parametrize("name,vt_float,direct,rtol", [
    ("merge_tiny", 0, 1, 1e-9), ("merge_tiny", 0, 0, 1e-9), ("merge_tail_g1", 0, 1, 1e-9),
    ("merge_tiny_d128", 0, 0, 1e-9), ("merge_tiny_d128", 1, 0, 1e-5),
    ("merge_tiny_d128", 1, 1, 1e-9), ("merge_rank_deficient", 0, 1, 1e-9)])
def test_pair_stage_against_oracle(host, name, vt_float, direct, rtol):
    """Both ways to the pseudoinverse: the Gauss-Jordan inverse where it
    provably equals it (full-rank calibration sets), the Jacobi
    eigen-decomposition otherwise (forced with direct = 0, and taken by
    itself on the rank-deficient set)."""
    w = mw.MERGE_WORKLOADS[name]
    X, W, Q, S, C = gram_inputs(w)
    d, n = w.d, w.h_k
    ref_w, Ms = km.pair_weights(X, W, Q, w.h_q, n, d, rcond=1e-6)
    for a in range(n):
        for b in range(a + 1, n):
            Ag = np.zeros((2, d, d))
            sw = np.zeros(1, np.int32)
            got = host.km_host_pair(d, vt_float, direct, dptr(np.ascontiguousarray(S[a])),
                                    dptr(np.ascontiguousarray(S[b])), dptr(C), n * d, a, b,
                                    1e-6, dptr(Ag), iptr(sw))
            assert got == pytest.approx(ref_w[a, b], rel=rtol)
            if direct and w.d_eff is None:
                assert sw[0] == 0                      # full rank: the inverse was taken
            else:
                assert sw[0] >= 1                      # the eigen-decomposition ran
            out = np.zeros((d, w.d_model))
            Wa = np.ascontiguousarray(W[a * d:(a + 1) * d])
            Wb = np.ascontiguousarray(W[b * d:(b + 1) * d])
            host.km_host_merged(d, w.d_model, dptr(Wa), dptr(Wb), dptr(Ag[0]), dptr(Ag[1]),
                                dptr(out))
            ref = Ms[(a, b)].T
            err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
            assert err <= rtol


def host_match(host, w):
    n = w.shape[0]
    pairs = np.zeros((n // 2, 2), np.int32)
    total = np.zeros(1)
    host.km_host_match(n, dptr(np.ascontiguousarray(w, dtype=np.float64)), iptr(pairs),
                       dptr(total))
    return [tuple(int(v) for v in p) for p in pairs], float(total[0])


@pytest.mark.parametrize("n", [2, 4, 6, 8, 10])
def test_matching_programme_against_enumeration(host, n):
    rng = np.random.default_rng(300 + n)
    for trial in range(6):
        if trial % 2:
            w = rng.integers(1, 4, (n, n)).astype(float)    # many exact ties
        else:
            w = rng.random((n, n))
        w = np.triu(w, 1)
        w = w + w.T
        pairs, total = host_match(host, w)
        ref_pairs, ref_total = km.min_weight_perfect_matching(w)
        assert pairs == ref_pairs
        assert total == ref_total                            # same summation order


def test_matching_programme_sixteen_nodes(host):
    rng = np.random.default_rng(16)
    w = rng.random((16, 16))
    w = np.triu(w, 1)
    w = w + w.T
    pairs, total = host_match(host, w)
    assert sorted(x for p in pairs for x in p) == list(range(16))
    G = nx.Graph()
    for a in range(16):
        for b in range(a + 1, 16):
            G.add_edge(a, b, weight=float(w[a, b]))
    ref = sorted(tuple(sorted(e)) for e in nx.min_weight_matching(G))
    assert pairs == ref
    assert total == pytest.approx(sum(w[a, b] for a, b in ref), rel=1e-12)


def test_pair_index_round_trip(host):
    for n in (2, 4, 6, 16):
        idx = 0
        for a in range(n):
            for b in range(a + 1, n):
                assert host.km_host_pair_index(a, b, n) == idx
                ab = np.zeros(2, np.int32)
                host.km_host_pair_of(idx, n, iptr(ab))
                assert tuple(ab) == (a, b)
                idx += 1


@pytest.mark.parametrize("lam_min_rel,expect_direct", [(1e-2, True), (3e-7, False), (0.0, False)])
def test_pseudoinverse_route_and_cutoff(host, lam_min_rel, expect_direct):
    """The plain inverse is taken only when no eigenvalue can reach the
    cutoff rcond * lambda_max; otherwise the eigen-decomposition applies the
    cutoff. Either way A_a = S_a (S_a + S_b)^+ matches numpy's pinv with the
    same rcond (S_b = 0 here, so A_a is the projector onto the kept
    eigenvectors)."""
    rng = np.random.default_rng(41)
    d, rcond = 64, 1e-6
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    lam = np.exp(rng.uniform(0.0, 2.0, d))
    lam[0] = lam_min_rel * lam.max()
    Sa = np.ascontiguousarray((Qm * lam) @ Qm.T)
    Sa = 0.5 * (Sa + Sa.T)
    Sb = np.zeros((d, d))
    C = np.zeros((2 * d, 2 * d))
    Ag = np.zeros((2, d, d))
    sw = np.zeros(1, np.int32)
    got = host.km_host_pair(d, 0, 1, dptr(Sa), dptr(Sb), dptr(C), 2 * d, 0, 1, rcond, dptr(Ag),
                            iptr(sw))
    assert got == 0.0                                   # D = 0: nothing to lose
    assert (sw[0] == 0) == expect_direct
    ref = Sa @ np.linalg.pinv(Sa, rcond=rcond, hermitian=True)
    np.testing.assert_allclose(Ag[0], ref, rtol=0, atol=1e-9)
    np.testing.assert_array_equal(Ag[1], 0.0)
