"""Pins for the seeded input generator (host side)."""
import numpy as np
import torch

import synth
from synth.normal import ln_u1, sincos_2pi_u2
from synth.philox import philox4x32_10


def test_philox_known_answers():
    # Known-answer vectors published with the Philox4x32-10 definition
    # (Salmon et al., SC 2011, Random123 distribution).
    cases = [
        ((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
        ((0xffffffff,) * 4, (0xffffffff,) * 2, (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
        ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
         (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
    ]
    for ctr, key, want in cases:
        got = tuple(int(x) for x in philox4x32_10(*ctr, *key))
        assert got == want


def test_series_functions_match_libm():
    x = np.random.default_rng(0).integers(0, 2**32, 200_000, dtype=np.uint64).astype(np.uint32)
    x = np.concatenate([x, np.array([0, 1, 2**31, 2**32 - 1, 2**30, 3 * 2**30], np.uint32)])
    ln = ln_u1(x)
    ref = np.log((x.astype(np.float64) + 1.0) * 2.0 ** -32)
    assert np.max(np.abs(ln - ref) / np.maximum(np.abs(ref), 1e-300)) < 4e-15
    s, c = sincos_2pi_u2(x)
    ang = 2 * np.pi * x.astype(np.float64) * 2.0 ** -32
    assert np.max(np.abs(s - np.sin(ang))) < 4e-15
    assert np.max(np.abs(c - np.cos(ang))) < 4e-15


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(100_000) * 10.0 ** rng.integers(-5, 5, 100_000)
    # exact ties of the bf16 rounding (low 16 bits == 0x8000), both parities
    ties = (np.arange(0x3f800000, 0x3f800000 + 64 * 0x10000, 0x10000, dtype=np.uint32) | 0x8000)
    x = np.concatenate([x, ties.view(np.float32).astype(np.float64)])
    ours = synth.to_storage(x, synth.BF16)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = synth.widen(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_slices_are_consistent_and_moments():
    w = synth.WORKLOADS["llama1b_32k"]
    full = synth.cache_rows(w, 0, "K", 0, 1, 0, 4000)
    part = synth.cache_rows(w, 0, "K", 0, 1, 1234, 2345)
    np.testing.assert_array_equal(full[1234:2345], part)
    v = synth.widen(synth.cache_rows(w, 0, "V", 0, 3, 0, 8192))
    assert abs(v.mean()) < 0.01 and abs(v.var() - 1) < 0.01
    m = synth.planted(w.seed, 0, 0, 0, 0, 200_000)
    assert abs(m.mean() - 0.01) < 0.001
    u = synth.unit_direction(w.seed, 0, w.d)
    assert abs(np.linalg.norm(u) - 1) < 1e-12
    # planted rows lie along u: mean projection ~ 3
    k = synth.widen(synth.cache_rows(w, 0, "K", 0, 0, 0, 20000))
    pm = synth.planted(w.seed, 0, 0, 0, 0, 20000)
    assert abs((k[pm] @ u).mean() - 3.0) < 0.1


def test_ragged_lengths_in_range():
    w = synth.WORKLOADS["ragged_refresh_b16"]
    l = synth.seq_lens(w)
    assert l.shape == (16,) and l.min() >= 8192 and l.max() <= 524288
    assert len(set(l.tolist())) == 16


def test_queries_ar1():
    w = synth.WORKLOADS["tiny_f32"]
    qs = synth.widen(synth.queries(w, 0, 200))
    a = qs[:, 0, :, :].reshape(200, -1)
    # lag-1 autocorrelation of an AR(1) with rho = 0.95
    r = np.mean(a[1:] * a[:-1]) / np.mean(a * a)
    assert 0.85 < r < 1.0
