"""Seeded synthetic calibration inputs for the GQA-to-SAGA key-head merge.

This module draws inputs only; it holds none of the merge arithmetic.

Recipe (the shapes of the teacher models the SAGA paper converts, "More Value
per Key: Asymmetric Sparse Attention for Faster LLM Decoding", GQA-to-SAGA
Conversion; model shapes of Llama 3.2-1B and Qwen2.5-1.5B). No calibration
text or trained weights are used: these draws stand in for them.
  * Hidden states X [T][d_model]: i.i.d. N(0, 1), rounded to bf16.
  * Teacher key projection, stored as a linear layer's weight
    [h_k * d][d_model] in bf16: the key heads are split into planted pairs by
    a seeded random perfect matching; both heads of a planted pair share one
    base block B and add their own perturbation,
    W^a = B + 0.3 E_a, with B and E entries N(0, 1 / d_model). Real key heads
    are correlated like this, and it gives the matching a known answer.
  * Queries Q [T][h_q * d] in bf16: Q[t][j*d + c] = z * exp(0.4 n[j][c]) with
    z and n i.i.d. N(0, 1): every query head has its own anisotropic
    spectrum, so the S_r differ from head to head. Columns c >= d_eff are
    zero (rank-deficient calibration sets when d_eff < d).
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np

from .workload import BF16, normals, philox_words, to_storage

T_MX, T_MB, T_ME, T_MQ, T_MS, T_MP = 9, 10, 11, 12, 13, 14
PAIR_NOISE = 0.3
SPECTRUM_SPREAD = 0.4


@dataclass(frozen=True)
class MergeWorkload:
    name: str
    T: int            # calibration tokens
    d_model: int
    h_q: int
    h_k: int          # teacher key heads (even)
    d: int
    seed: int
    d_eff: Optional[int] = None   # query columns >= d_eff are zero

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return MergeWorkload(**d)


MERGE_WORKLOADS = {
    "merge_tiny": MergeWorkload("merge_tiny", T=256, d_model=128, h_q=8, h_k=4, d=64,
                                seed=20262001),
    "merge_tail_g1": MergeWorkload("merge_tail_g1", T=200, d_model=200, h_q=6, h_k=6, d=64,
                                   seed=20262002),
    "merge_tiny_d128": MergeWorkload("merge_tiny_d128", T=256, d_model=256, h_q=8, h_k=4,
                                     d=128, seed=20262003),
    "merge_rank_deficient": MergeWorkload("merge_rank_deficient", T=128, d_model=128, h_q=8,
                                          h_k=4, d=64, seed=20262004, d_eff=24),
    "merge_wide16": MergeWorkload("merge_wide16", T=512, d_model=256, h_q=16, h_k=16, d=64,
                                  seed=20262005),
    "llama1b_merge_8k": MergeWorkload("llama1b_merge_8k", T=8192, d_model=2048, h_q=32,
                                      h_k=8, d=64, seed=20262006),
    "qwen1p5b_merge_8k": MergeWorkload("qwen1p5b_merge_8k", T=8192, d_model=1536, h_q=12,
                                       h_k=2, d=128, seed=20262007),
}


def planted_pairs(w: MergeWorkload):
    """The planted pairing: a seeded random permutation read two by two,
    each pair as (a, b) with a < b, sorted by a."""
    n = w.h_k
    words, _, _, _ = philox_words(w.seed, T_MP, 0, 0, 0, np.arange(n, dtype=np.uint64))
    perm = list(range(n))
    for i in range(n - 1, 0, -1):          # Fisher-Yates from the top
        k = int(words[i]) % (i + 1)
        perm[i], perm[k] = perm[k], perm[i]
    pairs = [tuple(sorted(perm[2 * i:2 * i + 2])) for i in range(n // 2)]
    return sorted(pairs)


def hidden_states(w: MergeWorkload):
    """X as bf16 bits [T][d_model]."""
    z = normals(w.seed, T_MX, 0, 0, 0, 0, w.T * w.d_model)
    return to_storage(z.reshape(w.T, w.d_model), BF16)


def key_weight(w: MergeWorkload):
    """Teacher key projection as bf16 bits [h_k * d][d_model]."""
    s = 1.0 / np.sqrt(w.d_model)
    W = np.zeros((w.h_k * w.d, w.d_model))
    n = w.d * w.d_model
    for i, (a, b) in enumerate(planted_pairs(w)):
        base = normals(w.seed, T_MB, 0, 0, i, 0, n).reshape(w.d, w.d_model) * s
        for r in (a, b):
            e = normals(w.seed, T_ME, 0, 0, r, 0, n).reshape(w.d, w.d_model) * s
            W[r * w.d:(r + 1) * w.d] = base + PAIR_NOISE * e
    return to_storage(W, BF16)


def queries(w: MergeWorkload):
    """Calibration queries as bf16 bits [T][h_q * d]."""
    width = w.h_q * w.d
    z = normals(w.seed, T_MQ, 0, 0, 0, 0, w.T * width).reshape(w.T, width)
    n = normals(w.seed, T_MS, 0, 0, 0, 0, width)
    scale = np.exp(SPECTRUM_SPREAD * n)
    if w.d_eff is not None:
        scale = scale.reshape(w.h_q, w.d)
        scale[:, w.d_eff:] = 0.0
        scale = scale.reshape(-1)
    return to_storage(z * scale[None, :], BF16)


def merge_inputs(w: MergeWorkload):
    """(X, W_lin, Q) as bf16 bit arrays."""
    return hidden_states(w), key_weight(w), queries(w)
