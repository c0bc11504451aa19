"""Seeded synthetic workloads for the SAGA + Atop-N decode attention step.

This module draws inputs only; it holds none of the attention arithmetic.

Every value is a pure function of (seed, tensor id, layer, sequence b, head,
element index), computed by Philox4x32-10 and the Box-Muller transform in
``synth.philox`` / ``synth.normal``. The device generator in
``synth/csrc/synth_gen.cu`` evaluates the same functions in the same order, so
caches generated on the GPU are bit-identical to the slices this module
regenerates on the host.

Recipe (the shapes and distributions of the SAGA paper's decode workloads,
"More Value per Key: Asymmetric Sparse Attention for Faster LLM Decoding",
Methodology and Fig. 2; model shapes of Llama 3.2-1B and Qwen2.5-1.5B):
  * K, V entries i.i.d. N(0, 1), rounded to the cache dtype (fp32, or bf16 by
    round-to-nearest-even through fp32).
  * Planted keys: each (sequence, key head, position) is planted with
    probability 1/100 (a Bernoulli draw per position); a planted row is
    3 * u + 0.5 * xi, with u one unit direction per (seed, layer) and xi the
    row's own N(0, I) draw. This gives the heavy upper tail of scores that
    top-N selection is meant for.
  * Queries: AR(1) per (layer, b, head): q_0 = xi_0,
    q_t = 0.95 q_{t-1} + sqrt(1 - 0.95^2) xi_t, kept in float64 and rounded to
    the cache dtype at each step.
  * Ragged lengths (stress workload): l_kv[b] uniform on an integer range.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np

from .normal import box_muller
from .philox import philox4x32_10

# Tensor ids: the high bits of the Philox key.
T_K, T_V, T_Q, T_PLANT, T_U, T_LKV, T_KD, T_VD = 1, 2, 3, 4, 5, 6, 7, 8
PLANT_THRESH = 42949673           # round(0.01 * 2**32): P(plant) = 1/100
PLANT_SCALE = 3.0
PLANT_NOISE = 0.5
AR_RHO = 0.95

F32, BF16 = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: int                 # F32 or BF16
    B: int
    h_q: int
    h_k: int
    h_v: int
    d: int
    l_kv: int                  # length of every sequence (max for ragged)
    N: int
    R: int
    steps: int
    seed: int
    layers: int = 1
    dense_hkv: Optional[int] = None     # dense GQA comparison head count
    l_kv_range: Optional[Tuple[int, int]] = None  # ragged: inclusive range
    N_sweep: Tuple[int, ...] = field(default_factory=tuple)

    @property
    def elem_bytes(self):
        return 4 if self.dtype == F32 else 2

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five workloads: the tiny fp32 case, the two single-layer model shapes,
# the 16-layer batch-8 stack at 128K context, and the ragged refresh stress.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", F32, B=1, h_q=4, h_k=1, h_v=2, d=64,
                         l_kv=1024, N=64, R=8, steps=16, seed=20261000),
    "llama1b_32k": Workload("llama1b_32k", BF16, B=1, h_q=32, h_k=2, h_v=8,
                            d=64, l_kv=32768, N=1024, R=16, steps=64,
                            seed=20261001, dense_hkv=8),
    "qwen1p5b_128k": Workload("qwen1p5b_128k", BF16, B=1, h_q=12, h_k=1,
                              h_v=4, d=128, l_kv=131072, N=2048, R=16,
                              steps=64, seed=20261002, dense_hkv=2),
    "llama1b_stack16_b8_128k": Workload(
        "llama1b_stack16_b8_128k", BF16, B=8, h_q=32, h_k=2, h_v=8, d=64,
        l_kv=131072, N=2048, R=32, steps=32, seed=20261003, layers=16,
        dense_hkv=8),
    "ragged_refresh_b16": Workload(
        "ragged_refresh_b16", BF16, B=16, h_q=32, h_k=2, h_v=8, d=64,
        l_kv=524288, N=1024, R=1, steps=4, seed=20261004,
        l_kv_range=(8192, 524288), N_sweep=(256, 1024, 4096, 8192)),
}


def _key1(tensor, layer):
    return (tensor & 0xFF) | ((layer & 0xFF) << 8)


def philox_words(seed, tensor, layer, b, head, blocks):
    """The four Philox words for block indices ``blocks`` of one stream."""
    blocks = np.asarray(blocks, dtype=np.uint64)
    return philox4x32_10(blocks, head, b, 0, seed, _key1(tensor, layer))


def normals(seed, tensor, layer, b, head, e0, e1):
    """float64 N(0,1) draws for elements [e0, e1) of one (b, head) stream.

    Element e comes from block e // 4: words (w0, w1) give elements 4m, 4m+1
    and (w2, w3) give 4m+2, 4m+3.
    """
    m0, m1 = e0 // 4, (e1 + 3) // 4
    w0, w1, w2, w3 = philox_words(seed, tensor, layer, b, head,
                                  np.arange(m0, m1, dtype=np.uint64))
    z0, z1 = box_muller(w0, w1)
    z2, z3 = box_muller(w2, w3)
    z = np.stack([z0, z1, z2, z3], axis=1).reshape(-1)
    return z[e0 - 4 * m0: e1 - 4 * m0]


def planted(seed, layer, b, kh, t0, t1):
    """Boolean mask of planted key positions [t0, t1) of (b, key head kh)."""
    m0, m1 = t0 // 4, (t1 + 3) // 4
    w = philox_words(seed, T_PLANT, layer, b, kh,
                     np.arange(m0, m1, dtype=np.uint64))
    words = np.stack(w, axis=1).reshape(-1)
    return words[t0 - 4 * m0: t1 - 4 * m0] < np.uint32(PLANT_THRESH)


def unit_direction(seed, layer, d):
    """The fixed unit direction u of one (seed, layer), float64 [d].

    The squared norm is summed left to right so the device twin, which is
    handed these exact doubles, needs no reduction of its own.
    """
    g = normals(seed, T_U, layer, 0, 0, 0, d)
    ss = 0.0
    for x in g:
        ss = ss + float(x) * float(x)
    return g / np.sqrt(ss)


def to_storage(x64, dtype):
    """Round float64 values to the cache dtype; returns the storage array
    (float32, or uint16 bf16 bit patterns)."""
    f = np.asarray(x64, dtype=np.float64).astype(np.float32)
    if dtype == F32:
        return f
    bits = f.view(np.uint32).astype(np.uint64)
    r = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def widen(storage):
    """Exact float64 value of stored cache entries (float32 or bf16 bits)."""
    s = np.asarray(storage)
    if s.dtype == np.uint16:
        return (s.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return s.astype(np.float64)


def cache_rows(w: Workload, layer, kind, b, head, t0, t1):
    """Storage values of cache rows [t0, t1) of one (b, head): shape [t1-t0][d].

    kind: 'K' or 'V' (SAGA caches), 'KD' or 'VD' (dense GQA comparison caches).
    Keys ('K', 'KD') carry planted rows.
    """
    tensor = {"K": T_K, "V": T_V, "KD": T_KD, "VD": T_VD}[kind]
    d = w.d
    z = normals(w.seed, tensor, layer, b, head, t0 * d, t1 * d).reshape(t1 - t0, d)
    if kind in ("K", "KD"):
        # dense keys are planted under their own stream id so the two caches
        # stay independent
        plant_head = head if kind == "K" else 1000 + head
        mask = planted(w.seed, layer, b, plant_head, t0, t1)
        if mask.any():
            u = unit_direction(w.seed, layer, d)
            z = z.copy()
            z[mask] = PLANT_SCALE * u[None, :] + PLANT_NOISE * z[mask]
    return to_storage(z, w.dtype)


def cache(w: Workload, layer, kind, heads, cap=None, lens=None):
    """Whole cache [B][heads][cap][d] in storage dtype; rows t >= l_kv[b] are 0."""
    cap = w.l_kv if cap is None else cap
    lens = seq_lens(w) if lens is None else lens
    dt = np.float32 if w.dtype == F32 else np.uint16
    out = np.zeros((w.B, heads, cap, w.d), dtype=dt)
    for b in range(w.B):
        for h in range(heads):
            out[b, h, :lens[b]] = cache_rows(w, layer, kind, b, h, 0, int(lens[b]))
    return out


def seq_lens(w: Workload):
    """Per-sequence l_kv as int32 [B]."""
    if w.l_kv_range is None:
        return np.full(w.B, w.l_kv, dtype=np.int32)
    lo, hi = w.l_kv_range
    x, _, _, _ = philox_words(w.seed, T_LKV, 0, np.arange(w.B, dtype=np.uint64), 0, 0)
    span = np.uint64(hi - lo + 1)
    return (np.uint64(lo) + ((x.astype(np.uint64) * span) >> np.uint64(32))).astype(np.int32)


def queries(w: Workload, layer, steps, B=None, h_q=None):
    """AR(1) queries in storage dtype: [steps][B][h_q][d]."""
    B = w.B if B is None else B
    h_q = w.h_q if h_q is None else h_q
    d = w.d
    a = AR_RHO
    c = float(np.sqrt(1.0 - a * a))
    dt = np.float32 if w.dtype == F32 else np.uint16
    out = np.zeros((steps, B, h_q, d), dtype=dt)
    for b in range(B):
        for j in range(h_q):
            xi = normals(w.seed, T_Q, layer, b, j, 0, steps * d).reshape(steps, d)
            q = xi[0].copy()
            out[0, b, j] = to_storage(q, w.dtype)
            for t in range(1, steps):
                q = a * q + c * xi[t]
                out[t, b, j] = to_storage(q, w.dtype)
    return out


def cache_rows_at(w: Workload, layer, kind, b, head, ts):
    """Storage values of cache rows at arbitrary positions ``ts`` of one
    (b, head): shape [len(ts)][d]; identical to the same rows of cache_rows."""
    tensor = {"K": T_K, "V": T_V, "KD": T_KD, "VD": T_VD}[kind]
    ts = np.asarray(ts, dtype=np.int64)
    d = w.d
    if ts.size == 0:
        return to_storage(np.zeros((0, d)), w.dtype)
    blocks = (ts[:, None] * (d // 4) + np.arange(d // 4)[None, :]).reshape(-1)
    w0, w1, w2, w3 = philox_words(w.seed, tensor, layer, b, head, blocks.astype(np.uint64))
    z0, z1 = box_muller(w0, w1)
    z2, z3 = box_muller(w2, w3)
    z = np.stack([z0, z1, z2, z3], axis=1).reshape(ts.size, d)
    if kind in ("K", "KD"):
        plant_head = head if kind == "K" else 1000 + head
        pw = philox_words(w.seed, T_PLANT, layer, b, plant_head, (ts // 4).astype(np.uint64))
        words = np.stack(pw, axis=1)[np.arange(ts.size), ts % 4]
        mask = words < np.uint32(PLANT_THRESH)
        if mask.any():
            u = unit_direction(w.seed, layer, d)
            z[mask] = PLANT_SCALE * u[None, :] + PLANT_NOISE * z[mask]
    return to_storage(z, w.dtype)
