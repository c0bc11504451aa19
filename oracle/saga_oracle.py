"""Float64 CPU oracle for one SAGA + Atop-N decode attention step.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module. The CUDA library never calls it, and it
shares no code with the CUDA library.

What it follows (source: "More Value per Key: Asymmetric Sparse Attention for
Faster LLM Decoding", the SAGA paper as summarised on its pages):
  * Attention Mechanism Formalization, Eq. (2-4): A = Q K^T / sqrt(d),
    P = softmax(A), O = P V.
  * Top-N Attention, Eq. (6): the indices of the N largest entries of a row.
  * Methodology > Atop-N Attention, item 1: entries are kept by a per-element
    comparison against a threshold equal to the N-th largest value; item 2:
    the exact threshold is recomputed once every n tokens (called R here) and
    reused in between.
  * Methodology > Atop-N Attention, Eq. (7): O = softmax(A[i]) V[i].
  * SAGA Architecture: h_k key heads and h_v value heads, decoupled.

Readings where the pages are silent (each also listed in the design notes):
  * Head maps: query head j reads key head floor(j*h_k/h_q) and value head
    floor(j*h_v/h_q) (contiguous groups, the GQA convention).
  * The comparison is A >= tau; ties at tau are all kept.
  * tau is the N-th largest of the row when N < l_kv; when N >= l_kv every
    entry is kept (tau = -inf), which is exact top-N attention for every
    later step too. l_kv = 0 gives tau = -inf and an empty selection.
  * An empty selection gives an output row of zeros.
  * Refresh steps are t = 0, R, 2R, ...; the refreshed tau applies to the
    same step's selection.
  * Exact top-N attention (Eq. 6) keeps exactly min(N, l_kv) positions; among
    equal scores the lower position wins (the pages fix no tie-break).
  * Decoding appends the token's key and value rows at position l_kv[b] of
    every head and grows l_kv[b] by one before the step attends.

Everything is computed in float64 from the exact values of the stored inputs,
with no blocking, fusion or reordering beyond the definitions above.
"""
import numpy as np

NEG_INF = float("-inf")


# --------------------------------------------------------------------------
# head maps (SAGA Architecture; contiguous groups)
# --------------------------------------------------------------------------
def key_head(j, h_q, h_k):
    return (j * h_k) // h_q


def value_head(j, h_q, h_v):
    return (j * h_v) // h_q


# --------------------------------------------------------------------------
# Eq. (2): A = q K^T / sqrt(d) for one decode query per head
# --------------------------------------------------------------------------
def scores(q, K, l_kv):
    """Score rows. q: [B][h_q][d], K: [B][h_k][cap][d] (float64).

    Returns a list over b of arrays [h_q][l_kv[b]].
    """
    B, h_q, d = q.shape
    h_k = K.shape[1]
    out = []
    for b in range(B):
        L = int(l_kv[b])
        rows = np.empty((h_q, L))
        for j in range(h_q):
            kh = key_head(j, h_q, h_k)
            rows[j] = (K[b, kh, :L, :] @ q[b, j]) / np.sqrt(d)
        out.append(rows)
    return out


# --------------------------------------------------------------------------
# Eq. (6) + Atop-N item 1: the threshold is the N-th largest entry
# --------------------------------------------------------------------------
def nth_largest(row, N):
    """The N-th largest entry of ``row`` (float64); -inf when N >= len(row)."""
    row = np.asarray(row, dtype=np.float64)
    if N >= row.size:
        return NEG_INF
    return float(np.sort(row)[::-1][N - 1])


def select(row, tau):
    """Atop-N item 1: indices t with A[t] >= tau, increasing."""
    return np.nonzero(np.asarray(row) >= tau)[0]


# --------------------------------------------------------------------------
# Eq. (7): softmax over the selected entries only, then the V-row gather
# --------------------------------------------------------------------------
def sparse_attend(row, V_rows, idx):
    """O = softmax(A[idx]) V[idx]; zeros for an empty selection."""
    d = V_rows.shape[1]
    if len(idx) == 0:
        return np.zeros(d)
    a = np.asarray(row, dtype=np.float64)[idx]
    m = a.max()
    w = np.exp(a - m)
    return (w @ V_rows[idx]) / w.sum()


def decode_step(q, K, V, l_kv, tau):
    """One Atop-N step with given thresholds tau [B][h_q].

    Returns (sel, out): sel[b][j] is the selected index array and out is
    [B][h_q][d] float64.
    """
    B, h_q, d = q.shape
    h_v = V.shape[1]
    A = scores(q, K, l_kv)
    out = np.zeros((B, h_q, d))
    sel = []
    for b in range(B):
        L = int(l_kv[b])
        sel_b = []
        for j in range(h_q):
            idx = select(A[b][j], tau[b][j])
            vh = value_head(j, h_q, h_v)
            out[b, j] = sparse_attend(A[b][j], V[b, vh, :L, :], idx)
            sel_b.append(idx)
        sel.append(sel_b)
    return sel, out


def refresh(q, K, l_kv, N):
    """Atop-N item 2: the exact threshold, tau[b][j] = N-th largest of the row."""
    B, h_q, _ = q.shape
    A = scores(q, K, l_kv)
    tau = np.empty((B, h_q))
    for b in range(B):
        for j in range(h_q):
            tau[b, j] = nth_largest(A[b][j], N)
    return tau


def dense_attend(q, K, V, l_kv):
    """Eq. (2-4): full softmax attention over every position t < l_kv[b]."""
    B, h_q, d = q.shape
    h_v = V.shape[1]
    A = scores(q, K, l_kv)
    out = np.zeros((B, h_q, d))
    for b in range(B):
        L = int(l_kv[b])
        for j in range(h_q):
            vh = value_head(j, h_q, h_v)
            out[b, j] = sparse_attend(A[b][j], V[b, vh, :L, :], np.arange(L))
    return out


def decode_chain(qs, K, V, l_kv, N, R):
    """Run steps t = 0..len(qs)-1, refreshing tau when t mod R == 0.

    Returns (taus [T][B][h_q], sels, outs [T][B][h_q][d]).
    """
    taus, sels, outs = [], [], []
    tau = None
    for t, q in enumerate(qs):
        if t % R == 0:
            tau = refresh(q, K, l_kv, N)
        s, o = decode_step(q, K, V, l_kv, tau)
        taus.append(tau.copy())
        sels.append(s)
        outs.append(o)
    return np.array(taus), sels, np.array(outs)


# --------------------------------------------------------------------------
# The same selection applied to an fp32 score row (for checking a dumped row)
# --------------------------------------------------------------------------
def f32_order_key(x):
    """Order-preserving uint32 key of float32 values under IEEE totalOrder
    (non-NaN): larger float -> larger key, and -0 < +0."""
    bits = np.asarray(x, dtype=np.float32).view(np.uint32)
    neg = (bits >> np.uint32(31)) == 1
    return np.where(neg, ~bits, bits | np.uint32(0x80000000)).astype(np.uint32)


def f32_from_order_key(k):
    k = np.asarray(k, dtype=np.uint32)
    pos = (k >> np.uint32(31)) == 1
    bits = np.where(pos, k & np.uint32(0x7FFFFFFF), ~k).astype(np.uint32)
    return bits.view(np.float32)


def nth_largest_f32(row_f32, N):
    """N-th largest of a float32 row under totalOrder, as float32; -inf when
    N >= len(row). Used to recompute a threshold from a given fp32 row."""
    row_f32 = np.asarray(row_f32, dtype=np.float32)
    if N >= row_f32.size:
        return np.float32(NEG_INF)
    keys = np.sort(f32_order_key(row_f32))[::-1]
    return f32_from_order_key(keys[N - 1:N])[0]


# --------------------------------------------------------------------------
# exact top-N attention (Eq. 6), ties broken towards the lower position
# --------------------------------------------------------------------------
def top_n_exact(row, N):
    """Positions of the min(N, len(row)) largest entries of `row`; among equal
    entries the lower position is taken first."""
    row = np.asarray(row, dtype=np.float64)
    order = np.lexsort((np.arange(row.size), -row))   # by -value, then position
    return np.sort(order[:min(N, row.size)])


def topn_step(q, K, V, l_kv, N):
    """One exact top-N attention step (Eq. 6 + Eq. 7) for every (b, j)."""
    B, h_q, d = q.shape
    h_v = V.shape[1]
    A = scores(q, K, l_kv)
    sels, out = [], np.zeros((B, h_q, d))
    for b in range(B):
        row_sels = []
        for j in range(h_q):
            idx = top_n_exact(A[b][j], N)
            out[b, j] = sparse_attend(A[b][j], V[b, value_head(j, h_q, h_v)], idx)
            row_sels.append(idx)
        sels.append(row_sels)
    return sels, out


# --------------------------------------------------------------------------
# KV-cache append (the decode step's input side)
# --------------------------------------------------------------------------
def append(K, V, l_kv, k_new, v_new):
    """Write each sequence's new key rows k_new [B][h_k][d] and value rows
    v_new [B][h_v][d] at position l_kv[b] of every head; returns copies of
    K, V and l_kv + 1."""
    K, V = np.array(K, copy=True), np.array(V, copy=True)
    l_kv = np.array(l_kv, copy=True)
    for b in range(K.shape[0]):
        t = int(l_kv[b])
        if t >= K.shape[2]:
            raise ValueError("cache full")
        K[b, :, t, :] = k_new[b]
        V[b, :, t, :] = v_new[b]
        l_kv[b] = t + 1
    return K, V, l_kv
