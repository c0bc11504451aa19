"""Float64 CPU oracle of the GQA-to-SAGA key-head merge (closed-form stage).

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module. The CUDA library never calls it, and it
shares no code with the CUDA library.

What it follows (source: "More Value per Key: Asymmetric Sparse Attention for
Faster LLM Decoding", GQA-to-SAGA Conversion, Stage 1: Closed-Form
Initialization):
  * Eq. (13): the loss of replacing key heads a and b by one merged key
    projection M is the squared Frobenius distance between the logits each of
    their query heads sees through M and through its own key projection,
    summed over the query heads of a and of b.
  * Eq. (15), Lemma 4.1: the minimising M is
    (W_K^a S_a + W_K^b S_b) (S_a + S_b)^+, with S_r the sum of Q^j^T Q^j over
    the query heads j of key head r and + the Moore-Penrose pseudoinverse.
  * Eq. (14), Theorem 4.2: the pairing of the teacher's key heads minimises
    the summed pair losses; it is a minimum-weight perfect matching of the
    complete graph whose edge (a, b) weighs L_{a,b} at the Eq. (15) optimum.

Readings where the pages are silent (each also listed in the design notes):
  * Query head j of the teacher belongs to key head floor(j * h_k / h_q) (the
    GQA grouping of the attention step), so Q_r holds h_q / h_k heads.
  * X is [T][d_model] (one calibration token per row), Q^j is [T][d] (the
    columns j*d .. j*d+d of the queries [T][h_q*d]) and W_K^r is the
    [d_model][d] block whose product X W_K^r gives key head r's keys; the
    stored key projection is the linear layer's weight [h_k*d][d_model], so
    W_K^r[i][c] = W_lin[r*d + c][i].
  * Merging is by pairs (m = 2, as Eq. (14) and Theorem 4.2 are written): the
    student has h_k / 2 key heads, merged head i coming from the i-th pair,
    pairs listed as (a, b) with a < b and sorted by a.
  * The pseudoinverse drops the eigenvalues of the symmetric positive
    semi-definite S_a + S_b that are at most rcond times the largest one.
  * Among perfect matchings of equal total weight the first one in the
    enumeration order below wins (the pages fix no tie-break).

Everything is computed in float64 from the exact values of the stored inputs.
"""
import numpy as np


# --------------------------------------------------------------------------
# query groups and their Gram matrices (the S_r under Eq. 15)
# --------------------------------------------------------------------------
def query_groups(h_q, h_k):
    """Query heads of each teacher key head: list over r of lists of j."""
    groups = [[] for _ in range(h_k)]
    for j in range(h_q):
        groups[(j * h_k) // h_q].append(j)
    return groups


def query_block(Q, j, d):
    """Q^j: the [T][d] queries of head j out of Q [T][h_q*d]."""
    return Q[:, j * d:(j + 1) * d]


def key_block(W_lin, r, d):
    """W_K^r [d_model][d] out of the linear layer's weight [h_k*d][d_model]."""
    return W_lin[r * d:(r + 1) * d, :].T


def query_gram(Q, h_q, h_k, d):
    """S_r = sum over j in Q_r of Q^j^T Q^j, float64 [h_k][d][d]."""
    S = np.zeros((h_k, d, d))
    for r, js in enumerate(query_groups(h_q, h_k)):
        for j in js:
            Qj = query_block(Q, j, d)
            S[r] += Qj.T @ Qj
    return S


# --------------------------------------------------------------------------
# Eq. (15): the merged key projection of one pair
# --------------------------------------------------------------------------
def pinv_psd(S, rcond):
    """Moore-Penrose pseudoinverse of a symmetric PSD matrix; eigenvalues at
    most rcond * (largest) count as zero."""
    return np.linalg.pinv(S, rcond=rcond, hermitian=True)


def merged_projection(W_a, W_b, S_a, S_b, rcond):
    """Eq. (15): (W_a S_a + W_b S_b)(S_a + S_b)^+, float64 [d_model][d]."""
    return (W_a @ S_a + W_b @ S_b) @ pinv_psd(S_a + S_b, rcond)


# --------------------------------------------------------------------------
# Eq. (13): the pair loss, from the logits themselves
# --------------------------------------------------------------------------
def logit_gap(X, M, W_r, Qj, chunk=2048):
    """|| Q^j (X M)^T - Q^j (X W_r)^T ||_F^2, with the [T][T] logit matrices
    formed a block of query rows at a time."""
    K_m = X @ M
    K_r = X @ W_r
    total = 0.0
    for t0 in range(0, Qj.shape[0], chunk):
        q = Qj[t0:t0 + chunk]
        diff = q @ K_m.T - q @ K_r.T
        total += float(np.sum(diff * diff))
    return total


def pair_loss(X, W_lin, Q, h_q, h_k, d, a, b, M):
    """Eq. (13): L_{a,b}(M) for key heads a and b of the teacher."""
    groups = query_groups(h_q, h_k)
    total = 0.0
    for r in (a, b):
        W_r = key_block(W_lin, r, d)
        for j in groups[r]:
            total += logit_gap(X, M, W_r, query_block(Q, j, d))
    return total


def pair_weights(X, W_lin, Q, h_q, h_k, d, rcond, pairs=None):
    """Edge weights w(a, b) = L_{a,b}(Eq. 15 optimum) for a < b.

    Returns (w [h_k][h_k] symmetric with a zero diagonal, {(a, b): M}).
    `pairs` limits the work to the listed (a, b); the other weights are NaN.
    """
    S = query_gram(Q, h_q, h_k, d)
    w = np.full((h_k, h_k), np.nan)
    np.fill_diagonal(w, 0.0)
    Ms = {}
    todo = pairs if pairs is not None else [(a, b) for a in range(h_k) for b in range(a + 1, h_k)]
    for a, b in todo:
        M = merged_projection(key_block(W_lin, a, d), key_block(W_lin, b, d), S[a], S[b], rcond)
        w[a, b] = w[b, a] = pair_loss(X, W_lin, Q, h_q, h_k, d, a, b, M)
        Ms[(a, b)] = M
    return w, Ms


# --------------------------------------------------------------------------
# Eq. (14) / Theorem 4.2: minimum-weight perfect matching, by enumeration
# --------------------------------------------------------------------------
def perfect_matchings(nodes):
    """Every perfect matching of `nodes` (a sorted list): the lowest node is
    paired with each other node in increasing order, the rest recursively.
    Each matching is a list of (a, b), a < b, sorted by a."""
    if not nodes:
        yield []
        return
    a = nodes[0]
    for i in range(1, len(nodes)):
        b = nodes[i]
        rest = nodes[1:i] + nodes[i + 1:]
        for m in perfect_matchings(rest):
            yield [(a, b)] + m


def matching_total(w, pairs):
    """Summed weight of a matching, the pairs added from the last to the
    first (pairs sorted by their lower node)."""
    total = 0.0
    for a, b in reversed(pairs):
        total = float(w[a, b]) + total
    return total


def min_weight_perfect_matching(w):
    """Minimum-weight perfect matching of the complete graph with weights w
    (even node count). Returns (pairs, total)."""
    n = w.shape[0]
    if n % 2:
        raise ValueError("a perfect matching needs an even number of nodes")
    best, best_total = None, np.inf
    for m in perfect_matchings(list(range(n))):
        total = matching_total(w, m)
        if total < best_total:
            best, best_total = m, total
    return best, best_total


# --------------------------------------------------------------------------
# the whole closed-form stage
# --------------------------------------------------------------------------
def merge_keys(X, W_lin, Q, h_q, h_k, d, rcond):
    """Stage 1 of the conversion: pair weights, the optimal pairing, and the
    student's key projection (linear-layer layout [h_k/2 * d][d_model]).

    Returns a dict with w, pairs, total and W_S.
    """
    w, Ms = pair_weights(X, W_lin, Q, h_q, h_k, d, rcond)
    pairs, total = min_weight_perfect_matching(w)
    W_S = np.concatenate([Ms[p].T for p in pairs], axis=0)
    return {"w": w, "pairs": pairs, "total": total, "W_S": W_S}


def student_head_order(pairs):
    """Teacher key (and value) heads in the student's order: a_0, b_0, a_1,
    b_1, ... so that merged key head i serves the query heads of a_i then
    b_i as one contiguous group."""
    return [h for p in pairs for h in p]
