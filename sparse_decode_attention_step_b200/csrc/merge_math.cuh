// Small dense linear algebra of the closed-form key merge ("More Value per
// Key: Asymmetric Sparse Attention for Faster LLM Decoding", GQA-to-SAGA
// Conversion, Stage 1): the eigen-decomposition behind the pseudoinverse of
// Eq. (15), the pair weight of Theorem 4.2 in the form trace(D H), the
// minimum-weight perfect matching of Eq. (14), and one element of the merged
// key projection.
//
// Every routine is written for a team of threads that cooperate through
// `Team::sync()`: on the GPU a thread block, on the host one thread running
// the same loops in order. Within a phase between two syncs, every item
// writes locations no other item of the phase reads or writes, and every
// reduction runs in a fixed order independent of the team size, so a host
// build of these routines produces bit-for-bit the device results. Products
// with an add are written as explicit fma() for the same reason.
#pragma once

#include <math.h>
#include <stdint.h>

#if defined(__CUDACC__)
#define KM_HD __host__ __device__ __forceinline__
#else
#define KM_HD inline
#endif

namespace saga {
namespace merge {

struct Team {
  int tid, n;
  KM_HD void sync() const {
#if defined(__CUDA_ARCH__)
    __syncthreads();
#endif
  }
};

KM_HD int popcount32(uint32_t x) {
#if defined(__CUDA_ARCH__)
  return __popc(x);
#else
  return __builtin_popcount(x);
#endif
}

KM_HD int lowest_bit(uint32_t x) {
#if defined(__CUDA_ARCH__)
  return __ffs(static_cast<int>(x)) - 1;
#else
  return __builtin_ctz(x);
#endif
}

// ---- cyclic Jacobi eigen-decomposition ----------------------------------
// Round-robin (circle method) ordering: in round r of a sweep (0 <= r < d-1)
// slot k (0 <= k < d/2) rotates the pair (p, q), p < q. Seat 0 holds index 0;
// seat s > 0 holds 1 + (s - 1 + r) mod (d - 1); slot k pairs seats k and
// d-1-k, so every pair of indices meets once per sweep.
KM_HD void round_pair(int d, int r, int k, int &p, int &q) {
  const int x = k == 0 ? 0 : 1 + (k - 1 + r) % (d - 1);
  const int s = d - 1 - k;
  const int y = 1 + (s - 1 + r) % (d - 1);
  p = x < y ? x : y;
  q = x < y ? y : x;
}

// Rotation that zeroes the (p, q) entry of a symmetric 2 x 2 block
// [[app, apq], [apq, aqq]]: J = [[c, s], [-s, c]], J^T A J diagonal
// (the symmetric Schur decomposition of Golub and Van Loan, Matrix
// Computations, section 8.5: t is the smaller root of t^2 + 2 tau t - 1 = 0).
KM_HD void schur2(double app, double apq, double aqq, double &c, double &s) {
  if (apq == 0.0) {
    c = 1.0;
    s = 0.0;
    return;
  }
  const double tau = (aqq - app) / (2.0 * apq);
  const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(fma(tau, tau, 1.0)));
  c = 1.0 / sqrt(fma(t, t, 1.0));
  s = t * c;
}

KM_HD void rot_apply(double c, double s, double &x, double &y) {
  const double nx = fma(c, x, -(s * y));
  const double ny = fma(s, x, c * y);
  x = nx;
  y = ny;
}

KM_HD void rot_apply(double c, double s, float &x, float &y) {
  const float cf = static_cast<float>(c), sf = static_cast<float>(s);
  const float nx = fmaf(cf, x, -(sf * y));
  const float ny = fmaf(sf, x, cf * y);
  x = nx;
  y = ny;
}

// Eigen-decomposition of the symmetric d x d matrix S (row-major, d even),
// S = E^T diag(lambda) E. On return the diagonal of S holds lambda and row l
// of E (type VT: double, or float where shared memory is short) the unit
// eigenvector of lambda_l. Scratch: rc, rs [d/2]; rowbuf [d].
// Sweeps stop once the off-diagonal squared norm is at most tol^2 times the
// diagonal one, or after max_sweeps. Returns the number of sweeps run.
template <typename VT>
KM_HD int jacobi_eigh(const Team &tm, int d, double *S, VT *E, double *rc, double *rs,
                      double *rowbuf, int max_sweeps, double tol) {
  const int half = d / 2;
  for (int e = tm.tid; e < d * d; e += tm.n) E[e] = (e / d == e % d) ? VT(1) : VT(0);
  tm.sync();
  int sweep = 0;
  while (sweep < max_sweeps) {
    for (int r = 0; r < d - 1; ++r) {
      // rotations of this round, from the current 2 x 2 blocks
      for (int k = tm.tid; k < half; k += tm.n) {
        int p, q;
        round_pair(d, r, k, p, q);
        schur2(S[p * d + p], S[p * d + q], S[q * d + q], rc[k], rs[k]);
      }
      tm.sync();
      // rows p and q of S and of E: S <- J^T S, E <- J^T E
      for (int e = tm.tid; e < half * d; e += tm.n) {
        const int k = e / d, j = e % d;
        const double c = rc[k], s = rs[k];
        if (s == 0.0) continue;
        int p, q;
        round_pair(d, r, k, p, q);
        rot_apply(c, s, S[p * d + j], S[q * d + j]);
        rot_apply(c, s, E[p * d + j], E[q * d + j]);
      }
      tm.sync();
      // columns p and q of S: S <- S J; the rotated pair's entries are zero
      for (int e = tm.tid; e < d * half; e += tm.n) {
        const int i = e / half, k = e % half;
        const double c = rc[k], s = rs[k];
        if (s == 0.0) continue;
        int p, q;
        round_pair(d, r, k, p, q);
        double x = S[i * d + p], y = S[i * d + q];
        rot_apply(c, s, x, y);
        if (i == p) y = 0.0;
        if (i == q) x = 0.0;
        S[i * d + p] = x;
        S[i * d + q] = y;
      }
      tm.sync();
    }
    ++sweep;
    // convergence: row sums in column order, then the rows in order
    for (int i = tm.tid; i < d; i += tm.n) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j)
        if (j != i) acc = fma(S[i * d + j], S[i * d + j], acc);
      rowbuf[i] = acc;
    }
    tm.sync();
    double off = 0.0, dia = 0.0;
    for (int i = 0; i < d; ++i) {
      off += rowbuf[i];
      dia = fma(S[i * d + i], S[i * d + i], dia);
    }
    tm.sync();                      // rowbuf is rewritten by the next check
    if (off <= tol * tol * dia) break;
  }
  return sweep;
}

// Pseudoinverse weights: inv[l] = 1 / lambda_l where |lambda_l| > rcond * max |lambda|,
// else 0 (the Moore-Penrose convention for a symmetric matrix); lambda on the
// diagonal of S. Every thread forms the maximum in the same order.
KM_HD void pinv_weights(const Team &tm, int d, const double *S, double rcond, double *inv) {
  double mx = 0.0;
  for (int l = 0; l < d; ++l) mx = fmax(mx, fabs(S[l * d + l]));
  const double cut = rcond * mx;
  for (int l = tm.tid; l < d; l += tm.n) {
    const double lam = S[l * d + l];
    inv[l] = fabs(lam) > cut ? 1.0 / lam : 0.0;
  }
  tm.sync();
}

// The d x d products below are formed in 4 x 4 blocks per item (d a
// multiple of 4): each loaded operand value feeds four FMAs. Every element is
// still one sum over m (or l) in increasing order.
constexpr int kBlk = 4;

// P = E^T diag(inv) E, i.e. P[i][k] = sum_l inv_l E[l][i] E[l][k].
template <typename VT>
KM_HD void pinv_from_eigen(const Team &tm, int d, const VT *E, const double *inv, double *P) {
  const int nb = d / kBlk;
  for (int e = tm.tid; e < nb * nb; e += tm.n) {
    const int i0 = (e / nb) * kBlk, k0 = (e % nb) * kBlk;
    double acc[kBlk][kBlk];
    for (int r = 0; r < kBlk; ++r)
      for (int c = 0; c < kBlk; ++c) acc[r][c] = 0.0;
    for (int l = 0; l < d; ++l) {
      double x[kBlk], y[kBlk];
      for (int r = 0; r < kBlk; ++r) x[r] = inv[l] * static_cast<double>(E[l * d + i0 + r]);
      for (int c = 0; c < kBlk; ++c) y[c] = static_cast<double>(E[l * d + k0 + c]);
      for (int r = 0; r < kBlk; ++r)
        for (int c = 0; c < kBlk; ++c) acc[r][c] = fma(x[r], y[c], acc[r][c]);
    }
    for (int r = 0; r < kBlk; ++r)
      for (int c = 0; c < kBlk; ++c) P[(i0 + r) * d + k0 + c] = acc[r][c];
  }
}

// out = A B for d x d row-major matrices, sum over m in order.
KM_HD void matmul_dd(const Team &tm, int d, const double *A, const double *B, double *out) {
  const int nb = d / kBlk;
  for (int e = tm.tid; e < nb * nb; e += tm.n) {
    const int i0 = (e / nb) * kBlk, k0 = (e % nb) * kBlk;
    double acc[kBlk][kBlk];
    for (int r = 0; r < kBlk; ++r)
      for (int c = 0; c < kBlk; ++c) acc[r][c] = 0.0;
    for (int m = 0; m < d; ++m) {
      double x[kBlk], y[kBlk];
      for (int r = 0; r < kBlk; ++r) x[r] = A[(i0 + r) * d + m];
      for (int c = 0; c < kBlk; ++c) y[c] = B[m * d + k0 + c];
      for (int r = 0; r < kBlk; ++r)
        for (int c = 0; c < kBlk; ++c) acc[r][c] = fma(x[r], y[c], acc[r][c]);
    }
    for (int r = 0; r < kBlk; ++r)
      for (int c = 0; c < kBlk; ++c) out[(i0 + r) * d + k0 + c] = acc[r][c];
  }
}

// In-place inverse of the symmetric positive definite d x d matrix S by
// Gauss-Jordan sweeps without pivoting (the pivots of an SPD matrix are its
// Schur complements, all positive). Step k saves column and row k (col, row
// [d]), then updates every entry from the saved values. Returns false, with
// S undefined, as soon as a pivot is not a positive finite number.
KM_HD bool spd_inverse(const Team &tm, int d, double *S, double *col, double *row) {
  for (int k = 0; k < d; ++k) {
    for (int i = tm.tid; i < d; i += tm.n) {
      col[i] = S[i * d + k];
      row[i] = S[k * d + i];
    }
    tm.sync();
    const double p = col[k];
    if (!(p > 0.0) || !(p < INFINITY)) return false;   // every thread reads the same pivot
    const double ip = 1.0 / p;
    for (int e = tm.tid; e < d * d; e += tm.n) {
      const int i = e / d, j = e % d;
      double v;
      if (i == k && j == k) v = ip;
      else if (i == k) v = row[j] * ip;
      else if (j == k) v = -(col[i] * ip);
      else v = fma(-col[i], row[j] * ip, S[e]);
      S[e] = v;
    }
    tm.sync();
  }
  return true;
}

// Whether an inverse of S (its trace `tr`) is its pseudoinverse under the
// cutoff rcond: the smallest eigenvalue is at least 1 / ||S^-1||_F and the
// largest at most the trace, so 1 / ||S^-1||_F > rcond * trace keeps every
// eigenvalue. Row sums of squares in order, then the rows.
KM_HD bool inverse_is_pinv(const Team &tm, int d, const double *Sinv, double tr, double rcond,
                           double *rowbuf) {
  for (int i = tm.tid; i < d; i += tm.n) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc = fma(Sinv[i * d + j], Sinv[i * d + j], acc);
    rowbuf[i] = acc;
  }
  tm.sync();
  double fro2 = 0.0;
  for (int i = 0; i < d; ++i) fro2 += rowbuf[i];
  tm.sync();
  return fro2 < INFINITY && 1.0 > rcond * tr * sqrt(fro2);
}

// D[k][i] of the pair (a, b) from the key Gram matrix C [hd][hd]
// (C = K^T K, K = [K_0 ... K_{h_k-1}]): (K_a - K_b)^T (K_a - K_b).
KM_HD double pair_gap(const double *C, long long hd, int d, int a, int b, int k, int i) {
  const long long ra = static_cast<long long>(a) * d + k, rb = static_cast<long long>(b) * d + k;
  const long long ca = static_cast<long long>(a) * d + i, cb = static_cast<long long>(b) * d + i;
  return ((C[ra * hd + ca] - C[ra * hd + cb]) - C[rb * hd + ca]) + C[rb * hd + cb];
}

// Pair weight trace(D H) with H = A_a S_b (A_a = S_a (S_a + S_b)^+):
// items form 4 x 4 blocks of H[k][i] and D[i][k] H[k][i] (D symmetric, read as
// D[k][i]) into T; rows of T are summed in order, then the rows.
KM_HD double pair_weight(const Team &tm, int d, const double *A_a, const double *S_b,
                         const double *C, long long hd, int a, int b, double *T,
                         double *rowbuf) {
  const int nb = d / kBlk;
  for (int e = tm.tid; e < nb * nb; e += tm.n) {
    const int k0 = (e / nb) * kBlk, i0 = (e % nb) * kBlk;
    double h[kBlk][kBlk];
    for (int r = 0; r < kBlk; ++r)
      for (int c = 0; c < kBlk; ++c) h[r][c] = 0.0;
    for (int m = 0; m < d; ++m) {
      double x[kBlk], y[kBlk];
      for (int r = 0; r < kBlk; ++r) x[r] = A_a[(k0 + r) * d + m];
      for (int c = 0; c < kBlk; ++c) y[c] = S_b[m * d + i0 + c];
      for (int r = 0; r < kBlk; ++r)
        for (int c = 0; c < kBlk; ++c) h[r][c] = fma(x[r], y[c], h[r][c]);
    }
    for (int r = 0; r < kBlk; ++r)
      for (int c = 0; c < kBlk; ++c)
        T[(k0 + r) * d + i0 + c] = pair_gap(C, hd, d, a, b, k0 + r, i0 + c) * h[r][c];
  }
  tm.sync();
  for (int k = tm.tid; k < d; k += tm.n) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += T[k * d + i];
    rowbuf[k] = acc;
  }
  tm.sync();
  double w = 0.0;
  for (int k = 0; k < d; ++k) w += rowbuf[k];
  tm.sync();
  return w;
}

// Pairs (a, b), a < b, of n nodes in the order (0,1), (0,2), ..., (0,n-1),
// (1,2), ...: index <-> pair.
KM_HD int pair_index(int a, int b, int n) { return a * (2 * n - a - 1) / 2 + (b - a - 1); }

KM_HD void pair_of(int idx, int n, int &a, int &b) {
  a = 0;
  while (idx >= n - 1 - a) {
    idx -= n - 1 - a;
    ++a;
  }
  b = a + 1 + idx;
}

constexpr int kMaxSweeps = 40;
constexpr double kJacobiTol = 1e-13;   // off-diagonal norm / diagonal norm at convergence

// Everything one pair (a, b) needs, from the query Gram matrices S_a, S_b
// [d][d] and the key Gram matrix C [hd][hd] (all float64):
//   P = (S_a + S_b)^+, A_a = S_a P and A_b = S_b P into Ag [2][d][d]
//   (Eq. 15 is W^a A_a + W^b A_b), and returns w(a, b) = trace(D A_a S_b), the
//   Eq. (13) loss at the optimum.
// P is the plain inverse when `direct` is set, the Gauss-Jordan sweeps
// succeed and the inverse provably keeps every eigenvalue above the cutoff
// (then it is the pseudoinverse); otherwise the Jacobi eigen-decomposition
// gives it with the cutoff applied. *path receives 0 for the inverse, else
// the number of Jacobi sweeps.
// Shared scratch: S [d][d] (float64), E [d][d] (VT), rc, rs [d/2], rowbuf, inv [d].
template <typename VT>
KM_HD double pair_stage(const Team &tm, int d, const double *Sa, const double *Sb,
                        const double *C, long long hd, int a, int b, double rcond, double *S,
                        VT *E, double *rc, double *rs, double *rowbuf, double *inv, double *Ag,
                        bool direct, int *path) {
  for (int e = tm.tid; e < d * d; e += tm.n) S[e] = Sa[e] + Sb[e];
  tm.sync();
  bool have = false;
  if (direct) {
    double tr = 0.0;
    for (int l = 0; l < d; ++l) tr += S[l * d + l];
    tm.sync();                               // the trace is read before the sweeps
    have = spd_inverse(tm, d, S, inv, rowbuf) && inverse_is_pinv(tm, d, S, tr, rcond, rowbuf);
  }
  int sw = 0;
  if (!have) {
    for (int e = tm.tid; e < d * d; e += tm.n) S[e] = Sa[e] + Sb[e];
    tm.sync();
    sw = jacobi_eigh(tm, d, S, E, rc, rs, rowbuf, kMaxSweeps, kJacobiTol);
    pinv_weights(tm, d, S, rcond, inv);
    pinv_from_eigen(tm, d, E, inv, S);      // P replaces S (its diagonal was read above)
    tm.sync();
  }
  matmul_dd(tm, d, Sa, S, Ag);
  matmul_dd(tm, d, Sb, S, Ag + d * d);
  tm.sync();
  const double w = pair_weight(tm, d, Ag, Sb, C, hd, a, b, S, rowbuf);
  if (path != nullptr && tm.tid == 0) *path = sw;
  return w;
}

// ---- Eq. (14) / Theorem 4.2: minimum-weight perfect matching ------------
// Exact dynamic programme over node subsets (n even, n <= 16):
// f(mask) = min over j in mask, j > low(mask), of w[low][j] + f(mask - {low, j}),
// the first j attaining the minimum; subsets are filled by increasing size.
// The matching's total is then summed as w(pair_1) + (w(pair_2) + ...), the
// pairs in increasing order of their lower node.
KM_HD void match_dp(const Team &tm, int n, const double *w, double *f, int8_t *choice) {
  const uint32_t full = (1u << n) - 1u;
  for (uint32_t m = tm.tid; m <= full; m += tm.n) {
    f[m] = m == 0 ? 0.0 : INFINITY;
    choice[m] = -1;
  }
  tm.sync();
  for (int level = 1; 2 * level <= n; ++level) {
    for (uint32_t m = tm.tid; m <= full; m += tm.n) {
      if (popcount32(m) != 2 * level) continue;
      const int low = lowest_bit(m);
      double best = INFINITY;
      int bj = -1;
      for (int j = low + 1; j < n; ++j) {
        if (!((m >> j) & 1u)) continue;
        const double v = w[low * n + j] + f[m ^ (1u << low) ^ (1u << j)];
        if (bj < 0 || v < best) {
          best = v;
          bj = j;
        }
      }
      f[m] = best;
      choice[m] = static_cast<int8_t>(bj);
    }
    tm.sync();
  }
}

// Read the matching off the table: pairs[2i], pairs[2i+1] of the i-th pair.
KM_HD void match_pairs(int n, const int8_t *choice, int32_t *pairs) {
  uint32_t m = (1u << n) - 1u;
  int i = 0;
  while (m != 0u) {
    const int low = lowest_bit(m);
    int j = choice[m];
    if (j <= low || j >= n || !((m >> j) & 1u)) {   // unreachable for a filled table
      j = low + 1;
      while (j < n && !((m >> j) & 1u)) ++j;
    }
    pairs[2 * i] = low;
    pairs[2 * i + 1] = j;
    m ^= (1u << low) | (1u << j);
    ++i;
  }
}

// ---- Eq. (15): one element of the merged key projection -----------------
// W_S[c][x] = sum_m W_K^a[x][m] A_a[m][c] + sum_m W_K^b[x][m] A_b[m][c], with
// W_K^r[x][m] the linear layer's W_lin[r*d + m][x] (given as the widened
// bf16 values wa[m], wb[m]), A_r = S_r (S_a + S_b)^+.
KM_HD double merged_elem(int d, const double *wa, const double *wb, const double *A_a,
                         const double *A_b, int c) {
  double acc = 0.0;
  for (int m = 0; m < d; ++m) acc = fma(wa[m], A_a[m * d + c], acc);
  for (int m = 0; m < d; ++m) acc = fma(wb[m], A_b[m * d + c], acc);
  return acc;
}

}  // namespace merge
}  // namespace saga
