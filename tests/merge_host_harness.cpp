// Host build of the key-merge routines the CUDA kernels run (merge_math.cuh),
// for the CPU tests: one thread plays the whole team, so every result is the
// one the device computes from the same float64 inputs. Test infrastructure;
// the library never links it.
#include <stdint.h>
#include <stdlib.h>

#include <vector>

#include "merge_math.cuh"

using namespace saga::merge;

extern "C" {

// Eigen-decomposition of the symmetric d x d S (overwritten: lambda on the
// diagonal); E receives the eigenvectors as rows. Returns the sweeps run.
int km_host_jacobi(int d, double *S, double *E) {
  std::vector<double> rc(d / 2), rs(d / 2), rowbuf(d);
  const Team tm{0, 1};
  return jacobi_eigh<double>(tm, d, S, E, rc.data(), rs.data(), rowbuf.data(), kMaxSweeps,
                             kJacobiTol);
}

// The (p, q) slots of every round of a sweep: out [d-1][d/2][2].
void km_host_rounds(int d, int32_t *out) {
  for (int r = 0; r < d - 1; ++r)
    for (int k = 0; k < d / 2; ++k) {
      int p, q;
      round_pair(d, r, k, p, q);
      out[(r * (d / 2) + k) * 2] = p;
      out[(r * (d / 2) + k) * 2 + 1] = q;
    }
}

// The per-pair stage as the pair kernel runs it (direct = 1; 0 forces the
// eigen-decomposition); vt_float selects the float eigenvector storage of the
// d = 128 kernel. Ag receives A_a, A_b [2][d][d]; *path 0 for the inverse,
// else the Jacobi sweeps.
double km_host_pair(int d, int vt_float, int direct, const double *Sa, const double *Sb,
                    const double *C, long long hd, int a, int b, double rcond, double *Ag,
                    int *path) {
  std::vector<double> S(d * d), rc(d / 2), rs(d / 2), rowbuf(d), inv(d);
  const Team tm{0, 1};
  if (vt_float) {
    std::vector<float> E(d * d);
    return pair_stage<float>(tm, d, Sa, Sb, C, hd, a, b, rcond, S.data(), E.data(), rc.data(),
                             rs.data(), rowbuf.data(), inv.data(), Ag, direct != 0, path);
  }
  std::vector<double> E(d * d);
  return pair_stage<double>(tm, d, Sa, Sb, C, hd, a, b, rcond, S.data(), E.data(), rc.data(),
                            rs.data(), rowbuf.data(), inv.data(), Ag, direct != 0, path);
}

// The matching kernel's programme on w [n][n]: pairs [n/2][2], total.
void km_host_match(int n, const double *w, int32_t *pairs, double *total) {
  std::vector<double> f(1u << n);
  std::vector<int8_t> choice(1u << n);
  const Team tm{0, 1};
  match_dp(tm, n, w, f.data(), choice.data());
  match_pairs(n, choice.data(), pairs);
  *total = f[(1u << n) - 1u];
}

// Column c of merged head rows: W_S[c][x] for x < d_model, from the widened
// teacher rows W_a [d][d_model], W_b [d][d_model] and A_a, A_b [d][d].
void km_host_merged(int d, int d_model, const double *W_a, const double *W_b,
                    const double *A_a, const double *A_b, double *out /* [d][d_model] */) {
  std::vector<double> wa(d), wb(d);
  for (int x = 0; x < d_model; ++x) {
    for (int m = 0; m < d; ++m) {
      wa[m] = W_a[m * d_model + x];
      wb[m] = W_b[m * d_model + x];
    }
    for (int c = 0; c < d; ++c) out[c * d_model + x] = merged_elem(d, wa.data(), wb.data(), A_a, A_b, c);
  }
}

int km_host_pair_index(int a, int b, int n) { return pair_index(a, b, n); }

void km_host_pair_of(int idx, int n, int32_t *ab) {
  int a, b;
  pair_of(idx, n, a, b);
  ab[0] = a;
  ab[1] = b;
}
}
