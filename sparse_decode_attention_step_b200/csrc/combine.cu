// Merge per-split online-softmax states (m_s, l_s, acc_s) of one (b, j):
//   out = sum_s e^{m_s - m} acc_s / sum_s e^{m_s - m} l_s,  m = max_s m_s,
// the split-l_kv form of Eq. (7) (and of Eq. 2-4 for the dense kernel).
// Splits that kept nothing carry m_s = -inf and drop out; if every split is
// empty the output row is zero.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__global__ void __launch_bounds__(D)
combine_kernel(const float *__restrict__ partials, const int32_t *__restrict__ l_kv,
               int32_t *err, float *__restrict__ out, int32_t *__restrict__ sel_count,
               int h_q, int S, int64_t split_len, int64_t cap, int64_t max_l_kv) {
  const int bj = blockIdx.x;
  const int b = bj / h_q;
  const int tid = threadIdx.x;
  int64_t L = l_kv[b];
  const int64_t hi = cap < max_l_kv ? cap : max_l_kv;
  if (L < 0) L = 0;
  if (L > hi) L = hi;
  const int s_act = static_cast<int>((L + split_len - 1) / split_len);
  const float *rec = partials + static_cast<int64_t>(bj) * S * (D + kRecPad);

  float m = -INFINITY;
  for (int s = 0; s < s_act; ++s) m = fmaxf(m, rec[s * (D + kRecPad)]);
  float l = 0.f, a = 0.f;
  int cnt = 0;
  for (int s = 0; s < s_act; ++s) {
    const float *r = rec + s * (D + kRecPad);
    cnt += __float_as_int(r[2]);
    if (m == -INFINITY) continue;
    const float w = exp2f((r[0] - m) * kLog2e);
    l = fmaf(w, r[1], l);
    a = fmaf(w, r[kRecPad + tid], a);
  }
  out[static_cast<int64_t>(bj) * D + tid] = l > 0.f ? a / l : 0.f;
  if (tid == 0 && sel_count != nullptr) sel_count[bj] = cnt;
}

}  // namespace

cudaError_t launch_combine(const float *partials, const int32_t *l_kv, int32_t *err,
                           float *out, int32_t *sel_count, int B, int h_q, int d, int S,
                           int64_t split_len, int64_t cap, int64_t max_l_kv,
                           cudaStream_t st) {
  const int grid = B * h_q;
  if (d == 64)
    combine_kernel<64><<<grid, 64, 0, st>>>(partials, l_kv, err, out, sel_count, h_q, S,
                                            split_len, cap, max_l_kv);
  else if (d == 128)
    combine_kernel<128><<<grid, 128, 0, st>>>(partials, l_kv, err, out, sel_count, h_q, S,
                                              split_len, cap, max_l_kv);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace saga
