// Merge per-split online-softmax states (m_s, l_s, acc_s) of one (b, j):
//   out = sum_s e^{m_s - m} acc_s / sum_s e^{m_s - m} l_s,  m = max_s m_s,
// the split-l_kv form of Eq. (7) (and of Eq. 2-4 for the dense kernel).
// Splits that kept nothing carry m_s = -inf and drop out; if every split is
// empty the output row is zero.
//
// One CTA of 512 threads per (b, j): the split maximum is a block-wide
// reduction, then 512 / d groups of d threads each sum every (512/d)-th split
// for one output element (four splits' loads in flight per thread), and the
// groups' sums are added in shared memory. With one or two sequences the
// step plans a hundred or more splits per row, so this loop is the part of
// the call that does not shrink with the cache.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const float *__restrict__ partials, const int32_t *__restrict__ l_kv,
               float *__restrict__ out, int32_t *__restrict__ sel_count, int h_q, int S,
               int64_t split_len, int64_t cap, int64_t max_l_kv) {
  constexpr int NG = kThreads / D;             // split groups
  __shared__ float red[kThreads / 32];
  __shared__ float part_a[NG][D];
  __shared__ float part_l[NG];
  __shared__ int part_n[NG];
  const int bj = blockIdx.x;
  const int b = bj / h_q;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t L = l_kv[b];
  const int64_t hi = cap < max_l_kv ? cap : max_l_kv;
  if (L < 0) L = 0;
  if (L > hi) L = hi;
  const int s_act = static_cast<int>((L + split_len - 1) / split_len);
  const float *rec = partials + static_cast<int64_t>(bj) * S * (D + kRecPad);

  float m = -INFINITY;
  for (int s = tid; s < s_act; s += kThreads) m = fmaxf(m, rec[s * (D + kRecPad)]);
  m = warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);

  const int g = tid / D, i = tid % D;
  float a = 0.f, l = 0.f;
  int cnt = 0;
#pragma unroll 4
  for (int s = g; s < s_act; s += NG) {
    const float *r = rec + s * (D + kRecPad);
    cnt += __float_as_int(r[2]);
    const float w = m == -INFINITY ? 0.f : exp2f((r[0] - m) * kLog2e);
    l = fmaf(w, r[1], l);
    a = fmaf(w, r[kRecPad + i], a);
  }
  part_a[g][i] = a;
  if (i == 0) { part_l[g] = l; part_n[g] = cnt; }
  __syncthreads();
  if (tid < D) {
    float at = 0.f, lt = 0.f;
    int nt = 0;
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) { at += part_a[gg][tid]; lt += part_l[gg]; nt += part_n[gg]; }
    out[static_cast<int64_t>(bj) * D + tid] = lt > 0.f ? at / lt : 0.f;
    if (tid == 0 && sel_count != nullptr) sel_count[bj] = nt;
  }
}

}  // namespace

cudaError_t launch_combine(const float *partials, const int32_t *l_kv, int32_t *err,
                           float *out, int32_t *sel_count, int B, int h_q, int d, int S,
                           int64_t split_len, int64_t cap, int64_t max_l_kv,
                           cudaStream_t st) {
  (void)err;
  const int grid = B * h_q;
  if (d == 64)
    combine_kernel<64><<<grid, kThreads, 0, st>>>(partials, l_kv, out, sel_count, h_q, S,
                                                  split_len, cap, max_l_kv);
  else if (d == 128)
    combine_kernel<128><<<grid, kThreads, 0, st>>>(partials, l_kv, out, sel_count, h_q, S,
                                                   split_len, cap, max_l_kv);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace saga
