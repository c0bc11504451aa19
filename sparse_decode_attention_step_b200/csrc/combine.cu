// Merge per-split online-softmax states (m_s, l_s, acc_s) of one (b, j):
//   out = sum_s e^{m_s - m} acc_s / sum_s e^{m_s - m} l_s,  m = max_s m_s,
// the split-l_kv form of Eq. (7) (and of Eq. 2-4 for the dense kernel).
// Splits that kept nothing carry m_s = -inf and drop out; if every split is
// empty the output row is zero. A split whose record carries a negative
// count (a step that gave up on a bounded wait) makes the row NaN and its
// count -1.
//
// One CTA of 512 threads per (b, j). The split maximum is a block-wide
// reduction; then warp w sums splits w, w + 16, ... with each lane owning
// d/32 elements and eight splits' loads in flight, and the warps' sums are
// added in shared memory in warp order. Launched with programmatic stream
// serialisation, so its launch overlaps the tail of the split kernel.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;
constexpr float kLog2e = 1.4426950408889634f;

template <int VPL>
__device__ __forceinline__ void load_slice(const float *p, float (&v)[VPL]) {
  if constexpr (VPL == 2) {
    const float2 x = *reinterpret_cast<const float2 *>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const float *__restrict__ partials, const int32_t *__restrict__ l_kv,
               float *__restrict__ out, int32_t *__restrict__ sel_count, int32_t *abort_word,
               int h_q, int S, int64_t split_len, int64_t cap, int64_t max_l_kv) {
  constexpr int VPL = D / 32;                  // output elements per lane
  constexpr int R = D + kRecPad;
  __shared__ float red[kWarps];
  __shared__ int bad[kWarps];
  __shared__ float part_a[kWarps][D];
  __shared__ float part_l[kWarps];
  __shared__ int part_n[kWarps];
  pdl_wait();
  pdl_trigger();
  const int bj = blockIdx.x;
  const int b = bj / h_q;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t L = l_kv[b];
  const int64_t hi = cap < max_l_kv ? cap : max_l_kv;
  if (L < 0) L = 0;
  if (L > hi) L = hi;
  const int s_act = static_cast<int>((L + split_len - 1) / split_len);
  const float *rec = partials + static_cast<int64_t>(bj) * S * R;

  float m = -INFINITY;
  bool poison = false;
  for (int s = tid; s < s_act; s += kThreads) {
    const float4 x = *reinterpret_cast<const float4 *>(rec + static_cast<int64_t>(s) * R);
    m = fmaxf(m, x.x);
    poison |= __float_as_int(x.z) < 0;
  }
  m = warp_max(m);
  poison = __any_sync(0xffffffffu, poison);
  if (lane == 0) { red[warp] = m; bad[warp] = poison ? 1 : 0; }
  __syncthreads();
  m = red[0];
  int any_bad = bad[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) { m = fmaxf(m, red[w]); any_bad |= bad[w]; }

  float a[VPL], l = 0.f;
  int cnt = 0;
#pragma unroll
  for (int e = 0; e < VPL; ++e) a[e] = 0.f;
  for (int s0 = warp; s0 < s_act; s0 += kWarps * kUnroll) {
    float4 hd[kUnroll];
    float v[kUnroll][VPL];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int s = s0 + k * kWarps;
      if (s < s_act) {
        const float *r = rec + static_cast<int64_t>(s) * R;
        hd[k] = *reinterpret_cast<const float4 *>(r);
        load_slice<VPL>(r + kRecPad + lane * VPL, v[k]);
      } else {
        hd[k] = make_float4(-INFINITY, 0.f, 0.f, 0.f);
#pragma unroll
        for (int e = 0; e < VPL; ++e) v[k][e] = 0.f;
      }
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const float w = (m == -INFINITY || hd[k].x == -INFINITY) ? 0.f : exp2f((hd[k].x - m) * kLog2e);
      l = fmaf(w, hd[k].y, l);
      cnt += __float_as_int(hd[k].z);
#pragma unroll
      for (int e = 0; e < VPL; ++e) a[e] = fmaf(w, v[k][e], a[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < VPL; ++e) part_a[warp][lane * VPL + e] = a[e];
  if (lane == 0) { part_l[warp] = l; part_n[warp] = cnt; }
  __syncthreads();
  if (tid < D) {
    float at = 0.f, lt = 0.f;
    int nt = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) { at += part_a[w][tid]; lt += part_l[w]; nt += part_n[w]; }
    float o = lt > 0.f ? at / lt : 0.f;
    if (any_bad) {
      o = __int_as_float(0x7fc00000);
      nt = -1;
    }
    out[static_cast<int64_t>(bj) * D + tid] = o;
    if (tid == 0 && sel_count != nullptr) sel_count[bj] = nt;
  }
  // the step is over (its gather read the abort word before this launch
  // began): clear the word for the next step
  if (abort_word != nullptr && bj == 0 && tid == 0) *abort_word = 0;
}

}  // namespace

cudaError_t launch_combine(const float *partials, const int32_t *l_kv, int32_t *abort_word,
                           float *out, int32_t *sel_count, int B, int h_q, int d, int S,
                           int64_t split_len, int64_t cap, int64_t max_l_kv,
                           cudaStream_t st) {
  const dim3 grid(B * h_q), block(kThreads);
  if (d == 64)
    return launch_pdl(combine_kernel<64>, grid, block, 0, st, partials, l_kv, out, sel_count,
                      abort_word, h_q, S, split_len, cap, max_l_kv);
  if (d == 128)
    return launch_pdl(combine_kernel<128>, grid, block, 0, st, partials, l_kv, out, sel_count,
                      abort_word, h_q, S, split_len, cap, max_l_kv);
  return cudaErrorInvalidValue;
}

}  // namespace saga
