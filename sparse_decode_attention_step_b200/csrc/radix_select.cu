// Exact N-th largest score per row (Atop-N item 2: the exact threshold that
// is reused between refreshes), by MSB-first radix selection over the
// order-preserving uint32 keys of the fp32 scores.
//
// Pass p fixes bits [31-8p .. 24-8p] of the answer: a 256-bin histogram of
// that digit over the elements whose higher bits equal the prefix fixed so
// far, then a scan from the top bin down to the bin that holds the
// remaining rank. After four passes the prefix is the full key of an
// element of the row, so tau is always one of the row's own scores.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
radix_select_kernel(const float *__restrict__ scores, int64_t row_stride,
                    const int32_t *__restrict__ l_kv, int32_t *err, int N,
                    float *__restrict__ tau, int h_q, int64_t cap, int64_t max_l_kv) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_rem;
  const int bj = blockIdx.x;
  const int b = bj / h_q;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t L = l_kv[b];
  const int64_t hi = cap < max_l_kv ? cap : max_l_kv;
  if (L < 0) L = 0;
  if (L > hi) L = hi;
  if (static_cast<int64_t>(N) >= L) {
    if (tid == 0) tau[bj] = -INFINITY;
    return;
  }
  const float *row = scores + static_cast<int64_t>(bj) * row_stride;
  uint32_t prefix = 0, mask = 0, rem = static_cast<uint32_t>(N);

  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int64_t t0 = 0; t0 < L; t0 += kThreads) {
      const int64_t t = t0 + tid;
      bool in = false;
      uint32_t bin = 0;
      if (t < L) {
        const uint32_t k = order_key(row[t]);
        in = (k & mask) == prefix;
        bin = (k >> shift) & 0xFFu;
      }
      const uint32_t active = __ballot_sync(0xffffffffu, in);
      if (in) {
        // one shared atomic per distinct bin in the warp
        const uint32_t peers = __match_any_sync(active, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) { c[e] = hist[255 - 8 * lane - e]; sum += c[e]; }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= rem);
      const int owner = __ffs(hit) - 1;   // rem <= count of the prefix bucket, so hit != 0
      if (lane == owner) {
        uint32_t cum = incl - sum;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (cum + c[e] >= rem) {
            s_digit = 255 - 8 * lane - e;
            s_rem = rem - cum;
            break;
          }
          cum += c[e];
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 0xFFu << shift;
    rem = s_rem;
    __syncthreads();
  }
  if (tid == 0) tau[bj] = from_order_key(prefix);
}

}  // namespace

cudaError_t launch_radix_select(const float *scores, int64_t row_stride, const int32_t *l_kv,
                                int32_t *err, int N, float *tau, int B, int h_q, int64_t cap,
                                int64_t max_l_kv, cudaStream_t st) {
  radix_select_kernel<<<B * h_q, kThreads, 0, st>>>(scores, row_stride, l_kv, err, N, tau, h_q,
                                                   cap, max_l_kv);
  return cudaGetLastError();
}

}  // namespace saga
