// Exact N-th largest score per row (Atop-N item 2: the exact threshold that
// is reused between refreshes), by MSB-first radix selection over the
// order-preserving uint32 keys of the fp32 scores.
//
// Digit p (p = 0..3) is bits [31-8p .. 24-8p] of the answer: a 256-bin
// histogram of that digit over the elements whose higher bits equal the
// prefix fixed so far, then a scan from the top bin down to the bin that holds
// the remaining rank. After four digits the prefix is the full key of an
// element of the row, so tau is always one of the row's own scores.
//
// One CTA of 512 threads per row, two CTAs per SM, launched with programmatic
// stream serialisation after the score pass. Digit 0 comes from the histogram the score pass already
// built (or from one pass over the row). A second pass over the row fixes
// digit 1 and copies the keys of the digit-0 bucket into shared memory; the
// last two digits are found there. When that bucket does not fit (its scores
// share one binade), a third pass copies only the keys that match the first
// two digits; only if even those do not fit, digits 2 and 3 take one pass
// over the row each.
//
// Exact top-N (Eq. 6 with ties to the lower position) also needs, when tau is
// tied, how far along the row the taken ties reach: after the last digit the
// rank left inside tau's bucket is the number k of entries equal to tau that
// the N largest include, and one more pass in position order finds the
// position of the k-th of them.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2;                       // two rows streamed per SM at a time
constexpr int kCand = 16384;                        // candidate keys kept on chip (64 KB)
constexpr int kWarps = kThreads / 32;
constexpr int kMaxDevices = 64;

struct Shared {
  uint32_t hist[256];
  uint32_t digit, rem, n_cand;
  uint32_t wsum[kWarps];
  int32_t found;
};

// Histogram of digit `shift` over keys with (k & mask) == prefix, one shared
// atomic per distinct bin in a warp. All threads of the CTA call it.
__device__ __forceinline__ void count_key(uint32_t k, bool valid, uint32_t mask, uint32_t prefix,
                                          int shift, uint32_t *hist, int lane) {
  const bool in = valid && (k & mask) == prefix;
  const uint32_t active = __ballot_sync(0xffffffffu, in);
  if (in) {
    const uint32_t bin = (k >> shift) & 0xFFu;
    const uint32_t peers = __match_any_sync(active, bin);
    if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
  }
}

// Warp 0 finds the bin holding rank `rem` (1-based, counted from the top)
// and stores it with the rank left inside that bin.
__device__ __forceinline__ void pick_digit(Shared &sh, int lane) {
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) { c[e] = sh.hist[255 - 8 * lane - e]; sum += c[e]; }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t rem = sh.rem;
  const uint32_t hit = __ballot_sync(0xffffffffu, incl >= rem);
  const int owner = __ffs(hit) - 1;                 // rem <= bucket count, so hit != 0
  if (lane == owner) {
    uint32_t cum = incl - sum;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (cum + c[e] >= rem) {
        sh.digit = 255 - 8 * lane - e;
        sh.rem = rem - cum;
        break;
      }
      cum += c[e];
    }
  }
}

// Visit a row in steps of kThreads * kVec * 4 elements, all threads of the
// CTA in step: f(v, t0) gets this thread's kVec * 4 values, v[u][e] being
// element elem_index(t0, tid, u, e); elements at or past L read as 0 and the
// visitor checks the index against L. 16-byte loads when the row is 16-byte
// aligned; kVec * 16 bytes in flight per thread.
constexpr int kVec = 4;
constexpr int64_t kStep = static_cast<int64_t>(kThreads) * kVec * 4;

__device__ __forceinline__ int64_t elem_index(int64_t t0, int tid, int u, int e) {
  return t0 + (static_cast<int64_t>(u) * kThreads + tid) * 4 + e;
}

template <typename F>
__device__ __forceinline__ void for_row_steps(const float *row, int64_t L, int tid, F f) {
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  for (int64_t t0 = 0; t0 < L; t0 += kStep) {
    float v[kVec][4];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int64_t i = elem_index(t0, tid, u, 0);
      if (vec && i + 3 < L) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(row + i));
        v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[u][e] = i + e < L ? __ldg(row + i + e) : 0.f;
      }
    }
    f(v, t0);
  }
}

// Element-wise visit: f(key, valid) for every element of the row.
template <typename F>
__device__ __forceinline__ void for_row(const float *row, int64_t L, int tid, F f) {
  for_row_steps(row, L, tid, [&](const float (&v)[kVec][4], int64_t t0) {
#pragma unroll
    for (int u = 0; u < kVec; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) f(order_key(v[u][e]), elem_index(t0, tid, u, e) < L);
  });
}

// Copy the keys of the row with (key & mask) == prefix into cand (as many as
// fit; the returned count may exceed kCand) and, when `shift` >= 0, count
// digit `shift` of those keys into hist. One shared atomic per warp and step
// reserves the warp's candidate slots.
__device__ __forceinline__ void collect(const float *row, int64_t L, int tid, int lane,
                                        uint32_t mask, uint32_t prefix, int shift, Shared &sh,
                                        uint32_t *cand) {
  for_row_steps(row, L, tid, [&](const float (&v)[kVec][4], int64_t t0) {
    uint32_t c = 0;
#pragma unroll
    for (int u = 0; u < kVec; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        c += (elem_index(t0, tid, u, e) < L && (order_key(v[u][e]) & mask) == prefix) ? 1u : 0u;
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    if (total != 0u) {
      uint32_t base = 0;
      if (lane == 31) base = atomicAdd(&sh.n_cand, total);
      uint32_t at = __shfl_sync(0xffffffffu, base, 31) + incl - c;
#pragma unroll
      for (int u = 0; u < kVec; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t k = order_key(v[u][e]);
          const bool in = elem_index(t0, tid, u, e) < L && (k & mask) == prefix;
          if (in) {
            if (at < static_cast<uint32_t>(kCand)) cand[at] = k;
            ++at;
          }
          if (shift >= 0) count_key(k, in, 0u, 0u, shift, sh.hist, lane);
        }
    }
  });
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
radix_select_kernel(const float *__restrict__ scores, int64_t row_stride,
                    const int32_t *__restrict__ l_kv, int N, float *__restrict__ tau, int h_q,
                    int64_t cap, int64_t max_l_kv, const uint32_t *__restrict__ hist0,
                    int32_t *__restrict__ tie) {
  __shared__ Shared sh;
  extern __shared__ uint32_t cand[];
  pdl_wait();
  pdl_trigger();
  const int bj = blockIdx.x;
  const int b = bj / h_q;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t L = l_kv[b];
  const int64_t hi = cap < max_l_kv ? cap : max_l_kv;
  if (L < 0) L = 0;
  if (L > hi) L = hi;
  if (static_cast<int64_t>(N) >= L) {
    if (tid == 0) {
      tau[bj] = -INFINITY;
      if (tie != nullptr) tie[bj] = INT32_MAX;
    }
    return;
  }
  const float *row = scores + static_cast<int64_t>(bj) * row_stride;
  if (tid == 0) { sh.rem = static_cast<uint32_t>(N); sh.n_cand = 0; }

  // ---- digit 0: from the score pass's histogram, or one pass here ---------
  if (hist0 != nullptr) {
    for (int i = tid; i < 256; i += kThreads) sh.hist[i] = hist0[static_cast<int64_t>(bj) * 256 + i];
    __syncthreads();
  } else {
    for (int i = tid; i < 256; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    for_row(row, L, tid, [&](uint32_t k, bool valid) {
      count_key(k, valid, 0u, 0u, 24, sh.hist, lane);
    });
    __syncthreads();
  }
  if (warp == 0) pick_digit(sh, lane);
  __syncthreads();
  uint32_t prefix = sh.digit << 24, mask = 0xFF000000u;
  __syncthreads();

  // ---- digit 1: one pass over the row; keep the digit-0 bucket on chip -----
  for (int i = tid; i < 256; i += kThreads) sh.hist[i] = 0u;
  __syncthreads();
  collect(row, L, tid, lane, mask, prefix, 16, sh, cand);
  __syncthreads();
  if (warp == 0) pick_digit(sh, lane);
  __syncthreads();
  prefix |= sh.digit << 16;
  mask |= 0x00FF0000u;
  uint32_t n_cand = sh.n_cand;
  bool on_chip = n_cand <= static_cast<uint32_t>(kCand);
  __syncthreads();
  if (!on_chip) {
    // the top-byte bucket was too big: collect the (much smaller) bucket of
    // the 16-bit prefix instead, with one more pass over the row
    if (tid == 0) sh.n_cand = 0;
    __syncthreads();
    collect(row, L, tid, lane, mask, prefix, -1, sh, cand);
    __syncthreads();
    n_cand = sh.n_cand;
    on_chip = n_cand <= static_cast<uint32_t>(kCand);
    __syncthreads();
  }

  // ---- digits 2 and 3: over the candidates, else over the row -------------
  for (int shift = 8; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    if (on_chip) {
      for (uint32_t i0 = 0; i0 < n_cand; i0 += kThreads) {
        const uint32_t i = i0 + tid;
        const uint32_t k = i < n_cand ? cand[i] : 0u;
        count_key(k, i < n_cand, mask, prefix, shift, sh.hist, lane);
      }
    } else {
      for_row(row, L, tid, [&](uint32_t k, bool valid) {
        count_key(k, valid, mask, prefix, shift, sh.hist, lane);
      });
    }
    __syncthreads();
    if (warp == 0) pick_digit(sh, lane);
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  if (tid == 0) tau[bj] = from_order_key(prefix);
  if (tie == nullptr) return;

  // ---- position of the k-th entry equal to tau, in position order -------
  const uint32_t k = sh.rem;                    // 1 <= k <= #(entries equal to tau)
  if (tid == 0) sh.found = -1;
  __syncthreads();
  uint32_t before = 0;                          // matches in earlier chunks
  constexpr int64_t kSpan = static_cast<int64_t>(kThreads) * 4;
  for (int64_t t0 = 0; t0 < L; t0 += kSpan) {
    const int64_t i = t0 + static_cast<int64_t>(tid) * 4;
    uint32_t hits = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (i + e < L && order_key(row[i + e]) == prefix) hits |= 1u << e;
    const uint32_t c = __popc(hits);
    // exclusive prefix of c over the CTA, in thread (= position) order
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) sh.wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      uint32_t ws = lane < kWarps ? sh.wsum[lane] : 0u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += y;
      }
      if (lane < kWarps) sh.wsum[lane] = ws;    // inclusive over warps
    }
    __syncthreads();
    const uint32_t excl = before + (warp > 0 ? sh.wsum[warp - 1] : 0u) + (incl - c);
    if (c > 0 && excl < k && k <= excl + c) {
      uint32_t need = k - excl, hh = hits;
      while (--need) hh &= hh - 1u;
      sh.found = static_cast<int32_t>(i + __ffs(hh) - 1);
    }
    before += sh.wsum[kWarps - 1];
    __syncthreads();
    if (sh.found >= 0) break;
  }
  if (tid == 0) tie[bj] = sh.found;
}

}  // namespace

cudaError_t launch_radix_select(const float *scores, int64_t row_stride, const int32_t *l_kv,
                                int N, float *tau, int B, int h_q, int64_t cap, int64_t max_l_kv,
                                const uint32_t *hist0, int32_t *tie, cudaStream_t st) {
  // the dynamic shared-memory opt-in is per device; set once on each
  static std::atomic<bool> attr_set[kMaxDevices];
  const int smem = kCand * static_cast<int>(sizeof(uint32_t));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(radix_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  return launch_pdl(radix_select_kernel, dim3(B * h_q), dim3(kThreads), smem, st, scores,
                    row_stride, l_kv, N, tau, h_q, cap, max_l_kv, hist0, tie);
}

}  // namespace saga
