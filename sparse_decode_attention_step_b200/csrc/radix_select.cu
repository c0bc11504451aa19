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
// Digit 0 comes from the histogram the score pass already built (or from one
// pass over the row). With that histogram, a collect kernel spread over the
// whole GPU (about two CTAs per SM, each on one segment of a row) reads every
// row once, lists the keys of its digit-0 bucket (the keys that share the
// N-th largest's top byte: a few percent of an attention score row, up to a
// third when the N-th largest lies just below a power of two, since the top
// byte spans two binades) in global memory and counts their digit 1. Then
// one CTA of 512 threads per row takes digit 1 from that count, reads the
// list once to keep the keys of the 16-bit prefix (tens to hundreds) in
// shared memory, and finds the last two digits there. Without the histogram
// (or when the bucket overflows its list, half a row), a pass over the row
// fixes digit 1 and keeps the digit-0 bucket on chip; when that does not
// fit, a second pass keeps the 16-bit prefix's keys; only if even those do
// not fit, digits 2 and 3 take one pass each. Both kernels are launched with
// programmatic stream serialisation after the score pass.
//
// Exact top-N (Eq. 6 with ties to the lower position) also needs, when tau is
// tied, how far along the row the taken ties reach: after the last digit the
// rank left inside tau's bucket is the number k of entries equal to tau that
// the N largest include, and one more pass in position order finds the
// position of the k-th of them.
#include <algorithm>
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

// Append k to cand when `in` (as many as fit; sh.n_cand counts them all).
// All lanes of the warp call it together.
__device__ __forceinline__ void append(uint32_t k, bool in, int lane, Shared &sh, uint32_t *cand) {
  const uint32_t bal = __ballot_sync(0xffffffffu, in);
  if (bal == 0u) return;
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(&sh.n_cand, static_cast<uint32_t>(__popc(bal)));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (in) {
    const uint32_t at = base + __popc(bal & ((1u << lane) - 1u));
    if (at < static_cast<uint32_t>(kCand)) cand[at] = k;
  }
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

// The digit-0 bucket of a row (the keys whose top byte is that of the N-th
// largest, found from the score pass's histogram), collected by `segs` CTAs
// per row, each reading one segment of the row once: the keys go to the
// row's list in global memory (gcap of them at most; the count may exceed
// it, and the select then reads the row itself), one global atomic per warp
// and step reserving the warp's places, and their digit 1 is counted into
// the row's histogram hist1 (per-warp shared bins, added to hist1 at the
// end). The list's order depends on timing; the select uses it as a
// multiset only.
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
radix_collect_kernel(const float *__restrict__ scores, int64_t row_stride,
                     const int32_t *__restrict__ l_kv, int N, int h_q, int64_t cap,
                     int64_t max_l_kv, const uint32_t *__restrict__ hist0,
                     uint32_t *__restrict__ gcand, uint32_t *__restrict__ gcount,
                     uint32_t *__restrict__ hist1, int gcap, int segs) {
  __shared__ Shared sh;
  __shared__ uint32_t h1[kWarps][256];
  pdl_wait();
  pdl_trigger();
  const int bj = blockIdx.x / segs, seg = blockIdx.x % segs;
  const int b = bj / h_q;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t L = l_kv[b];
  const int64_t hi = cap < max_l_kv ? cap : max_l_kv;
  if (L < 0) L = 0;
  if (L > hi) L = hi;
  if (static_cast<int64_t>(N) >= L) return;
  const int64_t span = (L + segs - 1) / segs;
  const int64_t t_lo = min(L, (span + 15) / 16 * 16 * seg);
  const int64_t t_hi = min(L, t_lo + (span + 15) / 16 * 16);
  if (t_lo >= t_hi) return;
  if (tid == 0) sh.rem = static_cast<uint32_t>(N);
  for (int i = tid; i < 256; i += kThreads) sh.hist[i] = hist0[static_cast<int64_t>(bj) * 256 + i];
  for (int i = tid; i < kWarps * 256; i += kThreads) (&h1[0][0])[i] = 0u;
  __syncthreads();
  if (warp == 0) pick_digit(sh, lane);
  __syncthreads();
  const uint32_t d0 = sh.digit;
  const float *row = scores + static_cast<int64_t>(bj) * row_stride + t_lo;
  const int64_t len = t_hi - t_lo;
  uint32_t *dst = gcand + static_cast<int64_t>(bj) * gcap;
  uint32_t *mine = h1[warp];
  for_row_steps(row, len, tid, [&](const float (&v)[kVec][4], int64_t t0) {
    const bool full = t0 + kStep <= len;
    uint32_t key[kVec * 4], in = 0;
#pragma unroll
    for (int u = 0; u < kVec; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        key[u * 4 + e] = order_key(v[u][e]);
        const bool valid = full || elem_index(t0, tid, u, e) < len;
        if (valid && (key[u * 4 + e] >> 24) == d0) in |= 1u << (u * 4 + e);
      }
    const uint32_t c = __popc(in);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    if (total == 0u) return;
    uint32_t base = 0;
    if (lane == 31) base = atomicAdd(gcount + bj, total);
    uint32_t at = __shfl_sync(0xffffffffu, base, 31) + incl - c;
#pragma unroll
    for (int x = 0; x < kVec * 4; ++x) {
      if ((in >> x) & 1u) {
        if (at < static_cast<uint32_t>(gcap)) dst[at] = key[x];
        ++at;
        atomicAdd(&mine[(key[x] >> 16) & 0xFFu], 1u);
      }
    }
  });
  __syncthreads();
  uint32_t *h1_row = hist1 + static_cast<int64_t>(bj) * 256;
  for (int i = tid; i < 256; i += kThreads) {
    uint32_t sum = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sum += h1[w][i];
    if (sum != 0u) atomicAdd(h1_row + i, sum);
  }
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
radix_select_kernel(const float *__restrict__ scores, int64_t row_stride,
                    const int32_t *__restrict__ l_kv, int N, float *__restrict__ tau, int h_q,
                    int64_t cap, int64_t max_l_kv, const uint32_t *__restrict__ hist0,
                    int32_t *__restrict__ tie, const uint32_t *__restrict__ gcand,
                    const uint32_t *__restrict__ gcount, const uint32_t *__restrict__ hist1,
                    int gcap) {
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

  // ---- digit 1, and the keys kept on chip ---------------------------------
  // With the collect kernel's list of the digit-0 bucket (when it fit) and
  // its digit-1 histogram, digit 1 needs no pass; the list is read once to
  // keep the keys of the 16-bit prefix on chip. Otherwise one pass over the
  // row fixes digit 1 and keeps the digit-0 bucket on chip.
  const uint32_t n_g = gcand != nullptr ? gcount[bj] : 0xFFFFFFFFu;
  const bool listed = n_g <= static_cast<uint32_t>(gcap);
  const uint32_t *list = listed ? gcand + static_cast<int64_t>(bj) * gcap : nullptr;
  // visit the list (16-byte loads, kVec per thread in flight) or the row
  auto for_src = [&](auto f) {
    if (listed) {
      const uint4 *l4 = reinterpret_cast<const uint4 *>(list);
      const uint32_t n4 = (n_g + 3u) / 4u;            // within gcap (a multiple of 4)
      for (uint32_t i0 = 0; i0 < n4; i0 += kThreads * kVec) {
        uint4 x[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
          const uint32_t i = i0 + u * kThreads + tid;
          x[u] = i < n4 ? __ldcg(l4 + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
          const uint32_t i = (i0 + u * kThreads + tid) * 4u;
          f(x[u].x, i < n_g);
          f(x[u].y, i + 1u < n_g);
          f(x[u].z, i + 2u < n_g);
          f(x[u].w, i + 3u < n_g);
        }
      }
    } else {
      for_row(row, L, tid, f);
    }
  };
  uint32_t n_cand;
  if (listed) {
    for (int i = tid; i < 256; i += kThreads) sh.hist[i] = hist1[static_cast<int64_t>(bj) * 256 + i];
    __syncthreads();
    if (warp == 0) pick_digit(sh, lane);
    __syncthreads();
    prefix |= sh.digit << 16;
    mask |= 0x00FF0000u;
    for_src([&](uint32_t k, bool valid) {
      append(k, valid && (k & mask) == prefix, lane, sh, cand);
    });
    __syncthreads();
    n_cand = sh.n_cand;
  } else {
    for (int i = tid; i < 256; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    collect(row, L, tid, lane, mask, prefix, 16, sh, cand);
    __syncthreads();
    if (warp == 0) pick_digit(sh, lane);
    __syncthreads();
    prefix |= sh.digit << 16;
    mask |= 0x00FF0000u;
    n_cand = sh.n_cand;
    __syncthreads();
    if (n_cand > static_cast<uint32_t>(kCand)) {
      // the top-byte bucket was too big: keep the (much smaller) bucket of
      // the 16-bit prefix instead, with one more pass over the row
      if (tid == 0) sh.n_cand = 0;
      __syncthreads();
      collect(row, L, tid, lane, mask, prefix, -1, sh, cand);
      __syncthreads();
      n_cand = sh.n_cand;
    }
  }
  const bool on_chip = n_cand <= static_cast<uint32_t>(kCand);
  __syncthreads();

  // ---- digits 2 and 3: over the keys on chip, else over the list or row ---
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
      for_src([&](uint32_t k, bool valid) {
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
                                const uint32_t *hist0, int32_t *tie, uint32_t *gcand,
                                uint32_t *gcount, uint32_t *hist1, int gcap, int sms,
                                cudaStream_t st) {
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
  const int rows = B * h_q;
  const bool two_pass = hist0 != nullptr && gcand != nullptr && gcount != nullptr &&
                        hist1 != nullptr && gcap > 0 && gcap % 4 == 0;
  if (two_pass) {
    // enough segments per row to give every SM two CTAs, each at least 16K positions long
    const int64_t by_sms = std::max<int64_t>(1, static_cast<int64_t>(kCtasPerSm) * sms / rows);
    const int64_t by_len = std::max<int64_t>(1, max_l_kv / 16384);
    const int segs = static_cast<int>(std::min(by_sms, by_len));
    e = launch_pdl(radix_collect_kernel, dim3(rows * segs), dim3(kThreads), 0, st, scores,
                   row_stride, l_kv, N, h_q, cap, max_l_kv, hist0, gcand, gcount, hist1, gcap,
                   segs);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(radix_select_kernel, dim3(rows), dim3(kThreads), smem, st, scores,
                    row_stride, l_kv, N, tau, h_q, cap, max_l_kv, hist0, tie,
                    two_pass ? gcand : nullptr, two_pass ? gcount : nullptr,
                    two_pass ? hist1 : nullptr, gcap);
}

}  // namespace saga
