// Tensor-core split kernel for bf16 caches (sm_100a): Eq. 2 scores,
// Atop-N item 1 compare and compaction, Eq. 7 sparse softmax + V gather, and
// per-split online-softmax states, with the score contraction on tcgen05.
//
// One CTA per (sequence b, key head kh, split of l_kv): eight compute warps
// and one TMA producer warp.
//
//   producer    K tiles of 128 positions x d (bf16, 128B swizzle) stream by
//               TMA into kStages shared-memory stages.
//   scan phase  the compute warps walk the split in 256-position chunks.
//               Thread 0 issues one chunk ahead the d/16 tcgen05.mma
//               (M=128 keys, N=16 heads, K=16) per tile into a double-
//               buffered TMEM accumulator; each thread then reads one key's
//               16 head scores, scales them by 1/sqrt(d), compares them with
//               tau and, for every head that keeps the key, appends (key,
//               score) to its warp's list of that head (one ballot per head).
//               The warps never hand tiles to one another; one barrier per
//               chunk guards the TMEM reuse.
//   gather      when the split is done (or a list is close to full) all
//               eight warps turn to the V rows: 32 groups of 8 lanes, two per
//               query head (one per half of the scan warps' lists), each lane
//               gathering 16-byte chunks of 4 kept rows per round, with an
//               online softmax per group. The two halves of each head merge
//               at the end into the split's (m, l, acc) record.
// Query heads beyond the group (G < 16) are zero rows of Q and never kept.
// Every wait is bounded; on a timeout the CTA sets SAGA_DEVERR_TIMEOUT, lets
// its copies and MMAs in flight land, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace saga {

namespace {

constexpr int kWarps = 8;                                  // compute warps
constexpr int kComputeThreads = kWarps * 32;
constexpr int kProducerWarp = kWarps;
constexpr int kThreads = kComputeThreads + 32;             // 288
constexpr int kTileKeys = 128;
constexpr int kChunkKeys = 2 * kTileKeys;
constexpr int kN = 16;                                     // MMA N: query heads, padded
constexpr int kTmemCols = 64;                              // 2 chunks x 2 tiles x 16 heads
constexpr int kBar = 1;                                    // named barrier of the compute warps
constexpr int kUnroll = 4;                                 // kept rows in flight per lane group
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(kTileKeys, kN);
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kStages = D == 64 ? 3 : 2;
  static constexpr int kBoxes = D / 64;                     // 64-column TMA boxes per tile
  static constexpr int kBoxBytes = kTileKeys * 128;         // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQBlockBytes = kN * 128;             // 16 rows x 128 bytes per box
  static constexpr int kQBytes = kBoxes * kQBlockBytes;
  static constexpr int kCap = D == 64 ? 48 : 40;           // kept keys per (head, warp) list
};

struct Header {
  uint64_t full[4], empty[4];
  uint64_t mma_done[2];
  uint32_t tmem_base;
  int abort;
};

template <int D>
struct Layout {
  static constexpr int off_stage = 0;
  static constexpr int off_q = Cfg<D>::kStages * Cfg<D>::kTileBytes;
  static constexpr int off_key = off_q + Cfg<D>::kQBytes;                // int [kN][kWarps][kCap]
  static constexpr int off_sc = off_key + kN * kWarps * Cfg<D>::kCap * 4; // float, same shape
  static constexpr int off_cnt = off_sc + kN * kWarps * Cfg<D>::kCap * 4; // int [kN][kWarps]
  static constexpr int off_tau = off_cnt + kN * kWarps * 4;
  static constexpr int off_hdr = off_tau + kN * 4;
  static constexpr int bytes = off_hdr + static_cast<int>(sizeof(Header));
  static constexpr int alloc = bytes + 1024;               // slack for 1024-byte alignment
};

__device__ __forceinline__ bool bar_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(kBar), "r"(kComputeThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void fail(const StepParams &p, Header *h) {
  atomicOr(p.err, SAGA_DEVERR_TIMEOUT);
  *reinterpret_cast<volatile int *>(&h->abort) = 1;
}

__device__ __forceinline__ bool aborted(Header *h) {
  return *reinterpret_cast<volatile int *>(&h->abort) != 0;
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = sm100::mbar_wait(bar, parity);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

template <int D, int GP>
__global__ void __launch_bounds__(kThreads, 2)
saga_tc_kernel(const StepParams p, const int mode, const __grid_constant__ CUtensorMap kmap) {
  using C = Cfg<D>;
  using Lo = Layout<D>;
  constexpr int CPL = D / 64;                // 16-byte chunks of a V row per gather lane
  constexpr int EPL = 8 * CPL;               // row elements per gather lane

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = sm100::smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t *stages = smem + Lo::off_stage;
  uint16_t *qop = reinterpret_cast<uint16_t *>(smem + Lo::off_q);
  int(*lkey)[kWarps][C::kCap] = reinterpret_cast<int(*)[kWarps][C::kCap]>(smem + Lo::off_key);
  float(*lsc)[kWarps][C::kCap] = reinterpret_cast<float(*)[kWarps][C::kCap]>(smem + Lo::off_sc);
  int(*lcnt)[kWarps] = reinterpret_cast<int(*)[kWarps]>(smem + Lo::off_cnt);
  float *tau_s = reinterpret_cast<float *>(smem + Lo::off_tau);
  Header *hdr = reinterpret_cast<Header *>(smem + Lo::off_hdr);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x;
  const int b = blockIdx.y / p.h_k, kh = blockIdx.y % p.h_k;
  const int G = p.h_q / p.h_k;
  const int j0 = kh * G;
  const int64_t L = clamp_len(p, b);
  const int64_t t_begin = static_cast<int64_t>(s) * p.split_len;
  if (t_begin >= L) return;                      // uniform, before any barrier or TMEM
  const int64_t t_end = min(t_begin + p.split_len, L);
  const int n_tiles = static_cast<int>((t_end - t_begin + kTileKeys - 1) / kTileKeys);
  const int n_chunks = (n_tiles + 1) / 2;

  // ---- set-up --------------------------------------------------------------
  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      sm100::mbar_init(&hdr->full[i], 1);
      sm100::mbar_init(&hdr->empty[i], 1);
    }
    sm100::mbar_init(&hdr->mma_done[0], 1);
    sm100::mbar_init(&hdr->mma_done[1], 1);
    hdr->abort = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&hdr->tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  {
    const uint16_t *qg = static_cast<const uint16_t *>(p.q) + b * p.q_sb;
    for (int idx = tid; idx < kN * D; idx += kThreads) {
      const int n = idx / D, k = idx % D;
      const uint16_t v = n < G ? qg[(j0 + n) * p.q_sh + k] : static_cast<uint16_t>(0);
      const int box = k / 64, kk = k % 64;
      const int off = box * C::kQBlockBytes + (n / 8) * 1024 + (n % 8) * 128 +
                      ((((kk * 2) >> 4) ^ (n % 8)) << 4) + ((kk * 2) & 15);
      qop[off / 2] = v;
    }
    sm100::fence_proxy_async_smem();
    if (tid < kN) tau_s[tid] = (tid < G && mode != kModeDump) ? p.tau[b * p.h_q + j0 + tid] : 0.f;
    if (mode == kModeDump && p.hist != nullptr) {
      // the head lists are unused when dumping: they hold the score histograms
      uint32_t *hs = reinterpret_cast<uint32_t *>(smem + Lo::off_key);
      for (int i = tid; i < kN * 256; i += kThreads) hs[i] = 0u;
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = hdr->tmem_base;

  // ---- TMA producer ---------------------------------------------------------
  if (warp == kProducerWarp) {
    if (lane == 0) {
      sm100::prefetch_tensormap(&kmap);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % C::kStages, round = i / C::kStages;
        if (aborted(hdr)) break;
        if (!sm100::mbar_wait(&hdr->empty[st], (round & 1) ^ 1)) { fail(p, hdr); break; }
        sm100::mbar_arrive_expect_tx(&hdr->full[st], C::kTileBytes);
        const int y = static_cast<int>(t_begin) + i * kTileKeys;
#pragma unroll
        for (int bx = 0; bx < C::kBoxes; ++bx)
          sm100::tma_load_4d(stages + st * C::kTileBytes + bx * C::kBoxBytes, &kmap,
                             &hdr->full[st], bx * 64, y, kh, b);
        issued = i + 1;
      }
      // every copy still in flight lands before the CTA can exit
      for (int i = issued > C::kStages ? issued - C::kStages : 0; i < issued; ++i)
        sm100::mbar_wait(&hdr->full[i % C::kStages], (i / C::kStages) & 1);
    }
    return;
  }

  // ---- compute warps --------------------------------------------------------
  const uint32_t q_u32 = sm100::smem_u32(qop);
  const uint32_t st_u32 = sm100::smem_u32(stages);
  // Thread 0: the MMAs of chunk c (its one or two tiles) into TMEM set c & 1.
  auto issue_chunk = [&](int c) -> bool {
    for (int u = 0; u < 2 && 2 * c + u < n_tiles; ++u) {
      const int tt = 2 * c + u;
      const int st = tt % C::kStages;
      if (!sm100::mbar_wait(&hdr->full[st], (tt / C::kStages) & 1)) return false;
      sm100::tc_fence_after();
      const uint32_t a0 = st_u32 + st * C::kTileBytes;
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        const int bx = j / 4, kk = j % 4;
        const uint64_t ad = sm100::desc_k_sw128(a0 + bx * C::kBoxBytes + kk * 32);
        const uint64_t bd = sm100::desc_k_sw128(q_u32 + bx * C::kQBlockBytes + kk * 32);
        sm100::mma_bf16(tmem_base + (c & 1) * 2 * kN + u * kN, ad, bd, kIdesc, j > 0 ? 1u : 0u);
      }
      sm100::mma_commit(&hdr->empty[st]);
    }
    sm100::mma_commit(&hdr->mma_done[c & 1]);
    return true;
  };

  const int64_t row0 = static_cast<int64_t>(b * p.h_q + j0) * p.row_stride;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int my_cnt = 0;                      // lane g < 16: this warp's kept keys of head g
  // gather role: lane group (part, head)
  const int unit = warp * 4 + (lane >> 3);
  const int gh = unit % kN, part = unit / kN, c8 = lane & 7;
  const bool live = gh < G && mode != kModeDump;
  const int vh = live ? ((j0 + gh) * p.h_v) / p.h_q : 0;
  const uint16_t *vrow = static_cast<const uint16_t *>(p.V) + b * p.v_sb + vh * p.v_sh;
  float m_run = -INFINITY, l_run = 0.f, acc[EPL];
  int cnt_run = 0;
#pragma unroll
  for (int v = 0; v < EPL; ++v) acc[v] = 0.f;

  // All compute warps: fold the kept keys of every list into the lane
  // groups' softmax states, then empty the lists.
  auto gather = [&]() {
    if (lane < kN) lcnt[lane][warp] = my_cnt;
    sm100::named_bar(kBar, kComputeThreads);
    int q1 = 0, q2 = 0, q3 = 0, ntot = 0;
    if (live) {
      const int w0 = 4 * part;
      q1 = lcnt[gh][w0];
      q2 = q1 + lcnt[gh][w0 + 1];
      q3 = q2 + lcnt[gh][w0 + 2];
      ntot = q3 + lcnt[gh][w0 + 3];
    }
    // entry e -> (list of scan warp w, slot)
    auto locate = [&](int e, int &w, int &slot) {
      const int k = (e >= q1) + (e >= q2) + (e >= q3);
      const int base = k == 0 ? 0 : (k == 1 ? q1 : (k == 2 ? q2 : q3));
      w = 4 * part + k;
      slot = e - base;
    };
    const int gq = live ? gh : 0;
    float mc = -INFINITY;
    for (int e = c8; e < ntot; e += 8) {
      int w, slot;
      locate(e, w, slot);
      mc = fmaxf(mc, lsc[gq][w][slot]);
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, off));
    const float m_new = fmaxf(m_run, mc);
    const float corr = m_new == -INFINITY ? 1.f : exp2f((m_run - m_new) * kLog2e);
    l_run *= corr;
#pragma unroll
    for (int v = 0; v < EPL; ++v) acc[v] *= corr;
    m_run = m_new;
    int nmax = ntot;
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) nmax = max(nmax, __shfl_xor_sync(0xffffffffu, nmax, off));
    for (int e0 = 0; e0 < nmax; e0 += kUnroll) {
      uint4 raw[kUnroll][CPL];
      float sc[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = e0 + u;
        int64_t t = t_begin;                       // idle slots re-read a valid row
        sc[u] = -INFINITY;
        if (e < ntot) {
          int w, slot;
          locate(e, w, slot);
          sc[u] = lsc[gq][w][slot];
          t = t_begin + lkey[gq][w][slot];
        }
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc)
          raw[u][cc] = __ldg(reinterpret_cast<const uint4 *>(vrow + t * D) + c8 + 8 * cc);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (e0 + u < ntot) {
          const float pw = exp2f((sc[u] - m_run) * kLog2e);
          l_run += pw;
          cnt_run += 1;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) {
            const uint4 x = raw[u][cc];
            float *a8 = acc + 8 * cc;
            a8[0] = fmaf(pw, bf16lo(x.x), a8[0]);
            a8[1] = fmaf(pw, bf16hi(x.x), a8[1]);
            a8[2] = fmaf(pw, bf16lo(x.y), a8[2]);
            a8[3] = fmaf(pw, bf16hi(x.y), a8[3]);
            a8[4] = fmaf(pw, bf16lo(x.z), a8[4]);
            a8[5] = fmaf(pw, bf16hi(x.z), a8[5]);
            a8[6] = fmaf(pw, bf16lo(x.w), a8[6]);
            a8[7] = fmaf(pw, bf16hi(x.w), a8[7]);
          }
        }
      }
    }
    sm100::named_bar(kBar, kComputeThreads);      // lists read before they refill
    my_cnt = 0;
  };

  bool bad = false;
  int committed = 0;                   // chunks whose MMAs thread 0 committed
  if (tid == 0) {
    if (issue_chunk(0)) committed = 1;
    else { fail(p, hdr); bad = true; }
  }
  if (warp == 0) bad = __shfl_sync(0xffffffffu, bad ? 1 : 0, 0) != 0;

  for (int c = 0; c < n_chunks; ++c) {
    if (tid == 0 && !bad && c + 1 < n_chunks) {
      if (issue_chunk(c + 1)) committed = c + 2;
      else { fail(p, hdr); bad = true; }
    }
    if (warp == 0) bad = __shfl_sync(0xffffffffu, bad ? 1 : 0, 0) != 0;
    if (!bad && !warp_wait(&hdr->mma_done[c & 1], (c >> 1) & 1)) {
      if (lane == 0) fail(p, hdr);
      bad = true;
    }
    sm100::tc_fence_after();
    const int half = warp >> 2, quarter = warp & 3;
    const bool has_tile = 2 * c + half < n_tiles;
    const int kpos = half * kTileKeys + quarter * 32 + lane;
    const int64_t t = t_begin + static_cast<int64_t>(c) * kChunkKeys + kpos;
    const bool valid = !bad && has_tile && t < t_end;
    float A[kN];
#pragma unroll
    for (int g = 0; g < kN; ++g) A[g] = 0.f;
    if (!bad && has_tile)
      sm100::tmem_ld16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                           (c & 1) * 2 * kN + half * kN, A);
    sm100::tc_fence_before();
#pragma unroll
    for (int g = 0; g < kN; ++g) A[g] = A[g] * p.scale;

    bool over = false;
    if (mode == kModeDump) {
      if (valid) {
#pragma unroll
        for (int g = 0; g < GP; ++g)
          if (g < G) p.scores_out[row0 + g * p.row_stride + t] = A[g];
      }
      if (p.hist != nullptr) {
        // top byte of each score's order key, one shared atomic per distinct
        // bin in the warp
        uint32_t(*hs)[256] = reinterpret_cast<uint32_t(*)[256]>(smem + Lo::off_key);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const bool in = valid && g < G;
          const uint32_t active = __ballot_sync(0xffffffffu, in);
          if (in) {
            const uint32_t bin = order_key(A[g]) >> 24;
            const uint32_t peers = __match_any_sync(active, bin);
            if (lane == __ffs(peers) - 1) atomicAdd(&hs[g][bin], static_cast<uint32_t>(__popc(peers)));
          }
        }
      }
    } else {
      uint32_t selbits = 0;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const bool sel = valid && g < G && A[g] >= tau_s[g];
        const uint32_t bal = __ballot_sync(0xffffffffu, sel);
        const int before = __shfl_sync(0xffffffffu, my_cnt, g);
        if (sel) {
          const int off = before + __popc(bal & lt_mask);
          lkey[g][warp][off] = static_cast<int>(t - t_begin);
          lsc[g][warp][off] = A[g];
        }
        if (lane == g) my_cnt += __popc(bal);
        selbits |= static_cast<uint32_t>(sel) << g;
      }
      if (p.sel_mask != nullptr && valid) {
        for (int g = 0; g < G; ++g)
          p.sel_mask[row0 + g * p.row_stride + t] = static_cast<uint8_t>((selbits >> g) & 1u);
      }
      // one more chunk may add 32 keys per (head, warp)
      over = __any_sync(0xffffffffu, my_cnt > C::kCap - 32);
    }
    // every warp has read this chunk's TMEM before thread 0 reuses the set
    const bool any_bad = bar_any(bad);
    if (any_bad) { bad = true; break; }
    if (bar_any(over)) gather();
  }
  if (!bad && mode != kModeDump) gather();

  // ---- teardown: every MMA has landed before TMEM is freed -----------------
  if (tid == 0 && bad && committed > 0)
    sm100::mbar_wait(&hdr->mma_done[(committed - 1) & 1], ((committed - 1) >> 1) & 1);
  sm100::tc_fence_before();
  sm100::named_bar(kBar, kComputeThreads);
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, kTmemCols);
  }
  if (mode == kModeDump) {
    if (p.hist != nullptr && !bad && !aborted(hdr)) {
      const uint32_t *hs = reinterpret_cast<const uint32_t *>(smem + Lo::off_key);
      for (int i = tid; i < G * 256; i += kComputeThreads) {
        const uint32_t v = hs[i];
        if (v != 0u) atomicAdd(&p.hist[static_cast<int64_t>(b * p.h_q + j0 + i / 256) * 256 + (i % 256)], v);
      }
    }
    return;
  }
  if (bad || aborted(hdr)) return;

  // ---- merge the two halves of each head and write the split's record -----
  // (the K stages are idle now: every tile landed and was consumed)
  float *mrg = reinterpret_cast<float *>(stages);      // [kN][D + 4]
  if (part == 1 && live) {
    float *r = mrg + gh * (D + kRecPad);
    if (c8 == 0) { r[0] = m_run; r[1] = l_run; r[2] = __int_as_float(cnt_run); }
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
      for (int v = 0; v < 8; ++v) r[kRecPad + (c8 + 8 * cc) * 8 + v] = acc[8 * cc + v];
  }
  sm100::named_bar(kBar, kComputeThreads);
  if (part == 0 && live) {
    const float *r = mrg + gh * (D + kRecPad);
    const float m1 = r[0], l1 = r[1];
    const int n1 = __float_as_int(r[2]);
    const float m = fmaxf(m_run, m1);
    const float w0 = m_run == -INFINITY ? 0.f : exp2f((m_run - m) * kLog2e);
    const float w1 = m1 == -INFINITY ? 0.f : exp2f((m1 - m) * kLog2e);
    float *rec = p.partials + (static_cast<int64_t>(b * p.h_q + j0 + gh) * p.S + s) * (D + kRecPad);
    if (c8 == 0) {
      rec[0] = m;
      rec[1] = w0 * l_run + w1 * l1;
      rec[2] = __int_as_float(cnt_run + n1);
      rec[3] = 0.f;
    }
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc)
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int i = (c8 + 8 * cc) * 8 + v;
        rec[kRecPad + i] = w0 * acc[8 * cc + v] + w1 * r[kRecPad + i];
      }
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda); resolved once.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

template <int D, int GP>
cudaError_t launch_tc(const StepParams &p, int mode, const CUtensorMap &map, cudaStream_t st) {
  using Lo = Layout<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(saga_tc_kernel<D, GP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lo::alloc);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(p.S, p.B * p.h_k);
  saga_tc_kernel<D, GP><<<grid, kThreads, Lo::alloc, st>>>(p, mode, map);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_tc_d(const StepParams &p, int mode, int gp, const CUtensorMap &map,
                        cudaStream_t st) {
  switch (gp) {
    case 4: return launch_tc<D, 4>(p, mode, map, st);
    case 8: return launch_tc<D, 8>(p, mode, map, st);
    case 12: return launch_tc<D, 12>(p, mode, map, st);
    case 16: return launch_tc<D, 16>(p, mode, map, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_saga_tc(const StepParams &p, int mode, int d, int gp, cudaStream_t st) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(p.cap),
                              static_cast<cuuint64_t>(p.h_k), static_cast<cuuint64_t>(p.B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(p.k_sh) * 2,
                                 static_cast<cuuint64_t>(p.k_sb) * 2};
  const cuuint32_t box[4] = {64, kTileKeys, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(p.K), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (d == 64) return launch_tc_d<64>(p, mode, gp, map, st);
  if (d == 128) return launch_tc_d<128>(p, mode, gp, map, st);
  return cudaErrorInvalidValue;
}

}  // namespace saga
