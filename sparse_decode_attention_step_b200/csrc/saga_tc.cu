// Tensor-core scan kernel for bf16 caches (sm_100a): the K-streaming half of
// the decode step. Eq. 2 scores on tcgen05, the Atop-N item 1 compare, and
// the kept lists that the gather kernel (gather.cu) turns into Eq. 7
// per-split states; for a refresh, the score rows and their histograms.
//
// Persistent: one CTA per SM walks the work units (sequence b, key head kh,
// split s of l_kv) u = blockIdx.x, blockIdx.x + gridDim.x, ... Warp roles:
//
//   warp 0      TMA producer: the unit's 16 query rows (one 16 x d tile) into
//               a double-buffered Q operand, then the K tiles of 128
//               positions x d (128B swizzle) through a ring of kStages
//               stages. It runs ahead across unit boundaries.
//   warp 1      MMA issuer and TMEM owner: per K tile d/16 tcgen05.mma
//               (M = 128 keys, N = 16 query heads, K = 16) into one of kTBufs
//               16-column TMEM buffers; the commits free the K stage and
//               publish the scores.
//   workers     4 x kRanks warps. Tile g belongs to rank g % kRanks; each of
//               the four warps of that rank reads its TMEM lane quarter
//               (32 keys x 16 heads), scales by 1/sqrt(d), compares with tau
//               and, for each query head, writes the 32-bit mask of kept
//               keys of its 32-position block and each kept score at the
//               key's rank within the block.
//
// The scan never waits for a V row: the V gather runs in its own kernel at
// full occupancy, where enough rows can be in flight to cover the latency
// of random row reads under load (about 2-3 us), which a warp that also
// scans cannot do. The lists are written at fixed places, so the step is
// deterministic.
//
// Modes: dump (score rows and per-row top-byte histograms of the order keys,
// for a refresh), step (keep A >= tau), step with ties (exact top-N: keep A
// above tau under totalOrder, and A == tau up to a per-row position). The
// step modes also run from stored score rows (FS): the producer then streams
// [16 heads x 128 positions] fp32 tiles of the refresh's own rows instead of
// K and no MMA runs, so a refresh reads K only once.
//
// Query heads beyond the group (G < 16) are rows of other heads or zero rows
// of Q; their tau is +inf, so they are never kept, and they are never dumped.
// Every wait is bounded; on a timeout the CTA sets SAGA_DEVERR_TIMEOUT and the
// step's abort word, and all roles stop after the copies and MMAs in flight
// have landed; the gather then writes poisoned records (m = +inf, count = -1),
// which the combine turns into NaN outputs and counts of -1.
#include <cuda.h>

#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace saga {

namespace {

constexpr int kTileKeys = 128;
constexpr int kN = 16;                      // MMA N: query heads of a group, padded
constexpr int kWorkerBar = 1;               // named barrier of the worker warps
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(kTileKeys, kN);

// R: worker warps per lane quarter. The plain step's workers keep up with
// the MMA at 3 (d = 64) and 2 (d = 128); the dump and the steps from stored
// scores do more per tile and take 5 and 3.
template <int D, int R>
struct Cfg {
  static constexpr int kRanks = R;
  static constexpr int kWorkers = 4 * kRanks;
  static constexpr int kThreads = 32 * (2 + kWorkers);
  static constexpr int kStages = D == 64 ? 8 : 4;             // 128 KB of K in flight
  static constexpr int kTBufs = 2 * kRanks <= 8 ? 2 * kRanks : 8;   // TMEM score buffers
  static constexpr int kTmemCols = kTBufs * kN <= 32 ? 32 : (kTBufs * kN <= 64 ? 64 : 128);
  static_assert(kTBufs * kN <= kTmemCols, "TMEM buffers fit the allocation");
  static constexpr int kBoxes = D / 64;                        // 64-column TMA boxes per tile
  static constexpr int kBoxBytes = kTileKeys * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQBoxBytes = kN * 128;
  static constexpr int kQBytes = kBoxes * kQBoxBytes;
  static constexpr int kScoreTileBytes = kN * kTileKeys * 4;   // FS stage: [16][128] fp32
  static_assert(kScoreTileBytes <= kTileBytes, "a score tile fits a stage");
  static constexpr int kHistBytes = kN * 256 * 4;              // dump mode: per-head top-byte bins
  static constexpr int kScratchBytes = kHistBytes;
};

template <typename C>
struct Header {
  uint64_t full[C::kStages], empty[C::kStages];
  uint64_t tfull[C::kTBufs], tempty[C::kTBufs];
  uint64_t qfull[2], qempty[2];
  uint32_t tmem_base;
  int abort;
  alignas(16) float tau[kN];
  int32_t tie[kN];           // tie mode: last position at which A == tau is kept
};

template <typename C>
struct Layout {
  static constexpr int off_stage = 0;
  static constexpr int off_q = C::kStages * C::kTileBytes;
  static constexpr int off_scratch = off_q + 2 * C::kQBytes;
  static constexpr int off_hdr = off_scratch + C::kScratchBytes;
  static constexpr int bytes = off_hdr + static_cast<int>(sizeof(Header<C>));
  static constexpr int alloc = bytes + 1024;                  // slack for 1024-byte alignment
  static_assert(alloc <= 227 * 1024, "shared memory of one CTA");
  static_assert(off_hdr % 16 == 0 && off_q % 1024 == 0, "operand alignment");
};

struct Unit {
  int b, kh, s;
  int64_t t_begin, t_end;
  int n_tiles;
};

// Work unit u; false when its split lies beyond l_kv[b] (nothing to do).
__device__ __forceinline__ bool unit_at(const StepParams &p, int u, bool report, Unit &un) {
  const int bk = u % (p.B * p.h_k);
  un.s = u / (p.B * p.h_k);
  un.b = bk / p.h_k;
  un.kh = bk % p.h_k;
  int64_t L;
  if (report) {
    L = clamp_len(p, un.b);
  } else {
    L = p.l_kv[un.b];
    const int64_t hi = p.cap < p.max_l_kv ? p.cap : p.max_l_kv;
    L = L < 0 ? 0 : (L > hi ? hi : L);
  }
  un.t_begin = static_cast<int64_t>(un.s) * p.split_len;
  if (un.t_begin >= L) return false;
  un.t_end = min(un.t_begin + p.split_len, L);
  un.n_tiles = static_cast<int>((un.t_end - un.t_begin + kTileKeys - 1) / kTileKeys);
  return true;
}

template <typename C>
__device__ __forceinline__ bool aborted(Header<C> *h) {
  return *reinterpret_cast<volatile int *>(&h->abort) != 0;
}

template <typename C>
__device__ __forceinline__ void fail(const StepParams &p, Header<C> *h) {
  if (!aborted(h)) {
    atomicOr(p.err, SAGA_DEVERR_TIMEOUT);
    if (p.abort != nullptr) atomicExch(p.abort, 1);   // the gather poisons this step's records
  }
  *reinterpret_cast<volatile int *>(&h->abort) = 1;
}

// Bounded wait that also gives up as soon as another role has aborted.
template <typename C>
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Header<C> *h) {
  if (sm100::mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::global_ns();
  for (;;) {
    if (sm100::mbar_try_wait_sleep(bar, parity, sm100::kSuspendHintNs)) return true;
    if (aborted(h)) return false;
    if (sm100::global_ns() - t0 > sm100::kWaitLimitNs) return false;
  }
}

// Warp-uniform version: lane 0 waits, the verdict is broadcast.
template <typename C>
__device__ __forceinline__ bool warp_wait_bar(uint64_t *bar, uint32_t parity, Header<C> *h) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, h);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// OR of `pred` over the worker warps (a barrier among them).
template <typename C>
__device__ __forceinline__ bool workers_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(kWorkerBar), "r"(C::kWorkers * 32)
      : "memory");
  return r != 0;
}

template <typename C>
__device__ __forceinline__ void workers_sync() {
  sm100::named_bar(kWorkerBar, C::kWorkers * 32);
}

template <int D, int MODE, bool FS>
using CfgOf = Cfg<D, (MODE == kModeStep && !FS) ? (D == 64 ? 3 : 2) : (D == 64 ? 5 : 3)>;

template <int D, int MODE, bool FS>
__global__ void __launch_bounds__(CfgOf<D, MODE, FS>::kThreads, 1)
saga_tc_kernel(const StepParams p, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap qmap) {
  using C = CfgOf<D, MODE, FS>;
  using Lo = Layout<C>;
  constexpr bool kDump = MODE == kModeDump;
  static_assert(!(kDump && FS), "the dump reads K");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = sm100::smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t *stages = smem + Lo::off_stage;
  uint8_t *qbuf = smem + Lo::off_q;
  float *scratch = reinterpret_cast<float *>(smem + Lo::off_scratch);
  Header<C> *h = reinterpret_cast<Header<C> *>(smem + Lo::off_hdr);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.h_q / p.h_k;
  const int n_units = p.B * p.h_k * p.S;

  // ---- set-up ----------------------------------------------------------------
  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      sm100::mbar_init(&h->full[i], 1);
      sm100::mbar_init(&h->empty[i], FS ? 4 : 1);   // FS: the rank's four warps free a stage
    }
    for (int i = 0; i < C::kTBufs; ++i) {
      sm100::mbar_init(&h->tfull[i], 1);
      sm100::mbar_init(&h->tempty[i], 4);     // the four lane-quarter warps of the rank
    }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&h->qfull[i], 1);
      sm100::mbar_init(&h->qempty[i], 1);
    }
    h->abort = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1 && !FS) {
    sm100::tmem_alloc(&h->tmem_base, C::kTmemCols);
    sm100::tmem_relinquish();
  }
  if (kDump && p.hist != nullptr && warp >= 2) {
    uint32_t *hs = reinterpret_cast<uint32_t *>(scratch);
    for (int i = tid - 64; i < kN * 256; i += C::kWorkers * 32) hs[i] = 0u;
  }
  // While the previous launch in the stream finishes, bring the first K
  // tiles of this CTA's first unit into L2. K itself may still be written by
  // that launch (a KV append); L2 holds the one copy every SM reads, so a
  // line fetched early is updated by such a write, never stale.
  if (!kDump && !FS && warp == 0 && lane == 0 && static_cast<int>(blockIdx.x) < n_units) {
    const int u = blockIdx.x;
    const int bk = u % (p.B * p.h_k);
    const int64_t t0 = static_cast<int64_t>(u / (p.B * p.h_k)) * p.split_len;
    const int n = static_cast<int>(min(static_cast<int64_t>(C::kStages), p.split_len / kTileKeys));
    for (int i = 0; i < n; ++i)
      for (int bx = 0; bx < C::kBoxes; ++bx)
        sm100::tma_prefetch_4d(&kmap, bx * 64, static_cast<int>(t0) + i * kTileKeys, bk % p.h_k,
                               bk / p.h_k);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = FS ? 0u : h->tmem_base;
  // everything below may read what the previous launch in the stream wrote
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ---- TMA producer ------------------------------------------------------
    if (lane == 0) {
      sm100::prefetch_tensormap(&kmap);
      if (!FS) sm100::prefetch_tensormap(&qmap);
      uint32_t g = 0;
      int k = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        Unit un;
        if (!unit_at(p, u, true, un)) continue;
        if (!FS) {
          const int qb = k & 1;
          if (!wait_bar(&h->qempty[qb], ((k >> 1) & 1) ^ 1, h)) { ok = false; break; }
          sm100::mbar_arrive_expect_tx(&h->qfull[qb], C::kQBytes);
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            sm100::tma_load_3d(qbuf + qb * C::kQBytes + bx * C::kQBoxBytes, &qmap, &h->qfull[qb],
                               bx * 64, un.kh * G, un.b);
          ++k;
        }
        for (int i = 0; i < un.n_tiles; ++i) {
          const int st = g % C::kStages;
          if (!wait_bar(&h->empty[st], ((g / C::kStages) & 1) ^ 1, h)) { ok = false; break; }
          const int y = static_cast<int>(un.t_begin) + i * kTileKeys;
          uint8_t *dst = stages + st * C::kTileBytes;
          if (FS) {
            sm100::mbar_arrive_expect_tx(&h->full[st], C::kScoreTileBytes);
            sm100::tma_load_3d(dst, &kmap, &h->full[st], y, un.kh * G, un.b);
          } else {
            sm100::mbar_arrive_expect_tx(&h->full[st], C::kTileBytes);
#pragma unroll
            for (int bx = 0; bx < C::kBoxes; ++bx)
              sm100::tma_load_4d(dst + bx * C::kBoxBytes, &kmap, &h->full[st], bx * 64, y, un.kh,
                                 un.b);
          }
          ++g;
        }
      }
      if (!ok) {
        fail(p, h);
        // the copies still in flight land before the CTA can exit: the
        // last kStages tiles and the last two Q tiles
        for (uint32_t i = g > static_cast<uint32_t>(C::kStages) ? g - C::kStages : 0; i < g; ++i)
          sm100::mbar_wait(&h->full[i % C::kStages], (i / C::kStages) & 1);
        for (int i = k > 2 ? k - 2 : 0; i < k; ++i)
          sm100::mbar_wait(&h->qfull[i & 1], (i >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer (idle when the scores come from stored rows) ------------
    if (lane == 0 && !FS) {
      const uint32_t st_u32 = sm100::smem_u32(stages);
      const uint32_t q_u32 = sm100::smem_u32(qbuf);
      uint32_t g = 0, committed = 0;
      int k = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        Unit un;
        if (!unit_at(p, u, false, un)) continue;
        const int qb = k & 1;
        if (!wait_bar(&h->qfull[qb], (k >> 1) & 1, h)) { ok = false; break; }
        for (int i = 0; i < un.n_tiles; ++i) {
          const int st = g % C::kStages, tb = g % C::kTBufs;
          if (!wait_bar(&h->full[st], (g / C::kStages) & 1, h) ||
              !wait_bar(&h->tempty[tb], ((g / C::kTBufs) & 1) ^ 1, h)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t a0 = st_u32 + st * C::kTileBytes;
          const uint32_t b0 = q_u32 + qb * C::kQBytes;
#pragma unroll
          for (int j = 0; j < D / 16; ++j) {
            const int bx = j / 4, kk = j % 4;
            const uint64_t ad = sm100::desc_k_sw128(a0 + bx * C::kBoxBytes + kk * 32);
            const uint64_t bd = sm100::desc_k_sw128(b0 + bx * C::kQBoxBytes + kk * 32);
            sm100::mma_bf16(tmem_base + tb * kN, ad, bd, kIdesc, j > 0 ? 1u : 0u);
          }
          sm100::mma_commit(&h->empty[st]);
          sm100::mma_commit(&h->tfull[tb]);
          ++g;
          committed = g;
        }
        if (!ok) break;
        sm100::mma_commit(&h->qempty[qb]);
        ++k;
      }
      if (!ok) {
        fail(p, h);
        // every MMA issued has landed before TMEM and the stages go away
        if (committed > 0)
          sm100::mbar_wait(&h->tfull[(committed - 1) % C::kTBufs],
                           ((committed - 1) / C::kTBufs) & 1);
      }
    }
    __syncwarp();
  } else {
    // ---- workers ------------------------------------------------------------
    const int widx = warp - 2;
    const int quarter = warp & 3;             // TMEM lanes (keys) this warp reads
    const int rank = widx >> 2;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t g = 0;
    bool bad = false;

    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      Unit un;
      if (!unit_at(p, u, false, un)) continue;
      const int j0 = un.kh * G;
      const int64_t row0 = static_cast<int64_t>(un.b * p.h_q + j0) * p.row_stride;
      if (!kDump) {
        if (widx == 0 && lane < kN) {
          h->tau[lane] = lane < G ? p.tau[un.b * p.h_q + j0 + lane] : INFINITY;
          if (MODE == kModeStepTies) h->tie[lane] = lane < G ? p.tie[un.b * p.h_q + j0 + lane] : -1;
        }
        workers_sync<C>();
      }

      const int first = (rank - static_cast<int>(g % C::kRanks) + C::kRanks) % C::kRanks;
      for (int i = first; i < un.n_tiles; i += C::kRanks) {
        const uint32_t gg = g + i;
        float A[kN];
        if (FS) {
          const int st = gg % C::kStages;
          if (!warp_wait_bar(&h->full[st], (gg / C::kStages) & 1, h)) {
            if (lane == 0) fail(p, h);
            bad = true;
            break;
          }
          const float *sp = reinterpret_cast<const float *>(stages + st * C::kTileBytes);
#pragma unroll
          for (int a = 0; a < kN; ++a) A[a] = sp[a * kTileKeys + quarter * 32 + lane];
          // the stage is freed below, once every lane has used its scores
        } else {
          const int tb = gg % C::kTBufs;
          if (!warp_wait_bar(&h->tfull[tb], (gg / C::kTBufs) & 1, h)) {
            if (lane == 0) fail(p, h);
            bad = true;
            break;
          }
          sm100::tc_fence_after();
          sm100::tmem_ld16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + tb * kN, A);
          sm100::tc_fence_before();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&h->tempty[tb]);
        }

        const int64_t t0 = un.t_begin + static_cast<int64_t>(i) * kTileKeys + quarter * 32;
        const int64_t t = t0 + lane;
        const bool valid = t < un.t_end;

        if (kDump) {
#pragma unroll
          for (int a = 0; a < kN; ++a) {
            const float x = A[a] * p.scale;
            if (valid && a < G && saga_in_bounds(t < p.row_stride, p.err))
              p.scores_out[row0 + a * p.row_stride + t] = x;
            if (p.hist != nullptr) {
              // top byte of the score's order key, one shared atomic per
              // distinct bin in the warp
              const bool in = valid && a < G;
              const uint32_t active = __ballot_sync(0xffffffffu, in);
              if (in) {
                const uint32_t bin = order_key(x) >> 24;
                const uint32_t peers = __match_any_sync(active, bin);
                if (lane == __ffs(peers) - 1)
                  atomicAdd(reinterpret_cast<uint32_t *>(scratch) + a * 256 + bin,
                            static_cast<uint32_t>(__popc(peers)));
              }
            }
          }
          continue;
        }

        // ---- compare: the heads that keep this lane's key --------------------
        uint32_t sel = 0;
        {
          const float4 *tq = reinterpret_cast<const float4 *>(h->tau);
#pragma unroll
          for (int a4 = 0; a4 < kN / 4; ++a4) {
            const float4 tv = tq[a4];
            const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int a = 4 * a4 + e;
              const float x = FS ? A[a] : A[a] * p.scale;
              bool keep;
              if constexpr (MODE == kModeStepTies) {
                // totalOrder, as the threshold was selected: above tau, or
                // equal to it up to the last position the top N take
                const uint32_t kx = order_key(x), kt = order_key(tt[e]);
                keep = valid && (kx > kt || (kx == kt && t <= h->tie[a]));
              } else {
                keep = valid && x >= tt[e];
              }
              sel |= static_cast<uint32_t>(keep) << a;
              A[a] = keep ? x : -INFINITY;
            }
          }
        }
        if (p.sel_mask != nullptr && valid) {
          for (int a = 0; a < G; ++a)
            p.sel_mask[row0 + a * p.row_stride + t] = static_cast<uint8_t>((sel >> a) & 1u);
        }
        // ---- the kept lists of this 32-position block, per query head: the
        // mask, and each kept score at the key's rank within the block
        // (quarters of the last tile that lie past the row's nblk blocks
        // belong to no block of the row: nothing is written for them)
        const int64_t blk = t0 >> 5;
        if (blk < p.nblk) {
          const int64_t hrow0 = static_cast<int64_t>(un.b * p.h_q + j0) * p.nblk + blk;
          uint32_t mymask = 0;
#pragma unroll
          for (int a = 0; a < kN; ++a) {
            if (a >= G) break;
            const uint32_t bl = __ballot_sync(0xffffffffu, (sel >> a) & 1u);
            if (lane == a) mymask = bl;
            if (((bl >> lane) & 1u) && saga_in_bounds(valid, p.err))   // only real positions are kept
              p.lscore[(hrow0 + a * p.nblk) * 32 + __popc(bl & lt_mask)] = A[a];
          }
          if (lane < G) p.lmask[hrow0 + lane * p.nblk] = mymask;
        }
        // FS: every lane's scores have gone into `sel` and the ballots above,
        // so the stage can be refilled
        if (FS && lane == 0) sm100::mbar_arrive(&h->empty[gg % C::kStages]);
      }
      g += un.n_tiles;

      // ---- end of unit -------------------------------------------------------
      if (workers_any<C>(bad || aborted(h))) break;
      if (kDump && p.hist != nullptr) {
        uint32_t *hs = reinterpret_cast<uint32_t *>(scratch);
        for (int i = widx * 32 + lane; i < kN * 256; i += C::kWorkers * 32) {
          const uint32_t c = hs[i];
          if (c != 0u && i / 256 < G)
            atomicAdd(&p.hist[static_cast<int64_t>(un.b * p.h_q + j0 + i / 256) * 256 + (i % 256)], c);
          hs[i] = 0u;
        }
        workers_sync<C>();
      }
    }
  }

  // ---- teardown: every MMA has landed before TMEM is freed -----------------
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1 && !FS) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, C::kTmemCols);
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

constexpr int kMaxDevices = 64;

// SM count of a device, cached per device.
int sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return -1;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int D, int MODE, bool FS>
cudaError_t launch_tc(const StepParams &p, const CUtensorMap &kmap, const CUtensorMap &qmap,
                      int dev, cudaStream_t st) {
  using Lo = Layout<CfgOf<D, MODE, FS>>;
  static std::atomic<bool> attr_set[kMaxDevices];
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(saga_tc_kernel<D, MODE, FS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lo::alloc);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int sms = sm_count(dev);
  if (sms < 1) return cudaErrorInvalidDevice;
  const int n_units = p.B * p.h_k * p.S;
  const int grid = n_units < sms ? n_units : sms;
  if (grid < 1) return cudaSuccess;
  return launch_pdl(saga_tc_kernel<D, MODE, FS>, dim3(grid), dim3(CfgOf<D, MODE, FS>::kThreads), Lo::alloc,
                    st, p, kmap, qmap);
}

}  // namespace

bool saga_tc_supports(int dtype, int d, int h_q, int h_k, int h_v) {
  return dtype == SAGA_BF16 && (d == 64 || d == 128) && h_k >= 1 && h_v >= 1 &&
         h_q % h_v == 0 && h_v % h_k == 0 && h_q / h_k <= kN;
}

bool saga_tc_scores_streamable(const float *rows, int64_t row_stride) {
  return rows != nullptr && (reinterpret_cast<uintptr_t>(rows) % 16) == 0 && row_stride % 4 == 0 &&
         row_stride > 0;
}

cudaError_t launch_saga_tc(const StepParams &p, int mode, int d, cudaStream_t st) {
  if (!saga_tc_supports(SAGA_BF16, d, p.h_q, p.h_k, p.h_v)) return cudaErrorInvalidValue;
  if (mode != kModeDump && mode != kModeStep && mode != kModeStepTies) return cudaErrorInvalidValue;
  const bool fs = p.scores_in != nullptr;
  if (fs && (mode == kModeDump || !saga_tc_scores_streamable(p.scores_in, p.row_stride)))
    return cudaErrorInvalidValue;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMap kmap, qmap;
  std::memset(&qmap, 0, sizeof(qmap));
  if (fs) {
    // stored score rows [B][h_q][row_stride] fp32: a [16 heads x 128 positions] box
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.max_l_kv), static_cast<cuuint64_t>(p.h_q),
                                static_cast<cuuint64_t>(p.B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.row_stride) * 4,
                                   static_cast<cuuint64_t>(p.row_stride) * 4 * p.h_q};
    const cuuint32_t box[3] = {kTileKeys, kN, 1};
    if (enc(&kmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(p.scores_in), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    {
      const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(p.cap),
                                  static_cast<cuuint64_t>(p.h_k), static_cast<cuuint64_t>(p.B)};
      const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                     static_cast<cuuint64_t>(p.k_sh) * 2,
                                     static_cast<cuuint64_t>(p.k_sb) * 2};
      const cuuint32_t box[4] = {64, kTileKeys, 1, 1};
      if (enc(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(p.K), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    {
      const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(p.h_q),
                                  static_cast<cuuint64_t>(p.B)};
      const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.q_sh) * 2,
                                     static_cast<cuuint64_t>(p.q_sb) * 2};
      const cuuint32_t box[3] = {64, kN, 1};
      if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(p.q), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
#define SAGA_TC_LAUNCH(DD)                                                                    \
  if (d == DD) {                                                                              \
    if (mode == kModeDump) return launch_tc<DD, kModeDump, false>(p, kmap, qmap, dev, st); \
    if (mode == kModeStep)                                                                    \
      return fs ? launch_tc<DD, kModeStep, true>(p, kmap, qmap, dev, st)                  \
                : launch_tc<DD, kModeStep, false>(p, kmap, qmap, dev, st);                \
    return fs ? launch_tc<DD, kModeStepTies, true>(p, kmap, qmap, dev, st)                \
              : launch_tc<DD, kModeStepTies, false>(p, kmap, qmap, dev, st);              \
  }
  SAGA_TC_LAUNCH(64)
  SAGA_TC_LAUNCH(128)
#undef SAGA_TC_LAUNCH
  return cudaErrorInvalidValue;
}

}  // namespace saga
