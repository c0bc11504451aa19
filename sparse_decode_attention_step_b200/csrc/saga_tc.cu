// Tensor-core split kernel for bf16 caches (sm_100a): Eq. 2 scores,
// Atop-N item 1 compare, Eq. 7 sparse softmax with the V gather, and the
// per-split online-softmax states, with the score contraction on tcgen05.
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
//               and gathers V for its own kept keys: lane group v (8 lanes)
//               owns up to four query heads that share one value head, so
//               each kept V row is read once for all of them, and keeps their
//               online-softmax states (m, l, count, acc) in registers.
//
// Each worker folds a quarter tile's kept rows in rounds of kRows V rows per
// lane group (empty rows and heads no lane group kept are skipped, and the
// states are rescaled only when a round raises a maximum). At the end of a
// unit every worker writes its states to shared memory, the per-head
// weights e^{m_w - m} are formed once, and all workers write the unit's
// (m, l, count, acc) records.
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
// Every wait is bounded; on a timeout the CTA sets SAGA_DEVERR_TIMEOUT, all
// roles stop after the copies and MMAs in flight have landed, and the
// workers write poisoned records (m = +inf, count = -1) for every unit the
// CTA had left, which the combine turns into NaN outputs and counts of -1.
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
constexpr float kLog2e = 1.4426950408889634f;

constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int D>
struct Cfg {
  static constexpr int kRanks = D == 64 ? 3 : 2;              // worker warps per lane quarter
  static constexpr int kWorkers = 4 * kRanks;
  static constexpr int kThreads = 32 * (2 + kWorkers);
  static constexpr int kStages = D == 64 ? 8 : 4;             // 128 KB of K in flight
  static constexpr int kTBufs = 2 * kRanks;                    // TMEM score buffers
  static constexpr int kTmemCols = kTBufs * kN <= 32 ? 32 : (kTBufs * kN <= 64 ? 64 : 128);
  static_assert(kTBufs * kN <= kTmemCols, "TMEM buffers fit the allocation");
  static constexpr int kBoxes = D / 64;                        // 64-column TMA boxes per tile
  static constexpr int kBoxBytes = kTileKeys * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQBoxBytes = kN * 128;
  static constexpr int kQBytes = kBoxes * kQBoxBytes;
  static constexpr int kRows = 4;                              // kept V rows in flight per lane group
  static constexpr int kScoreTileBytes = kN * kTileKeys * 4;   // FS stage: [16][128] fp32
  static_assert(kScoreTileBytes <= kTileBytes, "a score tile fits a stage");
  static constexpr int CPL = D / 64;                           // 16-byte chunks per lane per V row
  static constexpr int EPL = 8 * CPL;                          // V row elements per lane
  static constexpr int kRec = D + kRecPad;
  static constexpr int kStateFloats = kN * kRec;               // one warp's 16 head states
  static constexpr int kScoreBytes = kWorkers * 2 * 32 * kN * 4;   // two kept-score row sets per warp
  static constexpr int kMergeBytes = kWorkers * (kStateFloats + kN) * 4;  // states + weights
  static constexpr int kHistBytes = kN * 256 * 4;
  static constexpr int kScratchBytes = cmax(cmax(kScoreBytes, kMergeBytes), kHistBytes);
};

template <int D>
struct Header {
  uint64_t full[Cfg<D>::kStages], empty[Cfg<D>::kStages];
  uint64_t tfull[Cfg<D>::kTBufs], tempty[Cfg<D>::kTBufs];
  uint64_t qfull[2], qempty[2];
  uint32_t tmem_base;
  int abort;
  alignas(16) float tau[kN];
  int32_t tie[kN];           // tie mode: last position at which A == tau is kept
};

template <int D>
struct Layout {
  using C = Cfg<D>;
  static constexpr int off_stage = 0;
  static constexpr int off_q = C::kStages * C::kTileBytes;
  static constexpr int off_scratch = off_q + 2 * C::kQBytes;
  static constexpr int off_hdr = off_scratch + C::kScratchBytes;
  static constexpr int bytes = off_hdr + static_cast<int>(sizeof(Header<D>));
  static constexpr int alloc = bytes + 1024;                  // slack for 1024-byte alignment
  static_assert(alloc <= 227 * 1024, "shared memory of one CTA");
  static_assert(off_hdr % 16 == 0 && off_q % 1024 == 0, "operand alignment");
};

// Lane group v of a worker warp owns query heads hbase[v] .. hbase[v] + nh[v] - 1
// of the group, all reading value head kh * (h_v / h_k) + vs[v]; smask[v] is
// the same set as a 16-bit mask.
struct HeadMap {
  int hbase[4], nh[4], vs[4];
  uint32_t smask[4];
};

// a[v] for a lane-dependent v without indexing the parameter array
__device__ __forceinline__ int pick4(const int (&a)[4], int v) {
  return v == 0 ? a[0] : (v == 1 ? a[1] : (v == 2 ? a[2] : a[3]));
}

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

template <int D>
__device__ __forceinline__ bool aborted(Header<D> *h) {
  return *reinterpret_cast<volatile int *>(&h->abort) != 0;
}

template <int D>
__device__ __forceinline__ void fail(const StepParams &p, Header<D> *h) {
  if (!aborted(h)) atomicOr(p.err, SAGA_DEVERR_TIMEOUT);
  *reinterpret_cast<volatile int *>(&h->abort) = 1;
}

// Bounded wait that also gives up as soon as another role has aborted.
template <int D>
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Header<D> *h) {
  if (sm100::mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::global_ns();
  for (;;) {
    if (sm100::mbar_try_wait_sleep(bar, parity, sm100::kSuspendHintNs)) return true;
    if (aborted(h)) return false;
    if (sm100::global_ns() - t0 > sm100::kWaitLimitNs) return false;
  }
}

// Warp-uniform version: lane 0 waits, the verdict is broadcast.
template <int D>
__device__ __forceinline__ bool warp_wait_bar(uint64_t *bar, uint32_t parity, Header<D> *h) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, h);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// OR of `pred` over the worker warps (a barrier among them).
template <int D>
__device__ __forceinline__ bool workers_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(kWorkerBar), "r"(Cfg<D>::kWorkers * 32)
      : "memory");
  return r != 0;
}

template <int D>
__device__ __forceinline__ void workers_sync() {
  sm100::named_bar(kWorkerBar, Cfg<D>::kWorkers * 32);
}

// Kept-score row of key k in a worker's scratch: 16 floats, 16-byte quads
// rotated by the key so the four row stores of a warp spread over the banks.
__device__ __forceinline__ int score_slot(int k, int h) {
  return k * kN + ((((h >> 2) ^ (k >> 1)) & 3) << 2) + (h & 3);
}

// One worker state (m, l, count, acc over its lane's slice) into a record
// laid out as {m, l, count, pad, acc[D]}; lane c8 == 0 writes the scalars.
template <int EPL>
__device__ __forceinline__ void put_state(float *r, int c8, float m, float l, int cnt,
                                          const float (&acc)[EPL]) {
  if (c8 == 0) {
    r[0] = m;
    r[1] = l;
    r[2] = __int_as_float(cnt);
    r[3] = 0.f;
  }
#pragma unroll
  for (int cc = 0; cc < EPL / 8; ++cc) {
    float4 *dst = reinterpret_cast<float4 *>(r + kRecPad + (c8 + 8 * cc) * 8);
    dst[0] = make_float4(acc[8 * cc], acc[8 * cc + 1], acc[8 * cc + 2], acc[8 * cc + 3]);
    dst[1] = make_float4(acc[8 * cc + 4], acc[8 * cc + 5], acc[8 * cc + 6], acc[8 * cc + 7]);
  }
}

// Poisoned record: the combine turns it into a NaN output and a count of -1.
__device__ __forceinline__ void put_poison(float *r) {
  r[0] = INFINITY;
  r[1] = __int_as_float(0x7fc00000);
  r[2] = __int_as_float(-1);
  r[3] = 0.f;
}

template <int D, int MODE, bool FS>
__global__ void __launch_bounds__(Cfg<D>::kThreads, 1)
saga_tc_kernel(const StepParams p, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap qmap, const HeadMap hm) {
  using C = Cfg<D>;
  using Lo = Layout<D>;
  constexpr int CPL = C::CPL, EPL = C::EPL, kRows = C::kRows;
  constexpr bool kDump = MODE == kModeDump;
  static_assert(!(kDump && FS), "the dump reads K");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = sm100::smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t *stages = smem + Lo::off_stage;
  uint8_t *qbuf = smem + Lo::off_q;
  float *scratch = reinterpret_cast<float *>(smem + Lo::off_scratch);
  Header<D> *h = reinterpret_cast<Header<D> *>(smem + Lo::off_hdr);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.h_q / p.h_k;
  const int vpg = p.h_v / p.h_k;
  const int n_units = p.B * p.h_k * p.S;

  // ---- set-up (touches no global memory) ---------------------------------
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
    const int v = lane >> 3, c8 = lane & 7;
    const int hbase = pick4(hm.hbase, v), nh = pick4(hm.nh, v), vsl = pick4(hm.vs, v);
    const bool quad = (hbase & 3) == 0 && nh == 4;   // the heads are one 16-byte quad of a row
    // two kept-score row sets, used in turn: the rows in flight keep theirs
    float *rows_base = scratch + widx * 2 * 32 * kN;
    uint32_t g = 0;
    bool bad = false;

    float m[4], l[4], acc[4][EPL];
    int cnt[4];
    const uint16_t *vrow = nullptr;
    // Fold the kept keys `mine` of this lane group (keys t0 + bit) into the
    // lane group's online-softmax states, kRows V rows in flight per round.
    auto gather = [&](uint32_t mine, int64_t t0, int64_t t_any, const float *rows) {
      const int nmax = static_cast<int>(__reduce_max_sync(0xffffffffu, __popc(mine)));
      for (int r0 = 0; r0 < nmax; r0 += kRows) {
        uint4 raw[kRows][CPL];
        float sc[kRows][4];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (r0 + r >= nmax) {
#pragma unroll
            for (int a = 0; a < 4; ++a) sc[r][a] = -INFINITY;
            continue;
          }
          const int kk = mine != 0u ? __ffs(mine) - 1 : -1;

          mine &= mine - 1u;
          // idle slots re-read a row of the unit, which always exists
          const int64_t tr = kk >= 0 ? t0 + kk : t_any;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
            raw[r][cc] = __ldg(reinterpret_cast<const uint4 *>(vrow + tr * D) + c8 + 8 * cc);
          const int ks = kk >= 0 ? kk : 0;
          if (quad) {
            const float4 q4 = *reinterpret_cast<const float4 *>(rows + score_slot(ks, hbase));
            sc[r][0] = kk >= 0 ? q4.x : -INFINITY;
            sc[r][1] = kk >= 0 ? q4.y : -INFINITY;
            sc[r][2] = kk >= 0 ? q4.z : -INFINITY;
            sc[r][3] = kk >= 0 ? q4.w : -INFINITY;
          } else {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const int hd = min(hbase + a, kN - 1);
              sc[r][a] = (kk >= 0 && a < nh) ? rows[score_slot(ks, hd)] : -INFINITY;
            }
          }
        }
        float mnew[4];
        bool grow = false;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          float mx = sc[0][a];
#pragma unroll
          for (int r = 1; r < kRows; ++r) mx = fmaxf(mx, sc[r][a]);
          mnew[a] = fmaxf(m[a], mx);
          grow |= mnew[a] != m[a];
        }
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const float corr = mnew[a] == m[a] ? 1.f : exp2f((m[a] - mnew[a]) * kLog2e);
            m[a] = mnew[a];
            l[a] *= corr;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[a][e] *= corr;
          }
        }

#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (r0 + r >= nmax) break;
          float vf[EPL];

#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) {
            const uint4 x = raw[r][cc];
            vf[8 * cc + 0] = bf16lo(x.x); vf[8 * cc + 1] = bf16hi(x.x);
            vf[8 * cc + 2] = bf16lo(x.y); vf[8 * cc + 3] = bf16hi(x.y);
            vf[8 * cc + 4] = bf16lo(x.z); vf[8 * cc + 5] = bf16hi(x.z);
            vf[8 * cc + 6] = bf16lo(x.w); vf[8 * cc + 7] = bf16hi(x.w);
          }
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const bool in = sc[r][a] != -INFINITY;
            if (!__any_sync(0xffffffffu, in)) continue;
            const float pw = in ? exp2f((sc[r][a] - m[a]) * kLog2e) : 0.f;

            l[a] += pw;
            cnt[a] += in ? 1 : 0;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[a][e] = fmaf(pw, vf[e], acc[a][e]);
          }
        }
      }
    };

    int u = blockIdx.x;
    for (; u < n_units; u += gridDim.x) {
      Unit un;
      if (!unit_at(p, u, false, un)) continue;
      const int j0 = un.kh * G;
      const int64_t row0 = static_cast<int64_t>(un.b * p.h_q + j0) * p.row_stride;
      if (!kDump) {
        if (widx == 0 && lane < kN) {
          h->tau[lane] = lane < G ? p.tau[un.b * p.h_q + j0 + lane] : INFINITY;
          if (MODE == kModeStepTies) h->tie[lane] = lane < G ? p.tie[un.b * p.h_q + j0 + lane] : -1;
        }
        workers_sync<D>();
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        m[a] = -INFINITY; l[a] = 0.f; cnt[a] = 0;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[a][e] = 0.f;
      }
      vrow = static_cast<const uint16_t *>(p.V) + un.b * p.v_sb +
             static_cast<int64_t>(un.kh * vpg + vsl) * p.v_sh;
      int n_mine = 0;

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
            if (valid && a < G) p.scores_out[row0 + a * p.row_stride + t] = x;
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
        float *rows = rows_base + (n_mine & 1) * 32 * kN;
        ++n_mine;
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
        if (sel != 0u) {
#pragma unroll
          for (int a4 = 0; a4 < kN / 4; ++a4)
            *reinterpret_cast<float4 *>(rows + score_slot(lane, 4 * a4)) =
                make_float4(A[4 * a4], A[4 * a4 + 1], A[4 * a4 + 2], A[4 * a4 + 3]);
        }
        if (p.sel_mask != nullptr && valid) {
          for (int a = 0; a < G; ++a)
            p.sel_mask[row0 + a * p.row_stride + t] = static_cast<uint8_t>((sel >> a) & 1u);
        }
        uint32_t mine = 0;
#pragma unroll
        for (int vv = 0; vv < 4; ++vv) {
          const uint32_t bl = __ballot_sync(0xffffffffu, (sel & hm.smask[vv]) != 0u);
          if (v == vv) mine = bl;
        }
        // FS: every lane's scores have gone into `sel` and the ballots above,
        // so the stage can be refilled
        if (FS && lane == 0) sm100::mbar_arrive(&h->empty[gg % C::kStages]);
        __syncwarp();
        gather(mine, t0, un.t_begin, rows);
        __syncwarp();            // rows read before a later tile overwrites them
      }
      g += un.n_tiles;

      // ---- end of unit -------------------------------------------------------
      if (workers_any<D>(bad || aborted(h))) { bad = true; break; }
      if (kDump) {
        if (p.hist != nullptr) {
          uint32_t *hs = reinterpret_cast<uint32_t *>(scratch);
          for (int i = widx * 32 + lane; i < kN * 256; i += C::kWorkers * 32) {
            const uint32_t c = hs[i];
            if (c != 0u && i / 256 < G)
              atomicAdd(&p.hist[static_cast<int64_t>(un.b * p.h_q + j0 + i / 256) * 256 + (i % 256)], c);
            hs[i] = 0u;
          }
          workers_sync<D>();
        }
        continue;
      }
      // merge: every worker's 16 head states into shared memory, then
      // per head the weights e^{m_w - m} of the workers, then the records
      {
        float *st = scratch + widx * C::kStateFloats;
#pragma unroll
        for (int a = 0; a < 4; ++a)
          put_state<EPL>(st + (v * 4 + a) * C::kRec, c8, m[a], l[a], cnt[a], acc[a]);
      }
      workers_sync<D>();
      float *wts = scratch + C::kWorkers * C::kStateFloats;       // [kN][kWorkers]
      const int tw = widx * 32 + lane;
      if (tw < kN) {
        const int slot = tw, sv = slot >> 2, sa = slot & 3;
        float mm = -INFINITY;
        for (int w = 0; w < C::kWorkers; ++w) mm = fmaxf(mm, scratch[w * C::kStateFloats + slot * C::kRec]);
        float ll = 0.f;
        int nn = 0;
        for (int w = 0; w < C::kWorkers; ++w) {
          const float *r = scratch + w * C::kStateFloats + slot * C::kRec;
          const float wt = r[0] == -INFINITY ? 0.f : exp2f((r[0] - mm) * kLog2e);
          wts[slot * C::kWorkers + w] = wt;
          ll = fmaf(wt, r[1], ll);
          nn += __float_as_int(r[2]);
        }
        if (sa < pick4(hm.nh, sv)) {
          const int j = j0 + pick4(hm.hbase, sv) + sa;
          float *rec = p.partials + (static_cast<int64_t>(un.b * p.h_q + j) * p.S + un.s) * C::kRec;
          rec[0] = mm;
          rec[1] = ll;
          rec[2] = __int_as_float(nn);
          rec[3] = 0.f;
        }
      }
      workers_sync<D>();
      for (int idx = tw; idx < kN * D; idx += C::kWorkers * 32) {
        const int slot = idx / D, dd = idx % D, sv = slot >> 2, sa = slot & 3;
        if (sa >= pick4(hm.nh, sv)) continue;
        float a = 0.f;
        for (int w = 0; w < C::kWorkers; ++w)
          a = fmaf(wts[slot * C::kWorkers + w],
                   scratch[w * C::kStateFloats + slot * C::kRec + kRecPad + dd], a);
        const int j = j0 + pick4(hm.hbase, sv) + sa;
        p.partials[(static_cast<int64_t>(un.b * p.h_q + j) * p.S + un.s) * C::kRec + kRecPad + dd] = a;
      }
      workers_sync<D>();          // scratch read before the next unit reuses it
    }
    if (bad && !kDump && widx == 0 && lane < kN) {
      // this unit and every later one of this CTA: poisoned records
      for (; u < n_units; u += gridDim.x) {
        Unit un;
        if (!unit_at(p, u, false, un) || lane >= G) continue;
        const int j = un.kh * G + lane;
        put_poison(p.partials + (static_cast<int64_t>(un.b * p.h_q + j) * p.S + un.s) * C::kRec);
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
                      const HeadMap &hm, int dev, cudaStream_t st) {
  using Lo = Layout<D>;
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
  return launch_pdl(saga_tc_kernel<D, MODE, FS>, dim3(grid), dim3(Cfg<D>::kThreads), Lo::alloc,
                    st, p, kmap, qmap, hm);
}

// Lane-group slots: value head slot vs = v / chunks, chunk c = v % chunks of
// that value head's h_q / h_v query heads (four per chunk).
bool make_head_map(int h_q, int h_k, int h_v, HeadMap &hm) {
  if (h_k < 1 || h_v < 1 || h_q % h_v != 0 || h_v % h_k != 0) return false;
  const int G = h_q / h_k, hpv = h_q / h_v, vpg = h_v / h_k;
  const int chunks = (hpv + 3) / 4;
  if (G > kN || vpg * chunks > 4) return false;
  for (int v = 0; v < 4; ++v) {
    const int vs = v / chunks, c = v % chunks;
    if (vs < vpg && c * 4 < hpv) {
      hm.hbase[v] = vs * hpv + c * 4;
      hm.nh[v] = hpv - c * 4 < 4 ? hpv - c * 4 : 4;
      hm.vs[v] = vs;
    } else {
      hm.hbase[v] = 0;
      hm.nh[v] = 0;
      hm.vs[v] = 0;
    }
    hm.smask[v] = ((1u << hm.nh[v]) - 1u) << hm.hbase[v];
  }
  return true;
}

}  // namespace

bool saga_tc_supports(int dtype, int d, int h_q, int h_k, int h_v) {
  HeadMap hm;
  return dtype == SAGA_BF16 && (d == 64 || d == 128) && make_head_map(h_q, h_k, h_v, hm);
}

bool saga_tc_scores_streamable(const float *rows, int64_t row_stride) {
  return rows != nullptr && (reinterpret_cast<uintptr_t>(rows) % 16) == 0 && row_stride % 4 == 0 &&
         row_stride > 0;
}

cudaError_t launch_saga_tc(const StepParams &p, int mode, int d, cudaStream_t st) {
  HeadMap hm;
  if (!make_head_map(p.h_q, p.h_k, p.h_v, hm)) return cudaErrorInvalidValue;
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
    if (mode == kModeDump) return launch_tc<DD, kModeDump, false>(p, kmap, qmap, hm, dev, st); \
    if (mode == kModeStep)                                                                    \
      return fs ? launch_tc<DD, kModeStep, true>(p, kmap, qmap, hm, dev, st)                  \
                : launch_tc<DD, kModeStep, false>(p, kmap, qmap, hm, dev, st);                \
    return fs ? launch_tc<DD, kModeStepTies, true>(p, kmap, qmap, hm, dev, st)                \
              : launch_tc<DD, kModeStepTies, false>(p, kmap, qmap, hm, dev, st);              \
  }
  SAGA_TC_LAUNCH(64)
  SAGA_TC_LAUNCH(128)
#undef SAGA_TC_LAUNCH
  return cudaErrorInvalidValue;
}

}  // namespace saga
