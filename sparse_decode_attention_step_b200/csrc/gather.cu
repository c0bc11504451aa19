// Gather kernel: the V-row half of the tensor-core decode step (Eq. 7 over
// the kept entries of Atop-N item 1, split along l_kv).
//
// The tensor-core scan kernel leaves, for every 32-position block of every
// query head's row (b, j), a 32-bit mask of the kept positions and, at
// fixed places, their scores. This kernel turns them into per-split
// online-softmax records (m, l, count, acc[d]) for each query head, the
// records the combine kernel merges into out.
//
// One CTA of four warps per (b, j, split), eight CTAs per SM. A warp walks
// its share of the split's blocks, loading up to 256 blocks' masks at once
// (one lane per block), and lists the kept positions of each group of 32
// blocks in shared memory (block, key, rank), in position order. Each listed
// row is issued at once into the next free slot of the warp's staging area:
// each lane copies (cp.async) its 16-byte chunk of a row of value head
// floor(j * h_v / h_q) (d/8 lanes per row), and one lane per row the row's
// score, so the rows in flight cost no registers and every SM has several
// hundred of them in flight, which the latency of random row reads needs.
// When the kBatch slots are full, the copies land and each lane group folds
// its rows into one online-softmax state (every
// FMA does useful work: a row kept by several heads of one value head is
// read once per head, about 3% more rows on the workloads here); the lane
// groups and then the warps merge in a fixed order, so the result does not
// depend on timing, and the CTA writes the head's record.
//
// A scan that gave up on a bounded wait sets the step's abort word; this
// kernel then writes poisoned records (m = +inf, count = -1), which the
// combine turns into NaN outputs.
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace saga {

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct GCfg {
  static constexpr int LPG = D / 8;           // lanes per V row, 16 bytes each
  static constexpr int NG = 32 / LPG;         // lane groups per warp
  static constexpr int kRows = 8;             // rows per lane group and batch
  static constexpr int kBatch = NG * kRows;   // rows per warp and batch: 32 (d 64), 16 (d 128)
  static constexpr int kRec = D + kRecPad;
  // per warp: a 32-block group's list of kept rows (u16 entries), the staged
  // V rows and the staged scores
  static constexpr int kListBytes = 32 * 32 * 2;
  static constexpr int kVBytes = kBatch * D * 2;
  static constexpr int kScBytes = kBatch * 4;
  static constexpr int kWarpBytes = kListBytes + kVBytes + kScBytes;
  static constexpr int kMergeBytes = kWarps * kRec * 4;
  static constexpr int kSmem = kWarps * kWarpBytes > kMergeBytes ? kWarps * kWarpBytes : kMergeBytes;
};

// 2^x by the hardware's approximate exponential (relative error near 2^-22,
// well inside the step's tolerance); x <= 0 here, and 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 8) gather_kernel(const GatherParams p) {
  using C = GCfg<D>;
  constexpr int LPG = C::LPG, NG = C::NG, kRows = C::kRows, kBatch = C::kBatch;
  extern __shared__ __align__(16) uint8_t gsm[];
  pdl_wait();
  pdl_trigger();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lg = lane / LPG, c = lane % LPG;
  const int sb = blockIdx.x % p.SB;
  const int bj = blockIdx.x / p.SB;                  // b * h_q + j
  const int b = bj / p.h_q, j = bj % p.h_q;
  const int vh = j / p.hpv;

  int64_t L = p.l_kv[b];
  const int64_t hi = p.cap < p.max_l_kv ? p.cap : p.max_l_kv;
  L = L < 0 ? 0 : (L > hi ? hi : L);
  const int64_t nb_row = (L + 31) / 32;
  const int64_t blk0 = static_cast<int64_t>(sb) * p.blk_per_split;
  if (blk0 >= nb_row) return;                       // beyond l_kv: the combine skips it
  const int64_t blk1 = min(blk0 + p.blk_per_split, nb_row);

  float *rec = p.partials + (static_cast<int64_t>(bj) * p.SB + sb) * C::kRec;
  if (*reinterpret_cast<volatile const int32_t *>(p.abort) != 0) {
    // the scan of this step gave up: poison this split's record
    if (tid == 0) {
      rec[0] = INFINITY;
      rec[1] = __int_as_float(0x7fc00000);
      rec[2] = __int_as_float(-1);
      rec[3] = 0.f;
    }
    return;
  }

  const uint32_t *mask = p.lmask + static_cast<int64_t>(bj) * p.nblk;
  const float *sco = p.lscore + static_cast<int64_t>(bj) * p.nblk * 32;
  const uint16_t *vrow = p.V + b * p.v_sb + static_cast<int64_t>(vh) * p.v_sh;
  uint8_t *wbase = gsm + warp * C::kWarpBytes;
  uint16_t *list = reinterpret_cast<uint16_t *>(wbase);
  uint16_t *vst = reinterpret_cast<uint16_t *>(wbase + C::kListBytes);
  float *sst = reinterpret_cast<float *>(wbase + C::kListBytes + C::kVBytes);

  float m = -INFINITY, l = 0.f, acc[8];
  int cnt = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  // Staging: kBatch row slots per warp; slot i belongs to lane group i % NG.
  // Rows are issued into the next free slots as their group's list is read
  // (each lane copies its chunk of a row's V, one lane per row the row's
  // score); when all kBatch slots hold rows in flight, the warp waits for
  // them and folds them. So every wait covers a full batch, and the copies
  // of a partly filled batch stay in flight while the next groups' lists
  // are built.
  int nst = 0;                         // slots issued since the last fold
  auto fold = [&](int nb) {
    sm100::cp_async_commit();
    sm100::cp_async_wait_all();
    __syncwarp();
    float mnew = m;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int i = NG * r + lg;
      if (i < nb) mnew = fmaxf(mnew, sst[i]);
    }
    if (mnew != m) {
      const float corr = exp2f((m - mnew) * kLog2e);      // 0 while m = -inf
      m = mnew;
      l *= corr;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= corr;
    }
    cnt += max(0, min(kRows, (nb - lg + NG - 1) / NG));   // rows of this lane group
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (NG * r >= nb) break;
      const int i = NG * r + lg;
      if (i < nb) {
        const float pw = ex2((sst[i] - m) * kLog2e);
        const uint4 x = *reinterpret_cast<const uint4 *>(vst + i * D + c * 8);
        const float vf[8] = {bf16lo(x.x), bf16hi(x.x), bf16lo(x.y), bf16hi(x.y),
                             bf16lo(x.z), bf16hi(x.z), bf16lo(x.w), bf16hi(x.w)};
        l += pw;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(pw, vf[e], acc[e]);
      }
    }
    __syncwarp();            // the staged rows are read before the next copies
  };
  // Issue the listed rows [0, total) of the group of blocks from gb0.
  auto run_list = [&](int total, int64_t gb0) {
    // the group's V rows and kept scores, addressed from its first block
    const uint16_t *vg = vrow + gb0 * 32 * D + c * 8;
    const float *sg = sco + gb0 * 32;
    for (int pos = 0; pos < total;) {
      const int n = min(kBatch - nst, total - pos);
      // this lane group's slots i = NG * r + lg in [nst, nst + n)
      const int r_lo = max(0, (nst - lg + NG - 1) / NG);
      const int r_hi = min(kRows, (nst + n - lg + NG - 1) / NG);
      for (int r = r_lo; r < r_hi; ++r) {
        const int i = NG * r + lg;
        {
          const uint32_t en = list[pos + i - nst];
          const uint32_t bl = en >> 10;                        // block within the group
          // a listed row lies inside the sequence and the split
          if (saga_in_bounds(gb0 + bl < blk1 && (gb0 + bl) * 32 + ((en >> 5) & 31) < L, p.err)) {
            sm100::cp_async16(vst + i * D + c * 8, vg + (bl * 32 + ((en >> 5) & 31)) * D);
            if (c == 0) sm100::cp_async4(sst + i, sg + bl * 32 + (en & 31));
          }
        }
      }
      nst += n;
      pos += n;
      if (nst == kBatch) {
        fold(kBatch);
        nst = 0;
      }
    }
  };

  // this warp's blocks: an even share of the split, in order, taken in
  // chunks of up to kChunkGroups groups of 32 blocks whose masks are loaded
  // at once (one lane per block), so a group's list waits for no load; each
  // group's kept rows are listed as (block lane << 10 | key << 5 | rank)
  constexpr int kChunkGroups = 8;
  const int64_t nbs = blk1 - blk0;
  const int64_t per = (nbs + kWarps - 1) / kWarps;
  const int64_t wb0 = blk0 + min(nbs, per * warp), wb1 = blk0 + min(nbs, per * (warp + 1));
  for (int64_t cb = wb0; cb < wb1; cb += 32 * kChunkGroups) {
    uint32_t mks[kChunkGroups];
#pragma unroll
    for (int q = 0; q < kChunkGroups; ++q) {
      const int64_t blk = cb + q * 32 + lane;
      mks[q] = blk < wb1 ? __ldg(mask + blk) : 0u;
    }
#pragma unroll
    for (int q = 0; q < kChunkGroups; ++q) {
      const int64_t bb = cb + q * 32;
      if (bb >= wb1) break;
      uint32_t mk = mks[q];
      const int cn = __popc(mk);
      int incl = cn;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (total == 0) continue;
      for (int e = incl - cn, rank = 0; mk != 0u; ++e, ++rank) {
        const int k = __ffs(mk) - 1;
        mk &= mk - 1u;
        list[e] = static_cast<uint16_t>((lane << 10) | (k << 5) | rank);
      }
      __syncwarp();
      run_list(total, bb);
      __syncwarp();          // the list is read before the next group's is written
    }
  }
  if (nst > 0) fold(nst);

  // the warp's lane groups, merged by xor shuffles (a fixed order)
  {
    float mm = m;
#pragma unroll
    for (int o = LPG; o < 32; o <<= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
    const float s = m == -INFINITY ? 0.f : exp2f((m - mm) * kLog2e);
    l *= s;
#pragma unroll
    for (int o = LPG; o < 32; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = acc[e] * s;
#pragma unroll
      for (int o = LPG; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      acc[e] = x;
    }
    m = mm;
  }
  __syncthreads();                // every warp is done with its staging area
  float *st = reinterpret_cast<float *>(gsm);    // [kWarps][kRec]
  if (lg == 0) {
    float *r = st + warp * C::kRec;
    if (c == 0) {
      r[0] = m;
      r[1] = l;
      r[2] = __int_as_float(cnt);
    }
    float4 *dst = reinterpret_cast<float4 *>(r + kRecPad + c * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  __syncthreads();
  // the warps, merged in warp order: the head's record
  for (int e = tid; e < D; e += kThreads) {
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, st[w * C::kRec]);
    float ll = 0.f, aa = 0.f;
    int nn = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float *r = st + w * C::kRec;
      const float wt = r[0] == -INFINITY ? 0.f : exp2f((r[0] - mm) * kLog2e);
      ll = fmaf(wt, r[1], ll);
      nn += __float_as_int(r[2]);
      aa = fmaf(wt, r[kRecPad + e], aa);
    }
    rec[kRecPad + e] = aa;
    if (e == 0) {
      rec[0] = mm;
      rec[1] = ll;
      rec[2] = __int_as_float(nn);
      rec[3] = 0.f;
    }
  }
}

constexpr int kMaxDevices = 64;

template <int D>
cudaError_t launch_d(const GatherParams &p, unsigned grid, cudaStream_t st) {
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(gather_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  return launch_pdl(gather_kernel<D>, dim3(grid), dim3(kThreads), GCfg<D>::kSmem, st, p);
}

}  // namespace

cudaError_t launch_gather(const GatherParams &p, int d, cudaStream_t st) {
  const long long grid = static_cast<long long>(p.B) * p.h_q * p.SB;
  if (grid < 1) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (d == 64) return launch_d<64>(p, static_cast<unsigned>(grid), st);
  if (d == 128) return launch_d<128>(p, static_cast<unsigned>(grid), st);
  return cudaErrorInvalidValue;
}

}  // namespace saga
