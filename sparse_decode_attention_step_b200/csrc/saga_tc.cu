// Tensor-core split kernel for bf16 caches (sm_100a): the same work as the
// SIMT split kernel (Eq. 2 scores, Atop-N item 1 compare and compaction,
// Eq. 7 sparse softmax + V gather, per-split states), with the score
// contraction on tcgen05.
//
// Per CTA = (sequence b, key head kh, split of l_kv):
//   warp 8 (one lane)   TMA producer: K tiles of 128 positions x d (bf16, 128B
//                       swizzle) into a ring of shared-memory stages.
//   warps 0-7           per 256-position chunk: thread 0 issues the MMAs
//                       S[128 keys][16 heads] = K_tile * Q^T (M=128, N=16,
//                       K=16 per instruction) into TMEM, two tiles per chunk;
//                       all 256 threads read one position's 16 head scores
//                       back from TMEM, scale by 1/sqrt(d), compare with tau,
//                       compact per head, and fold the kept V rows into the
//                       running (m, l, acc) of the heads each warp owns.
// Query heads beyond the group (G < 16) are zero rows of Q and never kept.
// Every wait is bounded; on a timeout the CTA sets SAGA_DEVERR_TIMEOUT,
// lets its in-flight copies and MMAs land (again bounded), frees TMEM and
// returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace saga {

namespace {

constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;     // + producer warp
constexpr int kTileKeys = 128;
constexpr int kChunkKeys = 2 * kTileKeys;
constexpr int kTmemCols = 32;                       // two 16-column accumulators
constexpr int kN = 16;                              // MMA N: query heads, padded
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(kTileKeys, kN);
constexpr int kBar = 1;                             // named barrier of the compute warps
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kBoxes = D / 64;                     // 64-column TMA boxes per tile
  static constexpr int kBoxBytes = kTileKeys * 128;         // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQBlockBytes = kN * 128;             // 16 rows x 128 bytes per box
  static constexpr int kQBytes = kBoxes * kQBlockBytes;
};

struct Header {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

template <int D, int GP>
struct Layout {
  static constexpr int off_stage = 0;
  static constexpr int off_q = Cfg<D>::kStages * Cfg<D>::kTileBytes;
  static constexpr int off_sel_t = off_q + Cfg<D>::kQBytes;
  static constexpr int off_sel_a = off_sel_t + GP * kChunkKeys * 4;
  static constexpr int off_tau = off_sel_a + GP * kChunkKeys * 4;
  static constexpr int off_woff = off_tau + 16 * 4;
  static constexpr int off_hcnt = off_woff + kComputeWarps * GP * 4;
  static constexpr int off_hdr = (off_hcnt + GP * 4 + 15) / 16 * 16;
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

template <int VPL>
__device__ __forceinline__ void vslice_bf16(const uint16_t *row, int lane, float (&v)[VPL]) {
  if constexpr (VPL == 2) {
    uint32_t a = __ldg(reinterpret_cast<const uint32_t *>(row) + lane);
    v[0] = bf16lo(a); v[1] = bf16hi(a);
  } else {
    uint2 a = __ldg(reinterpret_cast<const uint2 *>(row) + lane);
    v[0] = bf16lo(a.x); v[1] = bf16hi(a.x); v[2] = bf16lo(a.y); v[3] = bf16hi(a.y);
  }
}

template <int D, int GP>
__global__ void __launch_bounds__(kThreads, 2)
saga_tc_kernel(const StepParams p, const int mode, const __grid_constant__ CUtensorMap kmap) {
  using C = Cfg<D>;
  using Lo = Layout<D, GP>;
  constexpr int HPW = (GP + kComputeWarps - 1) / kComputeWarps;
  constexpr int VPL = D / 32;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = sm100::smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t *stages = smem + Lo::off_stage;
  uint16_t *qop = reinterpret_cast<uint16_t *>(smem + Lo::off_q);
  int(*sel_t)[kChunkKeys] = reinterpret_cast<int(*)[kChunkKeys]>(smem + Lo::off_sel_t);
  float(*sel_a)[kChunkKeys] = reinterpret_cast<float(*)[kChunkKeys]>(smem + Lo::off_sel_a);
  float *tau_s = reinterpret_cast<float *>(smem + Lo::off_tau);
  int(*warp_off)[GP] = reinterpret_cast<int(*)[GP]>(smem + Lo::off_woff);
  int *head_cnt = reinterpret_cast<int *>(smem + Lo::off_hcnt);
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

  // ---- set-up: barriers, TMEM, the Q operand, thresholds -------------------
  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      sm100::mbar_init(&hdr->full[i], 1);
      sm100::mbar_init(&hdr->empty[i], 1);
    }
    sm100::mbar_init(&hdr->mma_done, 1);
    hdr->abort = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&hdr->tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  if (tid < kComputeThreads) {
    const uint16_t *qg = static_cast<const uint16_t *>(p.q) + b * p.q_sb;
    for (int idx = tid; idx < kN * D; idx += kComputeThreads) {
      const int n = idx / D, k = idx % D;
      const uint16_t v = n < G ? qg[(j0 + n) * p.q_sh + k] : static_cast<uint16_t>(0);
      const int box = k / 64, kk = k % 64;
      const int off = box * C::kQBlockBytes + (n / 8) * 1024 + (n % 8) * 128 +
                      ((((kk * 2) >> 4) ^ (n % 8)) << 4) + ((kk * 2) & 15);
      qop[off / 2] = v;
    }
    sm100::fence_proxy_async_smem();
    if (tid < 16) tau_s[tid] = (tid < G && mode != kModeDump) ? p.tau[b * p.h_q + j0 + tid] : 0.f;
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = hdr->tmem_base;

  // ---- producer warp --------------------------------------------------------
  if (warp == kComputeWarps) {
    if (lane == 0) {
      sm100::prefetch_tensormap(&kmap);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % C::kStages, round = i / C::kStages;
        if (*reinterpret_cast<volatile int *>(&hdr->abort)) break;
        if (!sm100::mbar_wait(&hdr->empty[st], (round & 1) ^ 1)) { fail(p, hdr); break; }
        sm100::mbar_arrive_expect_tx(&hdr->full[st], C::kTileBytes);
        const int y = static_cast<int>(t_begin) + i * kTileKeys;
#pragma unroll
        for (int bx = 0; bx < C::kBoxes; ++bx)
          sm100::tma_load_4d(stages + st * C::kTileBytes + bx * C::kBoxBytes, &kmap,
                             &hdr->full[st], bx * 64, y, kh, b);
        issued = i + 1;
      }
      // let every copy still in flight land before the CTA can exit
      for (int i = issued > C::kStages ? issued - C::kStages : 0; i < issued; ++i)
        sm100::mbar_wait(&hdr->full[i % C::kStages], (i / C::kStages) & 1);
    }
    return;
  }

  // ---- compute warps --------------------------------------------------------
  const uint16_t *vbase0 = static_cast<const uint16_t *>(p.V) + b * p.v_sb;
  const int64_t row0 = static_cast<int64_t>(b * p.h_q + j0) * p.row_stride;
  float m_run[HPW], l_run[HPW], acc[HPW][VPL];
  int cnt_run[HPW];
#pragma unroll
  for (int r = 0; r < HPW; ++r) {
    m_run[r] = -INFINITY; l_run[r] = 0.f; cnt_run[r] = 0;
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[r][v] = 0.f;
  }
  const uint32_t q_u32 = sm100::smem_u32(qop);
  const uint32_t st_u32 = sm100::smem_u32(stages);
  bool bad = false;          // this thread saw a timeout
  int committed = 0;         // mma_done phases committed by thread 0

  for (int c = 0; c < n_chunks; ++c) {
    const int tile0 = 2 * c;
    const bool has1 = tile0 + 1 < n_tiles;
    if (tid == 0 && !bad) {
      sm100::tc_fence_after();
      for (int u = 0; u < (has1 ? 2 : 1); ++u) {
        const int tt = tile0 + u;
        const int st = tt % C::kStages, round = tt / C::kStages;
        if (!sm100::mbar_wait(&hdr->full[st], round & 1)) { fail(p, hdr); bad = true; break; }
        const uint32_t a0 = st_u32 + st * C::kTileBytes;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          const int bx = j / 4, kk = j % 4;
          const uint64_t ad = sm100::desc_k_sw128(a0 + bx * C::kBoxBytes + kk * 32);
          const uint64_t bd = sm100::desc_k_sw128(q_u32 + bx * C::kQBlockBytes + kk * 32);
          sm100::mma_bf16(tmem_base + u * kN, ad, bd, kIdesc, j > 0 ? 1u : 0u);
        }
        sm100::mma_commit(&hdr->empty[st]);
      }
      if (!bad) {
        sm100::mma_commit(&hdr->mma_done);
        ++committed;
      }
    }
    if (!bad && !sm100::mbar_wait(&hdr->mma_done, c & 1)) { fail(p, hdr); bad = true; }
    sm100::tc_fence_after();

    const int half = warp / 4, quarter = warp % 4;
    const int64_t base = t_begin + static_cast<int64_t>(c) * kChunkKeys;
    const int64_t t = base + half * kTileKeys + quarter * 32 + lane;
    const bool valid = !bad && t < t_end;
    float A[16];
    if (!bad && (half == 0 || has1)) {
      sm100::tmem_ld16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * kN, A);
    }
#pragma unroll
    for (int g = 0; g < 16; ++g) A[g] = A[g] * p.scale;
    sm100::tc_fence_before();

    if (mode == kModeDump) {
      if (valid) {
#pragma unroll
        for (int g = 0; g < GP; ++g)
          if (g < G) p.scores_out[row0 + g * p.row_stride + t] = A[g];
      }
      if (bar_any(bad)) break;
      continue;
    }

    // threshold compare + order-preserving compaction per head
    uint32_t selbits = 0;
    int pos[GP];
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const bool sel = valid && g < G && A[g] >= tau_s[g];
      const uint32_t bal = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) warp_off[warp][g] = __popc(bal);
      pos[g] = __popc(bal & lt_mask);
      selbits |= static_cast<uint32_t>(sel) << g;
    }
    if (p.sel_mask != nullptr && valid) {
      for (int g = 0; g < G; ++g)
        p.sel_mask[row0 + g * p.row_stride + t] = static_cast<uint8_t>((selbits >> g) & 1u);
    }
    sm100::named_bar(kBar, kComputeThreads);
    if (tid < GP) {
      int run = 0;
      for (int w = 0; w < kComputeWarps; ++w) {
        const int cc = warp_off[w][tid];
        warp_off[w][tid] = run;
        run += cc;
      }
      head_cnt[tid] = run;
    }
    sm100::named_bar(kBar, kComputeThreads);
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if ((selbits >> g) & 1u) {
        const int o = warp_off[warp][g] + pos[g];
        sel_t[g][o] = static_cast<int>(t - base);
        sel_a[g][o] = A[g];
      }
    }
    sm100::named_bar(kBar, kComputeThreads);

#pragma unroll
    for (int r = 0; r < HPW; ++r) {
      const int g = warp + r * kComputeWarps;
      if (g >= G) continue;
      const int n = head_cnt[g];
      if (n == 0) continue;
      float mc = -INFINITY;
      for (int e = lane; e < n; e += 32) mc = fmaxf(mc, sel_a[g][e]);
      mc = warp_max(mc);
      const float m_new = fmaxf(m_run[r], mc);
      const float corr = exp2f((m_run[r] - m_new) * kLog2e);
      l_run[r] *= corr;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc[r][v] *= corr;
      const int vh = ((j0 + g) * p.h_v) / p.h_q;
      const uint16_t *vb = vbase0 + vh * p.v_sh;
      int e = 0;
      for (; e + 4 <= n; e += 4) {
        float vv[4][VPL], pw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          vslice_bf16<VPL>(vb + (base + sel_t[g][e + u]) * D, lane, vv[u]);
          pw[u] = exp2f((sel_a[g][e + u] - m_new) * kLog2e);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          l_run[r] += pw[u];
#pragma unroll
          for (int v = 0; v < VPL; ++v) acc[r][v] = fmaf(pw[u], vv[u][v], acc[r][v]);
        }
      }
      for (; e < n; ++e) {
        float vv[VPL];
        vslice_bf16<VPL>(vb + (base + sel_t[g][e]) * D, lane, vv);
        const float pw = exp2f((sel_a[g][e] - m_new) * kLog2e);
        l_run[r] += pw;
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc[r][v] = fmaf(pw, vv[v], acc[r][v]);
      }
      m_run[r] = m_new;
      cnt_run[r] += n;
    }
    if (bar_any(bad)) break;
  }

  // ---- teardown: every MMA has landed before TMEM is freed -----------------
  if (tid == 0 && bad && committed > 0)
    sm100::mbar_wait(&hdr->mma_done, (committed - 1) & 1);
  sm100::tc_fence_before();
  sm100::named_bar(kBar, kComputeThreads);
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, kTmemCols);
  }
  if (mode == kModeDump || *reinterpret_cast<volatile int *>(&hdr->abort)) return;
#pragma unroll
  for (int r = 0; r < HPW; ++r) {
    const int g = warp + r * kComputeWarps;
    if (g >= G) continue;
    float *rec = p.partials + (static_cast<int64_t>(b * p.h_q + j0 + g) * p.S + s) * (D + kRecPad);
    if (lane == 0) {
      rec[0] = m_run[r];
      rec[1] = l_run[r];
      rec[2] = __int_as_float(cnt_run[r]);
      rec[3] = 0.f;
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) rec[kRecPad + lane * VPL + v] = acc[r][v];
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
  using Lo = Layout<D, GP>;
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
  const int gpr = gp <= 8 ? 8 : 16;
  if (d == 64) return gpr == 8 ? launch_tc<64, 8>(p, mode, map, st) : launch_tc<64, 16>(p, mode, map, st);
  return gpr == 8 ? launch_tc<128, 8>(p, mode, map, st) : launch_tc<128, 16>(p, mode, map, st);
}

}  // namespace saga
