// Closed-form GQA-to-SAGA key-head merge on B200 ("More Value per Key:
// Asymmetric Sparse Attention for Faster LLM Decoding", GQA-to-SAGA
// Conversion, Stage 1: Eq. 13-15 and Theorem 4.2).
//
// Data flow (one call, all on `stream`):
//   1. transpose Q [T][h_q d] -> Qt [h_q d][T]                (bf16, 64x64 tiles)
//   2. K^T = (X W^T)^T as bf16 hi + lo rows, Kt [2][h_k d][T]  (tcgen05 GEMM)
//   3. C = K^T K over T as hi.hi + hi.lo + lo.hi, split over T (tcgen05 GEMM)
//      S_r = sum_{j of r} Q^j^T Q^j, split over T                (tcgen05 GEMM)
//   4. partial sums -> float64 C and S_r
//   5. one CTA per pair (a, b), float64: P = (S_a + S_b)^+ (Gauss-Jordan inverse
//      when it provably is the pseudoinverse, else Jacobi eigen-decomposition),
//      A_a = S_a P, A_b = S_b P, w(a,b) = trace(D A_a S_b)
//   6. one CTA: minimum-weight perfect matching by a subset programme
//   7. W_S rows of merged head i = (W^a A_a + W^b A_b)^T for pairs[i]
// The GEMMs are the dense contractions (T = thousands of tokens); the
// per-pair algebra is d x d with d <= 128 and runs on the FP64 pipes.
//
// GEMM kernel: D[M x N] = sum over segments of A_s[M x 64k] B_s[N x 64k]^T,
// both operands K-major bf16 tiles of 128 rows x 64 columns loaded by TMA with
// the 128-byte swizzle, accumulated by tcgen05.mma (M = N = 128) in TMEM.
// Warp 0 issues the loads, warp 1 the MMAs, warps 2-5 (one TMEM lane quarter
// each) read the accumulator back and store it transposed, out[n][m], so a
// warp's 32 lanes write 32 consecutive elements.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "kernels.h"
#include "merge_math.cuh"
#include "saga.h"
#include "saga_merge.h"
#include "sm100.cuh"

namespace saga {
namespace merge {
namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- tcgen05 GEMM ---------------------------------------------------------
constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kGStages = 6;
constexpr int kOpBytes = kBM * kBK * 2;          // one operand tile: 16 KB
constexpr int kStageBytes = 2 * kOpBytes;
constexpr int kGemmThreads = 192;
constexpr int kTmemCols = kBN;                    // fp32 accumulator columns
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(kBM, kBN);
static_assert(kBN == kBM, "one TMA box shape serves both operands");

struct GemmArgs {
  int m_tiles;                 // blockIdx.x = n_tile * m_tiles + m_tile
  int kb_per_seg;              // 64-wide contraction blocks per segment
  int n_seg;                   // segments of the contraction
  int kb_per_split;            // contraction blocks per CTA (blockIdx.y)
  int a_off[4], b_off[4];      // extra operand row offset of segments 0..3
  int a_seg, b_seg;            // operand row offset per segment index
  int a_z, b_z;                // operand row offset per blockIdx.z
  int m_valid, n_valid;        // stored part of the output (global m, n)
  int split_bf16;              // 1: bf16 hi at out[n][m], lo at out[lo_off + n][m]
  void *out;
  long long ldo, out_split, out_z, lo_off;
  int32_t *err;
};

struct GemmHeader {
  uint64_t full[kGStages], empty[kGStages], done;
  uint32_t tmem_base;
  int abort;
};
constexpr int kGemmSmem = kGStages * kStageBytes + static_cast<int>(sizeof(GemmHeader)) + 1024;
static_assert(kGemmSmem <= 227 * 1024, "shared memory of one CTA");

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(sm100::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(sm100::smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool aborted(GemmHeader *h) {
  return *reinterpret_cast<volatile int *>(&h->abort) != 0;
}

__device__ __forceinline__ void fail(const GemmArgs &g, GemmHeader *h) {
  if (!aborted(h)) atomicOr(g.err, SAGA_DEVERR_TIMEOUT);
  *reinterpret_cast<volatile int *>(&h->abort) = 1;
}

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, GemmHeader *h) {
  if (sm100::mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::global_ns();
  for (;;) {
    if (sm100::mbar_try_wait_sleep(bar, parity, sm100::kSuspendHintNs)) return true;
    if (aborted(h)) return false;
    if (sm100::global_ns() - t0 > sm100::kWaitLimitNs) return false;
  }
}

// Extra row offset of segment s (selects, so the table stays in registers).
__device__ __forceinline__ int seg_off(const int (&t)[4], int s) {
  return s == 0 ? t[0] : s == 1 ? t[1] : s == 2 ? t[2] : s == 3 ? t[3] : 0;
}

__device__ __forceinline__ void store_out(const GemmArgs &g, long long o, float x) {
  if (g.split_bf16) {
    uint16_t *out = static_cast<uint16_t *>(g.out);
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    out[o] = __bfloat16_as_ushort(hi);
    out[g.lo_off + o] = __bfloat16_as_ushort(lo);
  } else {
    static_cast<float *>(g.out)[o] = x;
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    km_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                   const __grid_constant__ CUtensorMap bmap, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *stages = base;
  GemmHeader *h = reinterpret_cast<GemmHeader *>(base + kGStages * kStageBytes);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int mt = blockIdx.x % g.m_tiles, nt = blockIdx.x / g.m_tiles;
  const int z = blockIdx.z;
  const int total = g.n_seg * g.kb_per_seg;
  const int kb0 = blockIdx.y * g.kb_per_split;
  const int nk = max(0, min(total, kb0 + g.kb_per_split) - kb0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      sm100::mbar_init(&h->full[i], 1);
      sm100::mbar_init(&h->empty[i], 1);
    }
    sm100::mbar_init(&h->done, 1);
    h->abort = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(&h->tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = h->tmem_base;

  if (warp == 0) {
    // ---- TMA producer --------------------------------------------------------
    if (lane == 0 && nk > 0) {
      sm100::prefetch_tensormap(&amap);
      sm100::prefetch_tensormap(&bmap);
      int i = 0;
      bool ok = true;
      for (; i < nk; ++i) {
        const int st = i % kGStages;
        if (!wait_bar(&h->empty[st], ((i / kGStages) & 1) ^ 1, h)) {
          ok = false;
          break;
        }
        const int gk = kb0 + i, s = gk / g.kb_per_seg, kb = gk % g.kb_per_seg;
        const int ar = seg_off(g.a_off, s) + s * g.a_seg + z * g.a_z + mt * kBM;
        const int br = seg_off(g.b_off, s) + s * g.b_seg + z * g.b_z + nt * kBN;
        sm100::mbar_arrive_expect_tx(&h->full[st], kStageBytes);
        tma_load_2d(stages + st * kStageBytes, &amap, &h->full[st], kb * kBK, ar);
        tma_load_2d(stages + st * kStageBytes + kOpBytes, &bmap, &h->full[st], kb * kBK, br);
      }
      if (!ok) {
        fail(g, h);
        // the copies still in flight land before the CTA can exit
        for (int j = i > kGStages ? i - kGStages : 0; j < i; ++j)
          sm100::mbar_wait(&h->full[j % kGStages], (j / kGStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer ------------------------------------------------------------
    if (lane == 0 && nk > 0) {
      int i = 0;
      bool ok = true;
      for (; i < nk; ++i) {
        const int st = i % kGStages;
        if (!wait_bar(&h->full[st], (i / kGStages) & 1, h)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t a0 = sm100::smem_u32(stages + st * kStageBytes);
        const uint32_t b0 = a0 + kOpBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          sm100::mma_bf16(tmem, sm100::desc_k_sw128(a0 + kk * 32),
                          sm100::desc_k_sw128(b0 + kk * 32), kIdesc,
                          (i > 0 || kk > 0) ? 1u : 0u);
        sm100::mma_commit(&h->empty[st]);
      }
      if (ok) {
        sm100::mma_commit(&h->done);
      } else {
        fail(g, h);
        // every MMA issued has landed before TMEM and the stages go away
        if (i > 0) sm100::mbar_wait(&h->empty[(i - 1) % kGStages], ((i - 1) / kGStages) & 1);
      }
    }
    __syncwarp();
  } else {
    // ---- epilogue: TMEM lane quarter (warp % 4) -> out[n][m] ---------------------
    const int quarter = warp % 4;
    bool ok = true;
    if (nk > 0) {
      if (lane == 0) ok = wait_bar(&h->done, 0, h);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok && lane == 0) fail(g, h);
    }
    if (ok) {
      sm100::tc_fence_after();
      const int m = mt * kBM + quarter * 32 + lane;
      const long long obase = static_cast<long long>(z) * g.out_z +
                              static_cast<long long>(blockIdx.y) * g.out_split;
      for (int c0 = 0; c0 < kBN; c0 += 16) {
        float v[16];
        if (nk > 0) {
          sm100::tmem_ld16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + c0, v);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.0f;
        }
        if (m < g.m_valid) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = nt * kBN + c0 + j;
            if (n < g.n_valid) store_out(g, obase + static_cast<long long>(n) * g.ldo + m, v[j]);
          }
        }
      }
    }
  }

  // ---- teardown: every MMA and TMEM read is done before TMEM is freed -----------
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- transpose of the queries -----------------------------------------------
// out[c][t] = in[t][c], in [rows][cols] bf16 bits, rows and cols even.
__global__ void __launch_bounds__(256)
    km_transpose_kernel(const uint16_t *__restrict__ in, int rows, int cols,
                        uint16_t *__restrict__ out) {
  __shared__ uint16_t tile[64][66];
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + ty + 8 * i, c = c0 + 2 * tx;
    uint32_t v = 0;
    if (r < rows && c < cols)
      v = *reinterpret_cast<const uint32_t *>(in + static_cast<size_t>(r) * cols + c);
    tile[ty + 8 * i][2 * tx] = static_cast<uint16_t>(v & 0xFFFFu);
    tile[ty + 8 * i][2 * tx + 1] = static_cast<uint16_t>(v >> 16);
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = c0 + ty + 8 * i, r = r0 + 2 * tx;
    if (c < cols && r < rows) {
      const uint32_t v = static_cast<uint32_t>(tile[2 * tx][ty + 8 * i]) |
                         (static_cast<uint32_t>(tile[2 * tx + 1][ty + 8 * i]) << 16);
      *reinterpret_cast<uint32_t *>(out + static_cast<size_t>(c) * rows + r) = v;
    }
  }
}

// out[e] = sum over splits s (in order) of part[s * stride + e], in float64.
__global__ void __launch_bounds__(256)
    km_reduce_kernel(const float *__restrict__ part, long long n, int splits, long long stride,
                     double *__restrict__ out) {
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    double acc = 0.0;
    for (int s = 0; s < splits; ++s) acc += static_cast<double>(part[s * stride + e]);
    out[e] = acc;
  }
}

// ---- one CTA per pair ----------------------------------------------------------
constexpr int kPairThreads = 512;

template <int D, typename VT>
struct PairSmem {
  static constexpr size_t bytes = sizeof(double) * D * D + sizeof(VT) * D * D +
                                  sizeof(double) * (D / 2) * 2 + sizeof(double) * D * 2;
  static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

template <int D, typename VT>
__global__ void __launch_bounds__(kPairThreads, 1)
    km_pair_kernel(const double *__restrict__ S_sum, const double *__restrict__ C_sum, int h_k,
                   double rcond, double *__restrict__ Ag, double *__restrict__ w) {
  extern __shared__ __align__(16) uint8_t pair_smem[];
  double *S = reinterpret_cast<double *>(pair_smem);
  VT *E = reinterpret_cast<VT *>(S + D * D);
  double *rc = reinterpret_cast<double *>(E + D * D);
  double *rs = rc + D / 2;
  double *rowbuf = rs + D / 2;
  double *inv = rowbuf + D;
  int a, b;
  pair_of(blockIdx.x, h_k, a, b);
  const Team tm{static_cast<int>(threadIdx.x), static_cast<int>(blockDim.x)};
  const double wab = pair_stage<VT>(tm, D, S_sum + static_cast<size_t>(a) * D * D,
                                    S_sum + static_cast<size_t>(b) * D * D, C_sum,
                                    static_cast<long long>(h_k) * D, a, b, rcond, S, E, rc, rs,
                                    rowbuf, inv, Ag + static_cast<size_t>(blockIdx.x) * 2 * D * D,
                                    true, nullptr);
  if (threadIdx.x == 0) {
    w[a * h_k + b] = wab;
    w[b * h_k + a] = wab;
  }
}

// ---- the matching ------------------------------------------------------------------
constexpr int kMatchThreads = 1024;

__global__ void __launch_bounds__(kMatchThreads)
    km_match_kernel(double *__restrict__ w, int n, double *__restrict__ f,
                    int8_t *__restrict__ choice, int32_t *__restrict__ pairs,
                    double *__restrict__ total) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) w[i * n + i] = 0.0;
  __syncthreads();
  const Team tm{static_cast<int>(threadIdx.x), static_cast<int>(blockDim.x)};
  match_dp(tm, n, w, f, choice);
  if (threadIdx.x == 0) {
    match_pairs(n, choice, pairs);
    if (total != nullptr) *total = f[(1u << n) - 1u];
  }
}

// ---- the student's key projection ------------------------------------------------
// W_S[i*d + c][x] = sum_m W_lin[a*d + m][x] A_a[m][c] + sum_m W_lin[b*d + m][x] A_b[m][c]
// for (a, b) = pairs[i]; the sum runs as in merged_elem. Grid
// (ceil(d_model / 128), d / 16, h_k / 2); a thread owns one x and 16 c.
constexpr int kProjX = 128, kProjC = 16;

template <int D>
__global__ void __launch_bounds__(kProjX)
    km_project_kernel(const uint16_t *__restrict__ W_lin, int d_model, int h_k,
                      const int32_t *__restrict__ pairs, const double *__restrict__ Ag,
                      float *__restrict__ W_S) {
  __shared__ double sA[2][D][kProjC];
  const int i = blockIdx.z, c0 = blockIdx.y * kProjC;
  const int a = pairs[2 * i], b = pairs[2 * i + 1];
  const double *A = Ag + static_cast<size_t>(pair_index(a, b, h_k)) * 2 * D * D;
  for (int e = threadIdx.x; e < 2 * D * kProjC; e += blockDim.x) {
    const int r = e / (D * kProjC), m = (e / kProjC) % D, c = e % kProjC;
    sA[r][m][c] = A[static_cast<size_t>(r) * D * D + static_cast<size_t>(m) * D + c0 + c];
  }
  __syncthreads();
  const int x = blockIdx.x * kProjX + threadIdx.x;
  if (x >= d_model) return;
  double acc[kProjC];
#pragma unroll
  for (int c = 0; c < kProjC; ++c) acc[c] = 0.0;
  for (int r = 0; r < 2; ++r) {
    const uint16_t *Wr = W_lin + static_cast<size_t>(r == 0 ? a : b) * D * d_model + x;
#pragma unroll 4
    for (int m = 0; m < D; ++m) {
      const double wv = static_cast<double>(
          __uint_as_float(static_cast<uint32_t>(Wr[static_cast<size_t>(m) * d_model]) << 16));
#pragma unroll
      for (int c = 0; c < kProjC; ++c) acc[c] = fma(wv, sA[r][m][c], acc[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < kProjC; ++c)
    W_S[(static_cast<size_t>(i) * D + c0 + c) * d_model + x] = static_cast<float>(acc[c]);
}

// ---- host side -------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point; resolved once.
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

// 2-D bf16 map of a row-major [rows][inner] matrix: 128-row x 64-column boxes,
// 128-byte swizzle, zero fill outside.
bool make_map(EncodeTiledFn enc, CUtensorMap *map, const void *ptr, int64_t inner, int64_t rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * 2};
  const cuuint32_t box[2] = {kBK, kBM};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;
constexpr int64_t kSms = 148;   // B200: the split-K plans aim at one wave of CTAs

// Opt in to the dynamic shared memory a kernel needs (per device, once).
template <typename K>
cudaError_t set_smem(K kernel, int bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

cudaError_t launch_gemm(const CUtensorMap &amap, const CUtensorMap &bmap, const GemmArgs &g,
                        int n_tiles, int splits, int batches, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = set_smem(km_gemm_kernel, kGemmSmem, attr);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(g.m_tiles * n_tiles), static_cast<unsigned>(splits),
                  static_cast<unsigned>(batches));
  km_gemm_kernel<<<grid, kGemmThreads, kGemmSmem, st>>>(amap, bmap, g);
  return cudaGetLastError();
}

template <int D, typename VT>
cudaError_t launch_pair(const double *S_sum, const double *C_sum, int h_k, double rcond,
                        double *Ag, double *w, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  const int bytes = static_cast<int>(PairSmem<D, VT>::bytes);
  cudaError_t e = set_smem(km_pair_kernel<D, VT>, bytes, attr);
  if (e != cudaSuccess) return e;
  const int n_pairs = h_k * (h_k - 1) / 2;
  km_pair_kernel<D, VT><<<n_pairs, kPairThreads, bytes, st>>>(S_sum, C_sum, h_k, rcond, Ag, w);
  return cudaGetLastError();
}

// Split of a contraction of `total` blocks over about `want` CTAs, none empty.
void split_plan(int64_t total, int64_t want, int &splits, int &per_split) {
  const int64_t s = std::max<int64_t>(1, std::min<int64_t>(total, want));
  per_split = static_cast<int>(ceil_div(total, s));
  splits = static_cast<int>(ceil_div(total, per_split));
}

struct MergePlan {
  int HD, splits_c, per_c, splits_s, per_s, n_pairs;
  size_t off_qt, off_kt, off_cpart, off_spart, off_csum, off_ssum, off_ag, off_f, off_choice,
      total;
};

bool valid_shape(const saga_merge_shape *s) {
  return s != nullptr && s->T >= 128 && s->T % 8 == 0 && s->d_model >= 64 &&
         s->d_model % 8 == 0 && s->h_k >= 2 && s->h_k % 2 == 0 && s->h_q >= s->h_k &&
         s->h_q % s->h_k == 0 && s->d > 0;
}

// Sizes the kernels' index types and grids take: the transpose grid spans
// T / 64 rows of blocks (at most 65535), the subset table 2^h_k entries.
bool supported_shape(const saga_merge_shape *s) {
  return (s->d == 64 || s->d == 128) && s->h_k <= 16 &&
         static_cast<int64_t>(s->h_q) * s->d <= (1 << 20) && s->T <= (1 << 21) &&
         s->d_model <= (1 << 20);
}

MergePlan make_plan(const saga_merge_shape &s) {
  const int64_t sms = kSms;
  MergePlan p{};
  p.HD = s.h_k * s.d;
  const int64_t t_blocks = ceil_div(s.T, kBK);
  const int64_t c_tiles = ceil_div(p.HD, kBM) * ceil_div(p.HD, kBN);
  split_plan(3 * t_blocks, std::max<int64_t>(1, sms / c_tiles), p.splits_c, p.per_c);
  split_plan((s.h_q / s.h_k) * t_blocks, std::max<int64_t>(1, sms / s.h_k), p.splits_s,
             p.per_s);
  p.n_pairs = s.h_k * (s.h_k - 1) / 2;
  const size_t d2 = static_cast<size_t>(s.d) * s.d;
  p.off_qt = kAlign;   // [0, 256): device error word
  p.off_kt = align_up(p.off_qt + static_cast<size_t>(s.h_q) * s.d * s.T * 2);
  p.off_cpart = align_up(p.off_kt + 2 * static_cast<size_t>(p.HD) * s.T * 2);
  p.off_spart = align_up(p.off_cpart + static_cast<size_t>(p.splits_c) * p.HD * p.HD * 4);
  p.off_csum = align_up(p.off_spart + static_cast<size_t>(p.splits_s) * s.h_k * d2 * 4);
  p.off_ssum = align_up(p.off_csum + static_cast<size_t>(p.HD) * p.HD * 8);
  p.off_ag = align_up(p.off_ssum + static_cast<size_t>(s.h_k) * d2 * 8);
  p.off_f = align_up(p.off_ag + static_cast<size_t>(p.n_pairs) * 2 * d2 * 8);
  p.off_choice = align_up(p.off_f + (static_cast<size_t>(1) << s.h_k) * 8);
  p.total = align_up(p.off_choice + (static_cast<size_t>(1) << s.h_k));
  return p;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace merge
}  // namespace saga

using namespace saga::merge;
using saga::cuda_fail;

extern "C" size_t saga_merge_workspace_size(const saga_merge_shape *shape) {
  if (!valid_shape(shape) || !supported_shape(shape)) return 0;
  return make_plan(*shape).total;
}

extern "C" saga_status saga_merge_keys(const saga_merge_shape *shape, const void *X,
                                       const void *W_K, const void *Q, double rcond, double *w,
                                       int32_t *pairs, double *total, float *W_S, void *ws,
                                       size_t ws_bytes, saga_stream_t stream) {
  if (!valid_shape(shape)) return SAGA_ERR_INVALID_ARG;
  if (!supported_shape(shape)) return SAGA_ERR_UNSUPPORTED;
  if (!(rcond >= 0.0) || X == nullptr || W_K == nullptr || Q == nullptr || w == nullptr ||
      pairs == nullptr || W_S == nullptr)
    return SAGA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(W_K, 16) || !aligned(Q, 16) || !aligned(w, 8) ||
      !aligned(pairs, 4) || !aligned(W_S, 4) || (total != nullptr && !aligned(total, 8)))
    return SAGA_ERR_INVALID_ARG;
  const saga_merge_shape &s = *shape;
  const MergePlan p = make_plan(s);
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < p.total) return SAGA_ERR_WORKSPACE;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cuda_fail(cudaErrorNotSupported, "cuTensorMapEncodeTiled entry point");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *wsb = static_cast<char *>(ws);
  int32_t *err = reinterpret_cast<int32_t *>(wsb);
  uint16_t *Qt = reinterpret_cast<uint16_t *>(wsb + p.off_qt);
  uint16_t *Kt = reinterpret_cast<uint16_t *>(wsb + p.off_kt);
  float *C_part = reinterpret_cast<float *>(wsb + p.off_cpart);
  float *S_part = reinterpret_cast<float *>(wsb + p.off_spart);
  double *C_sum = reinterpret_cast<double *>(wsb + p.off_csum);
  double *S_sum = reinterpret_cast<double *>(wsb + p.off_ssum);
  double *Ag = reinterpret_cast<double *>(wsb + p.off_ag);
  double *f = reinterpret_cast<double *>(wsb + p.off_f);
  int8_t *choice = reinterpret_cast<int8_t *>(wsb + p.off_choice);
  const int d = s.d, HD = p.HD, T = s.T, G = s.h_q / s.h_k;

  CUtensorMap xmap, wmap, ktmap, qtmap;
  if (!make_map(enc, &xmap, X, s.d_model, T) || !make_map(enc, &wmap, W_K, s.d_model, HD) ||
      !make_map(enc, &ktmap, Kt, T, 2 * static_cast<int64_t>(HD)) ||
      !make_map(enc, &qtmap, Qt, T, static_cast<int64_t>(s.h_q) * d))
    return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled (key merge)");

  // 1. Qt = Q^T
  {
    const dim3 grid(static_cast<unsigned>(ceil_div(static_cast<int64_t>(s.h_q) * d, 64)),
                    static_cast<unsigned>(ceil_div(T, 64)));
    km_transpose_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t *>(Q), T, s.h_q * d, Qt);
    if (const cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_fail(e, "transpose kernel");
  }
  // 2. Kt[n][t] = (X W^T)[t][n] as bf16 hi and lo rows
  {
    GemmArgs g{};
    g.m_tiles = static_cast<int>(ceil_div(T, kBM));
    g.kb_per_seg = static_cast<int>(ceil_div(s.d_model, kBK));
    g.n_seg = 1;
    g.kb_per_split = g.kb_per_seg;
    g.m_valid = T;
    g.n_valid = HD;
    g.split_bf16 = 1;
    g.out = Kt;
    g.ldo = T;
    g.lo_off = static_cast<long long>(HD) * T;
    g.err = err;
    const cudaError_t e = launch_gemm(xmap, wmap, g, static_cast<int>(ceil_div(HD, kBN)), 1, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "key GEMM");
  }
  // 3a. C partials: segments hi.hi, hi.lo, lo.hi over T
  {
    GemmArgs g{};
    g.m_tiles = static_cast<int>(ceil_div(HD, kBM));
    g.kb_per_seg = static_cast<int>(ceil_div(T, kBK));
    g.n_seg = 3;
    g.kb_per_split = p.per_c;
    g.a_off[0] = 0; g.b_off[0] = 0;
    g.a_off[1] = 0; g.b_off[1] = HD;
    g.a_off[2] = HD; g.b_off[2] = 0;
    g.m_valid = HD;
    g.n_valid = HD;
    g.out = C_part;
    g.ldo = HD;
    g.out_split = static_cast<long long>(HD) * HD;
    g.err = err;
    const cudaError_t e = launch_gemm(ktmap, ktmap, g, static_cast<int>(ceil_div(HD, kBN)),
                                      p.splits_c, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "key Gram GEMM");
  }
  // 3b. S partials: batch r, one segment per query head j = r*G + s; rows j*d ..
  {
    GemmArgs g{};
    g.m_tiles = 1;
    g.kb_per_seg = static_cast<int>(ceil_div(T, kBK));
    g.n_seg = G;
    g.kb_per_split = p.per_s;
    g.a_seg = d; g.b_seg = d;
    g.a_z = G * d; g.b_z = G * d;
    g.m_valid = d;
    g.n_valid = d;
    g.out = S_part;
    g.ldo = d;
    g.out_z = static_cast<long long>(d) * d;
    g.out_split = static_cast<long long>(s.h_k) * d * d;
    g.err = err;
    const cudaError_t e = launch_gemm(qtmap, qtmap, g, 1, p.splits_s, s.h_k, st);
    if (e != cudaSuccess) return cuda_fail(e, "query Gram GEMM");
  }
  // 4. float64 sums of the partials
  {
    const long long nc = static_cast<long long>(HD) * HD;
    const long long ns = static_cast<long long>(s.h_k) * d * d;
    km_reduce_kernel<<<static_cast<unsigned>(std::min<long long>(ceil_div(nc, 256), 4096)), 256,
                       0, st>>>(C_part, nc, p.splits_c, nc, C_sum);
    km_reduce_kernel<<<static_cast<unsigned>(std::min<long long>(ceil_div(ns, 256), 4096)), 256,
                       0, st>>>(S_part, ns, p.splits_s, ns, S_sum);
    if (const cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_fail(e, "reduce kernel");
  }
  // 5. per pair: pseudoinverse, A_a, A_b, w(a, b)
  {
    const cudaError_t e = d == 64 ? launch_pair<64, double>(S_sum, C_sum, s.h_k, rcond, Ag, w, st)
                                  : launch_pair<128, float>(S_sum, C_sum, s.h_k, rcond, Ag, w, st);
    if (e != cudaSuccess) return cuda_fail(e, "pair kernel");
  }
  // 6. the matching
  km_match_kernel<<<1, kMatchThreads, 0, st>>>(w, s.h_k, f, choice, pairs, total);
  if (const cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_fail(e, "matching kernel");
  // 7. the student's key projection
  {
    const dim3 grid(static_cast<unsigned>(ceil_div(s.d_model, kProjX)),
                    static_cast<unsigned>(d / kProjC), static_cast<unsigned>(s.h_k / 2));
    if (d == 64)
      km_project_kernel<64><<<grid, kProjX, 0, st>>>(static_cast<const uint16_t *>(W_K),
                                                    s.d_model, s.h_k, pairs, Ag, W_S);
    else
      km_project_kernel<128><<<grid, kProjX, 0, st>>>(static_cast<const uint16_t *>(W_K),
                                                     s.d_model, s.h_k, pairs, Ag, W_S);
    if (const cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_fail(e, "projection kernel");
  }
  return SAGA_OK;
}
