// Dense decode split kernel: full attention, Eq. (2-4) over every position,
// for GQA (h_k == h_v) and for SAGA's asymmetric heads (h_k < h_v: the G query
// heads of a key head read VPG value heads, G / VPG query heads each). One CTA
// per (b, key head, split of l_kv). Each sub-chunk of 256 positions is scored
// (one position per thread, all G query heads of the group), the chunk
// maximum updates the running softmax state, and the probabilities weight the
// V rows (the VPG rows of one position per warp-iteration, d split across the
// lanes). The per-split states go to the same combine kernel as the sparse
// step.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = kThreads;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int D, int GP>
__device__ __forceinline__ void dense_scores(const T *krow, const float *qs, float scale,
                                             float (&A)[GP]) {
  float acc[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) acc[g] = 0.f;
#pragma unroll 2
  for (int c = 0; c < D; c += 8) {
    float k[8];
    load8(krow + c, k);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float4 *qv = reinterpret_cast<const float4 *>(qs + (c + e) * GP);
#pragma unroll
      for (int g4 = 0; g4 < GP / 4; ++g4) {
        float4 w = qv[g4];
        acc[4 * g4 + 0] = fmaf(w.x, k[e], acc[4 * g4 + 0]);
        acc[4 * g4 + 1] = fmaf(w.y, k[e], acc[4 * g4 + 1]);
        acc[4 * g4 + 2] = fmaf(w.z, k[e], acc[4 * g4 + 2]);
        acc[4 * g4 + 3] = fmaf(w.w, k[e], acc[4 * g4 + 3]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) A[g] = acc[g] * scale;
}

// bf16 caches: the scores of one warp's 32 positions (two m16 row tiles)
// against the GP query heads on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate; bf16 products are exact in fp32, so only the summation
// order differs from the FMA chain). Rows past `last` re-read row `last`.
// qb: the heads' B fragments, per 16-column slice and 8-head tile.
template <int D, int NT>
__device__ __forceinline__ void mma_scores(const uint16_t *krow0, int64_t key0, int64_t last,
                                           const uint32_t (&qb)[D / 16][NT][2], float *sc,
                                           int gp, int lane) {
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int64_t r0 = min(key0 + mt * 16 + g, last), r1 = min(key0 + mt * 16 + g + 8, last);
    const uint32_t *p0 = reinterpret_cast<const uint32_t *>(krow0 + r0 * D);
    const uint32_t *p1 = reinterpret_cast<const uint32_t *>(krow0 + r1 * D);
    float d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t a0 = __ldg(p0 + ks * 8 + tq), a1 = __ldg(p1 + ks * 8 + tq);
      const uint32_t a2 = __ldg(p0 + ks * 8 + 4 + tq), a3 = __ldg(p1 + ks * 8 + 4 + tq);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[nt][0]), "+f"(d[nt][1]), "+f"(d[nt][2]), "+f"(d[nt][3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(qb[ks][nt][0]), "r"(qb[ks][nt][1]));
    }
    const int row = mt * 16 + g;            // within the warp's 32 positions
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int hd = nt * 8 + tq * 2 + i;
        if (hd < gp) {
          sc[row * gp + hd] = d[nt][i];
          sc[(row + 8) * gp + hd] = d[nt][2 + i];
        }
      }
  }
}

__device__ __forceinline__ float widen1(const float *p) { return *p; }
__device__ __forceinline__ float widen1(const uint16_t *p) {
  return __uint_as_float(static_cast<uint32_t>(*p) << 16);
}

template <int VPL>
__device__ __forceinline__ void vslice(const float *row, int lane, float (&v)[VPL]) {
  if constexpr (VPL == 2) {
    float2 a = __ldg(reinterpret_cast<const float2 *>(row) + lane);
    v[0] = a.x; v[1] = a.y;
  } else {
    float4 a = __ldg(reinterpret_cast<const float4 *>(row) + lane);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
}
template <int VPL>
__device__ __forceinline__ void vslice(const uint16_t *row, int lane, float (&v)[VPL]) {
  if constexpr (VPL == 2) {
    uint32_t a = __ldg(reinterpret_cast<const uint32_t *>(row) + lane);
    v[0] = bf16lo(a); v[1] = bf16hi(a);
  } else {
    uint2 a = __ldg(reinterpret_cast<const uint2 *>(row) + lane);
    v[0] = bf16lo(a.x); v[1] = bf16hi(a.x); v[2] = bf16lo(a.y); v[3] = bf16hi(a.y);
  }
}

template <typename T, int D, int GP, int VPG>
__global__ void __launch_bounds__(kThreads) dense_split_kernel(const StepParams p) {
  constexpr int VPL = D / 32;
  constexpr int HPV = GP / VPG;              // query heads per value head (VPG > 1: GP == G)
  constexpr bool kMma = sizeof(T) == 2;      // bf16: scores on the tensor cores
  constexpr int NT = (GP + 7) / 8;           // 8-head MMA tiles
  __shared__ __align__(16) float qs[kMma ? 4 : D * GP];
  __shared__ __align__(16) float ps[kChunk][GP];
  __shared__ float red[kWarps][GP];
  __shared__ float red_acc[kWarps][4][D];      // four heads at a time
  __shared__ float red_l[kWarps][GP];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x;
  const int b = blockIdx.y / p.h_k, kh = blockIdx.y % p.h_k;
  const int G = p.h_q / p.h_k;
  const int j0 = kh * G;
  const int64_t L = clamp_len(p, b);
  const int64_t t_begin = static_cast<int64_t>(s) * p.split_len;
  if (t_begin >= L) return;
  const int64_t t_end = min(t_begin + p.split_len, L);

  const T *qg = static_cast<const T *>(p.q) + b * p.q_sb;
  uint32_t qb[kMma ? D / 16 : 1][kMma ? NT : 1][2];
  if constexpr (kMma) {
    // B fragments: head n = nt*8 + lane/4, columns ks*16 + (lane%4)*2 (+8)
    const int n_lo = lane >> 2, kq = (lane & 3) * 2;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + n_lo;
        const uint32_t *qr = reinterpret_cast<const uint32_t *>(qg + (j0 + n) * p.q_sh);
        qb[ks][nt][0] = n < G ? __ldg(qr + (ks * 16 + kq) / 2) : 0u;
        qb[ks][nt][1] = n < G ? __ldg(qr + (ks * 16 + kq + 8) / 2) : 0u;
      }
  } else {
    for (int idx = tid; idx < D * GP; idx += kThreads) {
      int i = idx / GP, g = idx % GP;
      qs[idx] = g < G ? widen1(qg + (j0 + g) * p.q_sh + i) : 0.f;
    }
    __syncthreads();
  }

  const T *krow0 = static_cast<const T *>(p.K) + b * p.k_sb + kh * p.k_sh;
  const T *vrow0 = static_cast<const T *>(p.V) + b * p.v_sb + (kh * VPG) * p.v_sh;

  float m_run[GP], l_run[GP], acc[GP][VPL];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m_run[g] = -INFINITY; l_run[g] = 0.f;
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[g][v] = 0.f;
  }

  for (int64_t base = t_begin; base < t_end; base += kChunk) {
    const int64_t t = base + tid;
    const bool valid = t < t_end;
    float A[GP];
    if constexpr (kMma) {
      // scores of this warp's 32 positions into ps (rows of this warp only),
      // then each thread takes its own position's row
      float *sc = &ps[warp * 32][0];
      mma_scores<D, NT>(reinterpret_cast<const uint16_t *>(krow0), base + warp * 32, t_end - 1,
                        qb, sc, GP, lane);
      __syncwarp();
#pragma unroll
      for (int g = 0; g < GP; ++g) A[g] = valid ? sc[lane * GP + g] * p.scale : -INFINITY;
      __syncwarp();
    } else {
      if (valid) {
        dense_scores<T, D, GP>(krow0 + t * D, qs, p.scale, A);
      } else {
#pragma unroll
        for (int g = 0; g < GP; ++g) A[g] = -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float mx = warp_max(A[g]);
      if (lane == 0) red[warp][g] = mx;
    }
    __syncthreads();
    float m_new[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float mc = red[0][g];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) mc = fmaxf(mc, red[w][g]);
      m_new[g] = fmaxf(m_run[g], mc);
      const float corr = exp2f((m_run[g] - m_new[g]) * kLog2e);
      l_run[g] *= corr;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc[g][v] *= corr;
      m_run[g] = m_new[g];
      ps[tid][g] = valid ? exp2f((A[g] - m_new[g]) * kLog2e) : 0.f;
    }
    __syncthreads();
    const int n = static_cast<int>(t_end - base < kChunk ? t_end - base : kChunk);
    for (int kk = warp; kk < n; kk += kWarps) {
      float vv[VPG][VPL];
#pragma unroll
      for (int vs = 0; vs < VPG; ++vs) vslice<VPL>(vrow0 + vs * p.v_sh + (base + kk) * D, lane, vv[vs]);
      const float4 *pv = reinterpret_cast<const float4 *>(&ps[kk][0]);
#pragma unroll
      for (int g4 = 0; g4 < GP / 4; ++g4) {
        const float4 w = pv[g4];
        const float pw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int g = 4 * g4 + u;
          l_run[g] += pw[u];
#pragma unroll
          for (int v = 0; v < VPL; ++v) acc[g][v] = fmaf(pw[u], vv[g / HPV][v], acc[g][v]);
        }
      }
    }
    __syncthreads();
  }

  // Every warp holds the same m_run; sum the warps' l and acc, four heads at a time.
  if (tid == 0) {
#pragma unroll
    for (int g = 0; g < GP; ++g) red[0][g] = m_run[g];
  }
#pragma unroll
  for (int g = 0; g < GP; ++g)
    if (lane == 0) red_l[warp][g] = l_run[g];
#pragma unroll
  for (int g0 = 0; g0 < GP; g0 += 4) {
#pragma unroll
    for (int gg = 0; gg < 4; ++gg)
#pragma unroll
      for (int v = 0; v < VPL; ++v) red_acc[warp][gg][lane * VPL + v] = acc[g0 + gg][v];
    __syncthreads();
    for (int idx = tid; idx < 4 * D; idx += kThreads) {
      const int g = g0 + idx / D, i = idx % D;
      if (g >= G) continue;
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) a += red_acc[w][idx / D][i];
      float *rec = p.partials + (static_cast<int64_t>(b * p.h_q + j0 + g) * p.S + s) * (D + kRecPad);
      rec[kRecPad + i] = a;
      if (i == 0) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) l += red_l[w][g];
        rec[0] = red[0][g];
        rec[1] = l;
        rec[2] = __int_as_float(static_cast<int>(t_end - t_begin));
        rec[3] = 0.f;
      }
    }
    __syncthreads();
  }
}

}  // namespace

template <typename T, int D, int VPG>
static cudaError_t launch_dv(const StepParams &p, int gp, dim3 grid, cudaStream_t st) {
  switch (gp) {
    case 4: dense_split_kernel<T, D, 4, VPG><<<grid, kThreads, 0, st>>>(p); break;
    case 8: dense_split_kernel<T, D, 8, VPG><<<grid, kThreads, 0, st>>>(p); break;
    case 12: dense_split_kernel<T, D, 12, VPG><<<grid, kThreads, 0, st>>>(p); break;
    case 16: dense_split_kernel<T, D, 16, VPG><<<grid, kThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_dd(const StepParams &p, int gp, int vpg, dim3 grid, cudaStream_t st) {
  switch (vpg) {
    case 1: return launch_dv<T, D, 1>(p, gp, grid, st);
    case 2: return launch_dv<T, D, 2>(p, gp, grid, st);
    case 4: return launch_dv<T, D, 4>(p, gp, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D, int VPG>
static const void *kernel_dv(int gp) {
  switch (gp) {
    case 4: return reinterpret_cast<const void *>(dense_split_kernel<T, D, 4, VPG>);
    case 8: return reinterpret_cast<const void *>(dense_split_kernel<T, D, 8, VPG>);
    case 12: return reinterpret_cast<const void *>(dense_split_kernel<T, D, 12, VPG>);
    case 16: return reinterpret_cast<const void *>(dense_split_kernel<T, D, 16, VPG>);
    default: return nullptr;
  }
}

template <typename T, int D>
static const void *kernel_dd(int gp, int vpg) {
  switch (vpg) {
    case 1: return kernel_dv<T, D, 1>(gp);
    case 2: return kernel_dv<T, D, 2>(gp);
    case 4: return kernel_dv<T, D, 4>(gp);
    default: return nullptr;
  }
}

bool dense_supports(int h_q, int h_k, int h_v) {
  if (h_k < 1 || h_v % h_k != 0 || h_q % h_v != 0) return false;
  const int G = h_q / h_k, vpg = h_v / h_k;
  if (vpg == 1) return G <= 16;
  return (vpg == 2 || vpg == 4) && (G == 4 || G == 8 || G == 12 || G == 16) && G % vpg == 0;
}

int dense_ctas_per_sm(int dtype, int d, int h_q, int h_k, int h_v) {
  if (!dense_supports(h_q, h_k, h_v)) return 0;
  const int G = h_q / h_k, vpg = h_v / h_k;
  const int gp = vpg == 1 ? (G + 3) / 4 * 4 : G;
  const void *k = nullptr;
  if (dtype == SAGA_BF16)
    k = d == 64 ? kernel_dd<uint16_t, 64>(gp, vpg) : d == 128 ? kernel_dd<uint16_t, 128>(gp, vpg) : nullptr;
  else
    k = d == 64 ? kernel_dd<float, 64>(gp, vpg) : d == 128 ? kernel_dd<float, 128>(gp, vpg) : nullptr;
  int n = 0;
  if (k == nullptr || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, 0) != cudaSuccess)
    return 0;
  return n;
}

cudaError_t launch_dense_split(const StepParams &p, int dtype, int d, cudaStream_t st) {
  if (!dense_supports(p.h_q, p.h_k, p.h_v)) return cudaErrorInvalidValue;
  const int G = p.h_q / p.h_k, vpg = p.h_v / p.h_k;
  const int gp = vpg == 1 ? (G + 3) / 4 * 4 : G;
  dim3 grid(p.S, p.B * p.h_k);
  if (dtype == SAGA_BF16) {
    if (d == 64) return launch_dd<uint16_t, 64>(p, gp, vpg, grid, st);
    if (d == 128) return launch_dd<uint16_t, 128>(p, gp, vpg, grid, st);
  } else {
    if (d == 64) return launch_dd<float, 64>(p, gp, vpg, grid, st);
    if (d == 128) return launch_dd<float, 128>(p, gp, vpg, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace saga
