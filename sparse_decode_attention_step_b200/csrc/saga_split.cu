// SAGA + Atop-N split kernel: one CTA per (sequence b, key head kh, split s
// of the l_kv axis). It scores every position of its split against the
// h_q/h_k query heads that share key head kh (Eq. 2), keeps the entries with
// A >= tau (Atop-N item 1), compacts them per head with warp ballots and a
// prefix sum, and folds the kept V rows into a per-split online-softmax
// state (m, l, acc) for each head (Eq. 7). A separate combine kernel merges
// the split states into `out`.
//
// Modes:
//   kModeDump       scores only: A rows are written to scores_out (refresh
//                   pass one, and the score dump used for checking).
//   kModeStep       scores from K, then select + PV.
//   kModeFromScores scores read back from scores_in (the refresh step's own
//                   rows), then select + PV.
//
// The score of (head g, position t) is always computed by score_row with
// the same operation order, so every mode sees bit-identical scores.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = kThreads;          // positions per sub-chunk, one per thread
constexpr float kLog2e = 1.4426950408889634f;

// acc[g] = sum_i q[g][i] * k[i] as one fp32 FMA chain with i ascending, then
// A[g] = acc[g] * scale. qs is element-major: qs[i * GP + g].
template <typename T, int D, int GP>
__device__ __forceinline__ void score_row(const T *krow, const float *qs,
                                          float scale, float (&A)[GP]) {
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

__device__ __forceinline__ float widen1(const float *p) { return *p; }
__device__ __forceinline__ float widen1(const uint16_t *p) {
  return __uint_as_float(static_cast<uint32_t>(*p) << 16);
}

// VPL consecutive elements of a V row starting at element lane * VPL.
template <int VPL>
__device__ __forceinline__ void load_vslice(const float *row, int lane, float (&v)[VPL]) {
  if constexpr (VPL == 2) {
    float2 a = __ldg(reinterpret_cast<const float2 *>(row) + lane);
    v[0] = a.x; v[1] = a.y;
  } else {
    float4 a = __ldg(reinterpret_cast<const float4 *>(row) + lane);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
}
template <int VPL>
__device__ __forceinline__ void load_vslice(const uint16_t *row, int lane, float (&v)[VPL]) {
  if constexpr (VPL == 2) {
    uint32_t a = __ldg(reinterpret_cast<const uint32_t *>(row) + lane);
    v[0] = bf16lo(a); v[1] = bf16hi(a);
  } else {
    uint2 a = __ldg(reinterpret_cast<const uint2 *>(row) + lane);
    v[0] = bf16lo(a.x); v[1] = bf16hi(a.x); v[2] = bf16lo(a.y); v[3] = bf16hi(a.y);
  }
}

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads)
saga_split_kernel(const StepParams p, const int mode) {
  constexpr int HPW = (GP + kWarps - 1) / kWarps;   // heads owned per warp
  constexpr int VPL = D / 32;                       // acc values per lane

  __shared__ __align__(16) float qs[D * GP];
  __shared__ float tau_s[GP];
  __shared__ int32_t tie_s[GP];
  __shared__ int sel_t[GP][kChunk];
  __shared__ float sel_a[GP][kChunk];
  __shared__ int warp_off[kWarps][GP];
  __shared__ int head_cnt[GP];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x;
  const int b = blockIdx.y / p.h_k, kh = blockIdx.y % p.h_k;
  const int G = p.h_q / p.h_k;
  const int j0 = kh * G;
  const int64_t L = clamp_len(p, b);
  const int64_t t_begin = static_cast<int64_t>(s) * p.split_len;
  if (t_begin >= L) return;                         // nothing here; combine skips it
  const int64_t t_end = min(t_begin + p.split_len, L);

  const T *qg = static_cast<const T *>(p.q) + b * p.q_sb;
  for (int idx = tid; idx < D * GP; idx += kThreads) {
    int i = idx / GP, g = idx % GP;
    qs[idx] = g < G ? widen1(qg + (j0 + g) * p.q_sh + i) : 0.f;
  }
  if (tid < GP) {
    tau_s[tid] = (tid < G && mode != kModeDump) ? p.tau[b * p.h_q + j0 + tid] : 0.f;
    tie_s[tid] = (tid < G && p.tie != nullptr) ? p.tie[b * p.h_q + j0 + tid] : -1;
  }
  __syncthreads();

  const T *krow0 = static_cast<const T *>(p.K) + b * p.k_sb + kh * p.k_sh;
  const int64_t row0 = static_cast<int64_t>(b * p.h_q + j0) * p.row_stride;

  float m_run[HPW], l_run[HPW], acc[HPW][VPL];
  int cnt_run[HPW];
#pragma unroll
  for (int r = 0; r < HPW; ++r) {
    m_run[r] = -INFINITY; l_run[r] = 0.f; cnt_run[r] = 0;
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[r][v] = 0.f;
  }

  for (int64_t base = t_begin; base < t_end; base += kChunk) {
    const int64_t t = base + tid;
    const bool valid = t < t_end;
    float A[GP];
    if (mode == kModeFromScores) {
#pragma unroll
      for (int g = 0; g < GP; ++g)
        A[g] = (valid && g < G) ? p.scores_in[row0 + g * p.row_stride + t] : -INFINITY;
    } else if (valid) {
      score_row<T, D, GP>(krow0 + t * D, qs, p.scale, A);
    } else {
#pragma unroll
      for (int g = 0; g < GP; ++g) A[g] = -INFINITY;
    }

    if (mode == kModeDump) {
      if (valid) {
#pragma unroll
        for (int g = 0; g < GP; ++g)
          if (g < G) p.scores_out[row0 + g * p.row_stride + t] = A[g];
      }
      continue;
    }

    // Threshold compare and order-preserving compaction, per head.
    uint32_t selbits = 0;
    int pos[GP];
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      bool sel;
      if (p.tie != nullptr) {
        // exact top-N: totalOrder above tau, or equal up to the tie position
        const uint32_t kx = order_key(A[g]), kt = order_key(tau_s[g]);
        sel = valid && g < G && (kx > kt || (kx == kt && t <= tie_s[g]));
      } else {
        sel = valid && g < G && A[g] >= tau_s[g];
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) warp_off[warp][g] = __popc(bal);
      pos[g] = __popc(bal & lt_mask);
      selbits |= static_cast<uint32_t>(sel) << g;
    }
    if (p.sel_mask != nullptr && valid) {
      for (int g = 0; g < G; ++g)
        p.sel_mask[row0 + g * p.row_stride + t] = static_cast<uint8_t>((selbits >> g) & 1u);
    }
    __syncthreads();
    if (tid < GP) {
      int run = 0;
      for (int w = 0; w < kWarps; ++w) {
        int c = warp_off[w][tid];
        warp_off[w][tid] = run;
        run += c;
      }
      head_cnt[tid] = run;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if ((selbits >> g) & 1u) {
        const int o = warp_off[warp][g] + pos[g];
        sel_t[g][o] = static_cast<int>(t - base);
        sel_a[g][o] = A[g];
      }
    }
    __syncthreads();

    // Sparse softmax + V-row gather for the heads this warp owns.
#pragma unroll
    for (int r = 0; r < HPW; ++r) {
      const int g = warp + r * kWarps;
      if (g >= G) continue;
      const int n = head_cnt[g];
      if (n == 0) continue;
      float mc = -INFINITY;
      for (int e = lane; e < n; e += 32) mc = fmaxf(mc, sel_a[g][e]);
      mc = warp_max(mc);
      const float m_new = fmaxf(m_run[r], mc);
      const float corr = exp2f((m_run[r] - m_new) * kLog2e);   // 0 when m_run = -inf
      l_run[r] *= corr;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc[r][v] *= corr;
      const int vh = ((j0 + g) * p.h_v) / p.h_q;
      const T *vbase = static_cast<const T *>(p.V) + b * p.v_sb + vh * p.v_sh;
      int e = 0;
      for (; e + 4 <= n; e += 4) {
        float vv[4][VPL], pw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          load_vslice<VPL>(vbase + (base + sel_t[g][e + u]) * D, lane, vv[u]);
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
        load_vslice<VPL>(vbase + (base + sel_t[g][e]) * D, lane, vv);
        const float pw = exp2f((sel_a[g][e] - m_new) * kLog2e);
        l_run[r] += pw;
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc[r][v] = fmaf(pw, vv[v], acc[r][v]);
      }
      m_run[r] = m_new;
      cnt_run[r] += n;
    }
    __syncthreads();
  }

  if (mode == kModeDump) return;
#pragma unroll
  for (int r = 0; r < HPW; ++r) {
    const int g = warp + r * kWarps;
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

}  // namespace

template <typename T, int D>
static cudaError_t launch_d(const StepParams &p, int mode, int gp, dim3 grid, cudaStream_t st) {
  switch (gp) {
    case 4: saga_split_kernel<T, D, 4><<<grid, kThreads, 0, st>>>(p, mode); break;
    case 8: saga_split_kernel<T, D, 8><<<grid, kThreads, 0, st>>>(p, mode); break;
    case 12: saga_split_kernel<T, D, 12><<<grid, kThreads, 0, st>>>(p, mode); break;
    case 16: saga_split_kernel<T, D, 16><<<grid, kThreads, 0, st>>>(p, mode); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_saga_split(const StepParams &p, int mode, int dtype, int d, int gp,
                              cudaStream_t st) {
  dim3 grid(p.S, p.B * p.h_k);
  if (dtype == SAGA_BF16) {
    if (d == 64) return launch_d<uint16_t, 64>(p, mode, gp, grid, st);
    if (d == 128) return launch_d<uint16_t, 128>(p, mode, gp, grid, st);
  } else {
    if (d == 64) return launch_d<float, 64>(p, mode, gp, grid, st);
    if (d == 128) return launch_d<float, 128>(p, mode, gp, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace saga
