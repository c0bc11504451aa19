// Dense decode split kernels: full attention, Eq. (2-4) over every position,
// for GQA (h_k == h_v) and for SAGA's asymmetric heads (h_k < h_v: the G query
// heads of a key head read VPG value heads, G / VPG query heads each). One CTA
// per (b, key head, split of l_kv); the per-split states go to the same
// combine kernel as the sparse step.
//
// fp32 caches: each sub-chunk of 256 positions is scored (one position per
// thread, all G query heads of the group, fp32 FMA), the chunk maximum
// updates the running softmax state, and the probabilities weight the V rows
// (the VPG rows of one position per warp-iteration, d split across the
// lanes). bf16 caches: the staged kernel below.
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

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
template <int D, int GP, int VPG>
__global__ void __launch_bounds__(kThreads) dense_split_kernel(const StepParams p) {
  using T = float;
  constexpr int VPL = D / 32;
  constexpr int HPV = GP / VPG;              // query heads per value head (VPG > 1: GP == G)
  __shared__ __align__(16) float qs[D * GP];
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
  for (int idx = tid; idx < D * GP; idx += kThreads) {
    int i = idx / GP, g = idx % GP;
    qs[idx] = g < G ? qg[(j0 + g) * p.q_sh + i] : 0.f;
  }
  __syncthreads();

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
    if (valid) {
      dense_scores<T, D, GP>(krow0 + t * D, qs, p.scale, A);
    } else {
#pragma unroll
      for (int g = 0; g < GP; ++g) A[g] = -INFINITY;
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


// bf16 caches: the positions of a split are taken in chunks of kSC, whose K
// rows (padded to D + 8 elements, so the MMA fragment loads hit distinct
// banks) and VPG V rows are copied into shared memory by cp.async while the
// previous chunk is worked on (two stages), so each SM keeps a whole chunk
// of every resident CTA in flight. Per chunk: each warp scores 16 positions
// against the group's heads on the tensor cores (mma.sync m16n8k16); each
// head's chunk maximum and exponentials update its running softmax state
// (one warp per head, fixed reduction order); then every thread adds the
// probabilities times V for its items (up to four heads that read one value
// head, 8 dimensions) over its share of the chunk's rows: one 16-byte V
// load, converted once, per position and item.
template <int D, int GP, int VPG>
struct DS {
  static constexpr int kKRow = D + 8;                       // bf16 elements per staged K row
  static constexpr int stage_for(int sc) { return sc * kKRow * 2 + VPG * sc * D * 2; }
  static constexpr int kSC = 2 * stage_for(128) + 128 * GP * 4 <= 210 * 1024 ? 128 : 64;
  static constexpr int kKBytes = kSC * kKRow * 2;
  static constexpr int kStage = stage_for(kSC);
  static constexpr int kPsBytes = kSC * GP * 4;              // the chunk's probabilities
  static constexpr int kSmem = 2 * kStage + kPsBytes;
  static constexpr int HPV = GP / VPG;                      // query heads per value head
  // heads of one item: the largest of 4, 2, 1 that divides the heads of a value head
  static constexpr int HI = HPV % 4 == 0 ? 4 : (HPV % 2 == 0 ? 2 : 1);
  static constexpr int NP = GP / HI * (D / 8);              // (HI heads, 8 dimensions) items
  static constexpr int RS = NP >= kThreads ? 1 : kThreads / NP;   // row splits of a chunk
  static constexpr int IPT = (NP * RS + kThreads - 1) / kThreads; // items per thread
  static_assert(GP % HI == 0 && HPV % HI == 0, "an item's heads read one value head");
  static_assert(kStage % 16 == 0 && kKBytes % 16 == 0, "16-byte staging");
  static_assert(RS * GP * D * 4 <= 2 * kStage, "the row splits' sums fit the staging area");
};

template <int D, int GP, int VPG>
__global__ void __launch_bounds__(kThreads, 3) dense_stream_kernel(const StepParams p) {
  using C = DS<D, GP, VPG>;
  constexpr int kSC = C::kSC, NT = (GP + 7) / 8, HPV = C::HPV;
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float s_m[GP], s_l[GP], s_corr[GP];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x;
  const int b = blockIdx.y / p.h_k, kh = blockIdx.y % p.h_k;
  const int G = p.h_q / p.h_k;
  const int j0 = kh * G;
  const int64_t L = clamp_len(p, b);
  const int64_t t_begin = static_cast<int64_t>(s) * p.split_len;
  if (t_begin >= L) return;
  const int64_t t_end = min(t_begin + p.split_len, L);

  // B fragments of the group's queries: head n = nt*8 + lane/4, columns
  // ks*16 + (lane%4)*2 (+8); heads past G are zero
  const uint16_t *qg = static_cast<const uint16_t *>(p.q) + b * p.q_sb;
  uint32_t qb[D / 16][NT][2];
  {
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
  }
  const uint16_t *krow0 = static_cast<const uint16_t *>(p.K) + b * p.k_sb + kh * p.k_sh;
  const uint16_t *vrow0 = static_cast<const uint16_t *>(p.V) + b * p.v_sb + (kh * VPG) * p.v_sh;
  auto kst = [&](int st) { return reinterpret_cast<uint16_t *>(dsm + st * C::kStage); };
  auto vst = [&](int st) { return reinterpret_cast<uint16_t *>(dsm + st * C::kStage + C::kKBytes); };
  float *ps = reinterpret_cast<float *>(dsm + 2 * C::kStage);    // [kSC][GP]

  // stage the chunk at `base`; rows past t_end re-read row t_end - 1 (their
  // probabilities are zero)
  auto load = [&](int st, int64_t base) {
    constexpr int KP = D / 8;                                     // 16-byte pieces per row
    uint16_t *ks = kst(st), *vs = vst(st);
    for (int i = tid; i < kSC * KP; i += kThreads) {
      const int r = i / KP, c8 = i % KP;
      const int64_t t = min(base + r, t_end - 1);
      sm100::cp_async16(ks + r * C::kKRow + c8 * 8, krow0 + t * D + c8 * 8);
    }
    for (int i = tid; i < VPG * kSC * KP; i += kThreads) {
      const int vh = i / (kSC * KP), rem = i % (kSC * KP), r = rem / KP, c8 = rem % KP;
      const int64_t t = min(base + r, t_end - 1);
      sm100::cp_async16(vs + (vh * kSC + r) * D + c8 * 8, vrow0 + vh * p.v_sh + t * D + c8 * 8);
    }
    sm100::cp_async_commit();
  };

  if (tid < GP) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
  constexpr int HI = C::HI;
  float acc[C::IPT][HI][8];
#pragma unroll
  for (int it = 0; it < C::IPT; ++it)
#pragma unroll
    for (int u = 0; u < HI; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[it][u][e] = 0.f;

  const int nchunks = static_cast<int>((t_end - t_begin + kSC - 1) / kSC);
  load(0, t_begin);
  for (int c = 0; c < nchunks; ++c) {
    const int st = c & 1;
    const int64_t base = t_begin + static_cast<int64_t>(c) * kSC;
    if (c + 1 < nchunks) {
      load(st ^ 1, base + kSC);
      sm100::cp_async_wait_prior();
    } else {
      sm100::cp_async_wait_all();
    }
    __syncthreads();                                  // chunk c is staged

    // ---- scores of this warp's 16 rows, scaled, into ps ----------------------
    if (warp * 16 < kSC) {
      const int g = lane >> 2, tq = lane & 3;
      const uint16_t *k0 = kst(st) + (warp * 16 + g) * C::kKRow;
      const uint16_t *k1 = k0 + 8 * C::kKRow;
      float d[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t a0 = *reinterpret_cast<const uint32_t *>(k0 + ks * 16 + tq * 2);
        const uint32_t a1 = *reinterpret_cast<const uint32_t *>(k1 + ks * 16 + tq * 2);
        const uint32_t a2 = *reinterpret_cast<const uint32_t *>(k0 + ks * 16 + 8 + tq * 2);
        const uint32_t a3 = *reinterpret_cast<const uint32_t *>(k1 + ks * 16 + 8 + tq * 2);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
              "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
              : "+f"(d[nt][0]), "+f"(d[nt][1]), "+f"(d[nt][2]), "+f"(d[nt][3])
              : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(qb[ks][nt][0]), "r"(qb[ks][nt][1]));
      }
      const int r0 = warp * 16 + g, r1 = r0 + 8;
      const bool v0 = base + r0 < t_end, v1 = base + r1 < t_end;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int hd = nt * 8 + tq * 2 + i;
          if (hd < GP) {
            ps[r0 * GP + hd] = v0 ? d[nt][i] * p.scale : -INFINITY;
            ps[r1 * GP + hd] = v1 ? d[nt][2 + i] * p.scale : -INFINITY;
          }
        }
    }
    __syncthreads();

    // ---- per head: chunk maximum, exponentials, running state ---------------
    for (int h = warp; h < GP; h += kWarps) {
      float mx = -INFINITY;
      for (int r = lane; r < kSC; r += 32) mx = fmaxf(mx, ps[r * GP + h]);
      mx = warp_max(mx);
      const float m_old = s_m[h];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int r = lane; r < kSC; r += 32) {
        const float x = ps[r * GP + h];
        const float e = x == -INFINITY ? 0.f : exp2f((x - m_new) * kLog2e);
        ps[r * GP + h] = e;
        sum += e;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        const float corr = m_old == -INFINITY ? 0.f : exp2f((m_old - m_new) * kLog2e);
        s_l[h] = fmaf(s_l[h], corr, sum);
        s_m[h] = m_new;
        s_corr[h] = corr;
      }
    }
    __syncthreads();

    // ---- probabilities x V ------------------------------------------------------
    const uint16_t *vs = vst(st);
#pragma unroll
    for (int it = 0; it < C::IPT; ++it) {
      const int q = tid + it * kThreads;
      if (q < C::NP * C::RS) {
        const int rs = q / C::NP, item = q % C::NP;
        const int g0 = item / (D / 8) * HI, d8 = item % (D / 8);
#pragma unroll
        for (int u = 0; u < HI; ++u) {
          const float corr = s_corr[g0 + u];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[it][u][e] *= corr;
        }
        const uint16_t *vc = vs + (g0 / HPV) * kSC * D + 8 * d8;
        constexpr int kRows = kSC / C::RS;
#pragma unroll 2
        for (int r = rs * kRows; r < (rs + 1) * kRows; ++r) {
          const uint4 w = *reinterpret_cast<const uint4 *>(vc + r * D);
          const float vf[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                               bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
          float pr[HI];
          if constexpr (HI == 4) {
            const float4 p4 = *reinterpret_cast<const float4 *>(ps + r * GP + g0);
            pr[0] = p4.x; pr[1] = p4.y; pr[2] = p4.z; pr[3] = p4.w;
          } else {
#pragma unroll
            for (int u = 0; u < HI; ++u) pr[u] = ps[r * GP + g0 + u];
          }
#pragma unroll
          for (int u = 0; u < HI; ++u)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[it][u][e] = fmaf(pr[u], vf[e], acc[it][u][e]);
        }
      }
    }
    __syncthreads();                                  // stage st and ps are free again
  }

  // ---- the heads' records: row splits added in order ------------------------
  float *red = reinterpret_cast<float *>(dsm);        // [RS][GP][D], over the idle stages
#pragma unroll
  for (int it = 0; it < C::IPT; ++it) {
    const int q = tid + it * kThreads;
    if (q < C::NP * C::RS) {
      const int rs = q / C::NP, item = q % C::NP;
      const int g0 = item / (D / 8) * HI, d8 = item % (D / 8);
#pragma unroll
      for (int u = 0; u < HI; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[(rs * GP + g0 + u) * D + 8 * d8 + e] = acc[it][u][e];
    }
  }
  __syncthreads();
  for (int q = tid; q < GP * D; q += kThreads) {
    const int g = q / D, e = q % D;
    if (g >= G) continue;
    float a = 0.f;
#pragma unroll
    for (int rs = 0; rs < C::RS; ++rs) a += red[(rs * GP + g) * D + e];
    float *rec = p.partials + (static_cast<int64_t>(b * p.h_q + j0 + g) * p.S + s) * (D + kRecPad);
    rec[kRecPad + e] = a;
    if (e == 0) {
      rec[0] = s_m[g];
      rec[1] = s_l[g];
      rec[2] = __int_as_float(static_cast<int>(t_end - t_begin));
      rec[3] = 0.f;
    }
  }
}

}  // namespace

constexpr int kMaxDevices = 64;

template <int D, int GP, int VPG>
static cudaError_t launch_stream(const StepParams &p, dim3 grid, cudaStream_t st) {
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(dense_stream_kernel<D, GP, VPG>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DS<D, GP, VPG>::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  dense_stream_kernel<D, GP, VPG><<<grid, kThreads, DS<D, GP, VPG>::kSmem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int VPG>
static cudaError_t launch_dv(const StepParams &p, int gp, dim3 grid, cudaStream_t st) {
  if constexpr (sizeof(T) == 2) {
    switch (gp) {
      case 4: return launch_stream<D, 4, VPG>(p, grid, st);
      case 8: return launch_stream<D, 8, VPG>(p, grid, st);
      case 12: return launch_stream<D, 12, VPG>(p, grid, st);
      case 16: return launch_stream<D, 16, VPG>(p, grid, st);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (gp) {
      case 4: dense_split_kernel<D, 4, VPG><<<grid, kThreads, 0, st>>>(p); break;
      case 8: dense_split_kernel<D, 8, VPG><<<grid, kThreads, 0, st>>>(p); break;
      case 12: dense_split_kernel<D, 12, VPG><<<grid, kThreads, 0, st>>>(p); break;
      case 16: dense_split_kernel<D, 16, VPG><<<grid, kThreads, 0, st>>>(p); break;
      default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
  }
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

template <int D, int VPG>
static const void *kernel_dv(int gp) {
  switch (gp) {
    case 4: return reinterpret_cast<const void *>(dense_split_kernel<D, 4, VPG>);
    case 8: return reinterpret_cast<const void *>(dense_split_kernel<D, 8, VPG>);
    case 12: return reinterpret_cast<const void *>(dense_split_kernel<D, 12, VPG>);
    case 16: return reinterpret_cast<const void *>(dense_split_kernel<D, 16, VPG>);
    default: return nullptr;
  }
}

template <int D>
static const void *kernel_dd(int gp, int vpg) {
  switch (vpg) {
    case 1: return kernel_dv<D, 1>(gp);
    case 2: return kernel_dv<D, 2>(gp);
    case 4: return kernel_dv<D, 4>(gp);
    default: return nullptr;
  }
}

bool dense_supports(int h_q, int h_k, int h_v) {
  if (h_k < 1 || h_v % h_k != 0 || h_q % h_v != 0) return false;
  const int G = h_q / h_k, vpg = h_v / h_k;
  if (vpg == 1) return G <= 16;
  return (vpg == 2 || vpg == 4) && (G == 4 || G == 8 || G == 12 || G == 16) && G % vpg == 0;
}

template <int D, int VPG>
static int stream_smem(int gp) {
  switch (gp) {
    case 4: return DS<D, 4, VPG>::kSmem;
    case 8: return DS<D, 8, VPG>::kSmem;
    case 12: return DS<D, 12, VPG>::kSmem;
    case 16: return DS<D, 16, VPG>::kSmem;
    default: return -1;
  }
}

// The staged bf16 kernel's resident CTAs per SM, from its shared memory
// (its 256 threads and registers allow more).
static int stream_ctas_per_sm(int d, int gp, int vpg) {
  int smem = -1;
  if (d == 64) smem = vpg == 1 ? stream_smem<64, 1>(gp) : vpg == 2 ? stream_smem<64, 2>(gp) : stream_smem<64, 4>(gp);
  if (d == 128) smem = vpg == 1 ? stream_smem<128, 1>(gp) : vpg == 2 ? stream_smem<128, 2>(gp) : stream_smem<128, 4>(gp);
  if (smem <= 0) return 0;
  const int per_sm = 227 * 1024 / (smem + 1024);
  return per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
}

int dense_ctas_per_sm(int dtype, int d, int h_q, int h_k, int h_v) {
  if (!dense_supports(h_q, h_k, h_v)) return 0;
  const int G = h_q / h_k, vpg = h_v / h_k;
  const int gp = vpg == 1 ? (G + 3) / 4 * 4 : G;
  if (dtype == SAGA_BF16) return stream_ctas_per_sm(d, gp, vpg);
  const void *k = d == 64 ? kernel_dd<64>(gp, vpg) : d == 128 ? kernel_dd<128>(gp, vpg) : nullptr;
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
