// Device helpers shared by the SAGA kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "saga.h"

namespace saga {

constexpr int kMaxGroup = 16;       // h_q / h_k handled by the score kernels
constexpr int kRecPad = 4;          // partial record = {m, l, count, pad, acc[d]}

// Kernel parameter block shared by the split kernels. Strides in elements.
struct StepParams {
  const void *q;
  const void *K;
  const void *V;
  const int32_t *l_kv;
  const float *tau;
  const int32_t *tie;       // nullable [B][h_q]: exact top-N, keep A == tau only at t <= tie
  const float *scores_in;   // from-scores mode: [B][h_q][row_stride]
  float *scores_out;        // dump mode: [B][h_q][row_stride]
  float *partials;          // [B][h_q][S][d + kRecPad]
  uint8_t *sel_mask;        // nullable [B][h_q][row_stride]
  uint32_t *hist;           // nullable [B][h_q][256]: dump mode adds the top-byte histogram
                            // of each score row's order keys
  uint32_t *lmask;          // step modes (tensor-core scan): [B * h_q][nblk] kept-position
                            // mask of every 32-position block of each query head's row
  float *lscore;            // [B * h_q][nblk * 32] kept scores, at each key's rank in its block
  int64_t nblk;             // 32-position blocks per row (lists)
  int32_t *err;             // device error word
  int32_t *abort;           // the step's abort word: set when a bounded wait gives up
  int64_t q_sb, q_sh, k_sb, k_sh, v_sb, v_sh;
  int64_t cap, max_l_kv, row_stride;
  int64_t split_len;
  int32_t B, h_q, h_k, h_v, S;
  float scale;              // 1 / sqrt(d)
};

// Index checks of the bounds-checked build (-DSAGA_CHECK): a failed check
// sets SAGA_DEVERR_BOUNDS in the error word and the caller skips the access.
// In the ordinary build every check is true at compile time.
__device__ __forceinline__ bool saga_in_bounds(bool ok, int32_t *err) {
#ifdef SAGA_CHECK
  if (!ok && err != nullptr) atomicOr(err, SAGA_DEVERR_BOUNDS);
  return ok;
#else
  (void)ok;
  (void)err;
  return true;
#endif
}

// Clamp a device-side sequence length into [0, min(cap, max_l_kv)] and
// record any violation in the error word.
// Gather kernel parameters: the kept lists of a tensor-core scan, the V
// cache and the per-split records to write (strides in elements).
struct GatherParams {
  const uint16_t *V;
  int64_t v_sb, v_sh;
  const int32_t *l_kv;
  int64_t cap, max_l_kv;
  const uint32_t *lmask;    // [B * h_q][nblk]
  const float *lscore;      // [B * h_q][nblk * 32]
  int64_t nblk;
  float *partials;          // [B][h_q][SB][d + kRecPad]
  const int32_t *abort;     // the scan's abort word
  int32_t *err;             // device error word (index checks of the checked build)
  int32_t B, h_q, SB;
  int32_t hpv;              // h_q / h_v: query heads per value head
  int64_t blk_per_split;    // 32-position blocks per split
};

__device__ __forceinline__ int64_t clamp_len(const StepParams &p, int b) {
  int64_t L = p.l_kv[b];
  int64_t hi = p.cap < p.max_l_kv ? p.cap : p.max_l_kv;
  if (L < 0) {
    atomicOr(p.err, SAGA_DEVERR_LKV_NEGATIVE);
    L = 0;
  } else if (L > hi) {
    atomicOr(p.err, SAGA_DEVERR_LKV_TOO_LONG);
    L = hi;
  }
  return L;
}

// Eight consecutive stored elements widened to fp32.
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4 *>(p));
  float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void load8(const uint16_t *p, float (&x)[8]) {
  uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
  x[0] = bf16lo(a.x); x[1] = bf16hi(a.x);
  x[2] = bf16lo(a.y); x[3] = bf16hi(a.y);
  x[4] = bf16lo(a.z); x[5] = bf16hi(a.z);
  x[6] = bf16lo(a.w); x[7] = bf16hi(a.w);
}

// Order-preserving uint32 key of an fp32 value (IEEE totalOrder, non-NaN):
// larger float <-> larger key, -0 < +0.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_order_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace saga

namespace saga {

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel in the stream is still
// running; pdl_wait blocks until that kernel has completed and its memory
// is visible, so nothing the previous kernel writes is read before it.
// pdl_trigger lets the next kernel in the stream begin its own launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace saga
