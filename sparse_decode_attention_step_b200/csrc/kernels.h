// Launchers of the SAGA kernels (host side, internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "common.cuh"

namespace saga {

// kModeStepTies: a step that keeps A > tau, and A == tau only at positions
// t <= tie[b][j] (exact top-N with ties broken towards the lower position).
enum { kModeDump = 0, kModeStep = 1, kModeFromScores = 2, kModeStepTies = 3 };

// Split kernel over grid (S, B * h_k); gp = h_q / h_k rounded up to 4.
cudaError_t launch_saga_split(const StepParams &p, int mode, int dtype, int d, int gp,
                              cudaStream_t st);

// Persistent tensor-core split kernel: dump and step modes, bit-identical
// scores between the two; the step modes read stored score rows instead of K
// when p.scores_in is set. Shapes it takes: saga_tc_supports.
cudaError_t launch_saga_tc(const StepParams &p, int mode, int d, cudaStream_t st);

// bf16 caches, d in {64, 128}, G = h_q / h_k <= 16 (one MMA's N), h_q a
// multiple of h_v and h_v of h_k.
bool saga_tc_supports(int dtype, int d, int h_q, int h_k, int h_v);

// The V-row half of a tensor-core step: per-split records from the scan's
// kept lists (gather.cu).
cudaError_t launch_gather(const GatherParams &p, int d, cudaStream_t st);

// The tensor-core step kernel can stream stored score rows (StepParams::
// scores_in, [B][h_q][row_stride] fp32) in place of K: 16-byte aligned rows
// whose stride is a multiple of four floats.
bool saga_tc_scores_streamable(const float *rows, int64_t row_stride);

// Merge the per-split states of every (b, j) into out and sel_count; when
// abort_word is given, clear it afterwards (the step that set it is over).
cudaError_t launch_combine(const float *partials, const int32_t *l_kv, int32_t *abort_word,
                           float *out, int32_t *sel_count, int B, int h_q, int d, int S,
                           int64_t split_len, int64_t cap, int64_t max_l_kv,
                           cudaStream_t st);

// tau[b][j] = N-th largest of the stored score row (b, j), or -inf if N >= l_kv[b].
// hist0: nullable [B][h_q][256] top-byte histograms of the rows' order keys
// (from the score pass); without it the kernel makes one more pass.
// tie: nullable [B][h_q]; receives the position of the last entry equal to
// tau that the N largest take when ties go to the lower position (one more
// pass over the row), or INT32_MAX when N >= l_kv[b].
// gcand [B][h_q][gcap] (gcap a multiple of 4), gcount [B][h_q] and hist1
// [B][h_q][256] (both zeroed before the call): with hist0, a collect kernel
// first lists each row's digit-0 bucket in gcand and counts the bucket's
// digit 1 in hist1 (about two CTAs per SM across the rows), and the select
// resolves the other digits from those.
cudaError_t launch_radix_select(const float *scores, int64_t row_stride, const int32_t *l_kv,
                                int N, float *tau, int B, int h_q, int64_t cap, int64_t max_l_kv,
                                const uint32_t *hist0, int32_t *tie, uint32_t *gcand,
                                uint32_t *gcount, uint32_t *hist1, int gcap, int sms,
                                cudaStream_t st);

// Dense (full-attention) split kernel over grid (S, B * h_k): GQA (h_k == h_v,
// h_q / h_k <= 16) or SAGA heads (h_v / h_k in {2, 4}, h_q / h_k in {4, 8, 12, 16}).
bool dense_supports(int h_q, int h_k, int h_v);
cudaError_t launch_dense_split(const StepParams &p, int dtype, int d, cudaStream_t st);
// CTAs of the shape's dense kernel that fit one SM (0 if unknown).
int dense_ctas_per_sm(int dtype, int d, int h_q, int h_k, int h_v);

// KV-cache append over grid (B): rows k_new [B][h_k][d] and v_new [B][h_v][d]
// (contiguous) to position l_kv[b], then l_kv[b] += 1. Strides in elements.
cudaError_t launch_append(const void *k_new, const void *v_new, void *K, void *V, int32_t *l_kv,
                          int32_t *err, int B, int h_k, int h_v, int d, int esz, int64_t k_sb,
                          int64_t k_sh, int64_t v_sb, int64_t v_sh, int64_t cap,
                          cudaStream_t st);

// Record a failed CUDA call for saga_last_error (per calling thread) and
// return SAGA_ERR_CUDA; `where` names the launch or call that failed.
saga_status cuda_fail(cudaError_t e, const char *where);
// SAGA_OK for cudaSuccess, else cuda_fail(e, where).
inline saga_status cuda_check(cudaError_t e, const char *where) {
  return e == cudaSuccess ? SAGA_OK : cuda_fail(e, where);
}

// Plain step with a caller-chosen scratch buffer (see saga_decode_step_noalloc).
size_t plain_step_scratch_bytes(const saga_shape &s);
saga_status plain_step_with_scratch(const saga_shape *shape, const void *q, const void *K,
                                    const void *V, const int32_t *l_kv, const float *tau,
                                    float *out, int32_t *sel_count, void *scratch,
                                    size_t scratch_bytes, cudaStream_t st);

}  // namespace saga

namespace saga {

// Launch `kernel` on `st` with programmatic stream serialisation, so its
// blocks may start (and run up to pdl_wait) while the previous kernel in the
// stream finishes. Every kernel launched this way calls pdl_wait before it
// reads or writes memory that an earlier launch in the stream may touch.
// On the legacy default stream, which synchronises with every other stream,
// the launch is an ordinary one (pdl_wait then returns at once).
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, A &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (st == nullptr || st == cudaStreamLegacy) ? 0 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

}  // namespace saga
