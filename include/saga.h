/*
 * saga.h -- C ABI of the SAGA + Atop-N single-token decode attention step
 * on NVIDIA B200 (sm_100a).
 *
 * Source of the operations: "More Value per Key: Asymmetric Sparse Attention
 * for Faster LLM Decoding" (the SAGA paper), as summarised on its pages:
 *   - Attention Mechanism Formalization, Eq. (2-4): A = Q K^T / sqrt(d),
 *     P = softmax(A), O = P V;
 *   - Top-N Attention, Eq. (6): indices of the N largest entries per row;
 *   - Methodology > Atop-N Attention, item 1: entries are kept by comparing
 *     each score with a threshold equal to the N-th largest score; item 2:
 *     the exact threshold is recomputed once every n tokens and reused;
 *     Eq. (7): O = softmax(A[i]) V[i] over the kept entries only;
 *   - SAGA Architecture: h_k key heads decoupled from h_v value heads
 *     (h_k < h_v).
 *
 * One decode step, per sequence b and query head j (0 <= j < h_q):
 *   A[b,j,t] = (q[b,j,:] . K[b, floor(j*h_k/h_q), t, :]) / sqrt(d),  t < l_kv[b]
 *   S[b,j]   = { t : A[b,j,t] >= tau[b,j] }
 *   out[b,j] = sum_{t in S} e^{A[b,j,t]-m} V[b, floor(j*h_v/h_q), t, :]
 *              / sum_{t in S} e^{A[b,j,t]-m},   m = max_{t in S} A[b,j,t]
 *   out[b,j] = 0 when S is empty.
 * A refresh sets tau[b,j] to the exact N-th largest A[b,j,:] (under IEEE
 * totalOrder of the fp32 scores, so it is always one of them), or to -inf
 * when N >= l_kv[b] (every entry kept).
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers, owned by the caller. The
 *     library allocates nothing and keeps no global mutable state; calls
 *     that use distinct workspaces may run concurrently.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream) and returns after enqueueing its kernels. A returned error
 *     means nothing was enqueued, except SAGA_ERR_CUDA, which means a launch
 *     failed.
 *   - Arguments are checked on the host; a violation returns
 *     SAGA_ERR_INVALID_ARG or SAGA_ERR_UNSUPPORTED and enqueues nothing.
 *   - Per-sequence lengths are read on the device. A length outside
 *     [0, min(cap, max_l_kv)] is clamped into that range and sets a bit in
 *     the workspace's device error word (saga_read_device_error); kernels
 *     never trap.
 *   - Scores are computed in fp32 from the stored (fp32 or bf16) values;
 *     every entry point computes a given score with the same arithmetic, so
 *     a dumped score row is exactly the row the selection used.
 */
#ifndef SAGA_H_
#define SAGA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *saga_stream_t;

typedef enum saga_status {
  SAGA_OK = 0,
  SAGA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or shape */
  SAGA_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels handle */
  SAGA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  SAGA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  SAGA_ERR_DEVICE = 5        /* the device error word is non-zero */
} saga_status;

typedef enum saga_dtype {
  SAGA_F32 = 0,   /* q, K, V stored as IEEE binary32 */
  SAGA_BF16 = 1   /* q, K, V stored as bfloat16 */
} saga_dtype;

/* Device error word bits (saga_read_device_error). */
#define SAGA_DEVERR_LKV_NEGATIVE 1   /* some l_kv[b] < 0, treated as 0 */
#define SAGA_DEVERR_LKV_TOO_LONG 2   /* some l_kv[b] > min(cap, max_l_kv), clamped */
#define SAGA_DEVERR_TIMEOUT 4        /* a bounded on-chip wait gave up; outputs invalid */
#define SAGA_DEVERR_BOUNDS 8         /* bounds-checked build only: an index check failed and
                                        the access was skipped; outputs invalid */

/*
 * Problem shape. Layouts (element strides, d contiguous within a row):
 *   q   [B][h_q][d]       element (b,j,i)   at b*q_stride_b + j*q_stride_h + i
 *   K   [B][h_k][cap][d]  element (b,h,t,i) at b*k_stride_b + h*k_stride_h + t*d + i
 *   V   [B][h_v][cap][d]  element (b,h,t,i) at b*v_stride_b + h*v_stride_h + t*d + i
 *   l_kv [B] int32, tau [B][h_q] fp32, out [B][h_q][d] fp32, all contiguous.
 * Requirements: B >= 1; 1 <= h_k <= h_v <= h_q; h_q % h_v == 0;
 * h_v % h_k == 0; h_q / h_k <= 16; d in {64, 128}; dtype a saga_dtype;
 * 0 <= max_l_kv <= cap; every stride > 0 and a multiple of 16 bytes.
 * max_l_kv is the host-side bound on every l_kv[b]; it sizes the work split
 * and the workspace.
 */
typedef struct saga_shape {
  int32_t B, h_q, h_k, h_v, d;
  int32_t dtype;
  int64_t cap;
  int64_t max_l_kv;
  int64_t q_stride_b, q_stride_h;
  int64_t k_stride_b, k_stride_h;
  int64_t v_stride_b, v_stride_h;
} saga_shape;

/* Fill `s` for contiguous q, K and V with the given sizes. */
void saga_shape_contiguous(saga_shape *s, int32_t B, int32_t h_q, int32_t h_k,
                           int32_t h_v, int32_t d, int32_t dtype, int64_t cap,
                           int64_t max_l_kv);

/*
 * Bytes of device workspace that saga_decode_step, saga_refresh_threshold
 * (with this N) and gqa_dense_decode need for `shape`; 0 if the shape is
 * invalid. The workspace must be 256-byte aligned, must be passed to
 * saga_workspace_init once after allocation, and must not be used by two
 * calls that run concurrently. It holds the device error word, per-split
 * partial softmax states, the per-head kept lists of the tensor-core step
 * (a 32-bit mask and 32 fp32 kept scores per 32-position block) and, for
 * refresh, one fp32 score row per (sequence, query head) with the radix
 * select's histograms and bucket lists.
 */
size_t saga_workspace_size(const saga_shape *shape, int32_t N);

/* Zero the error and abort words at the head of a newly allocated workspace
 * (asynchronous on `stream`); nothing else in it needs clearing. */
saga_status saga_workspace_init(void *ws, size_t ws_bytes, saga_stream_t stream);

/*
 * One plain Atop-N step with stored thresholds (Atop-N item 1 and Eq. 7).
 *   q, K, V   inputs as described by `shape`.
 *   l_kv      [B] int32, valid positions per sequence.
 *   tau       [B][h_q] fp32 thresholds, read only.
 *   out       [B][h_q][d] fp32, written.
 *   sel_count nullable [B][h_q] int32: receives |S[b,j]|.
 *   sel_mask  nullable [B][h_q][max_l_kv] uint8: entry t < l_kv[b] receives
 *             1 if t was kept, else 0; entries t >= l_kv[b] are not written.
 */
saga_status saga_decode_step(const saga_shape *shape, const void *q,
                             const void *K, const void *V,
                             const int32_t *l_kv, const float *tau,
                             float *out, int32_t *sel_count,
                             uint8_t *sel_mask, void *ws, size_t ws_bytes,
                             saga_stream_t stream);

/*
 * Refresh step (Atop-N item 2): tau[b][j] = the exact N-th largest score of
 * row (b, j) under IEEE totalOrder, or -inf when N >= l_kv[b]. N >= 1.
 *   V, out    both NULL: only tau is written. Both non-NULL: the same call
 *             then runs this step's selection and PV with the fresh tau,
 *             exactly as saga_decode_step would (out, sel_count, sel_mask as
 *             there). One NULL and the other not: SAGA_ERR_INVALID_ARG.
 *   scores    nullable [B][h_q][max_l_kv] fp32: receives the score rows the
 *             thresholds were selected from (entries t < l_kv[b]).
 */
saga_status saga_refresh_threshold(const saga_shape *shape, const void *q,
                                   const void *K, const void *V,
                                   const int32_t *l_kv, int32_t N,
                                   float *tau, float *out,
                                   int32_t *sel_count, uint8_t *sel_mask,
                                   float *scores, void *ws, size_t ws_bytes,
                                   saga_stream_t stream);

/*
 * Exact top-N attention for this step (Top-N Attention, Eq. 6, then Eq. 7):
 * for every (b, j) the min(N, l_kv[b]) positions with the largest scores are
 * kept, ties broken towards the lower position (the paper fixes no
 * tie-break; scores are ordered by IEEE totalOrder, so -0 < +0), and
 * out[b][j] is the softmax-weighted sum of their value rows. It computes
 * the scores, selects the N-th largest (as a refresh does), finds the last
 * tied position taken, and runs the step with that rule; nothing persists
 * between calls (an R = 1 reference for Atop-N).
 *   Arguments as for saga_refresh_threshold without tau (kept in the
 *   workspace); V and out are required; scores, sel_count and sel_mask are
 *   nullable outputs with the same layouts. sel_count[b][j] is exactly
 *   min(N, l_kv[b]).
 */
saga_status saga_topn_step(const saga_shape *shape, const void *q,
                           const void *K, const void *V, const int32_t *l_kv,
                           int32_t N, float *out, int32_t *sel_count,
                           uint8_t *sel_mask, float *scores, void *ws,
                           size_t ws_bytes, saga_stream_t stream);

/*
 * Full-attention GQA decode (Eq. 2-4 over every t < l_kv[b]): the dense
 * baseline the sparse step is measured against. Requires h_k == h_v and
 * h_q / h_k <= 16 (else SAGA_ERR_INVALID_ARG / SAGA_ERR_UNSUPPORTED).
 */
saga_status gqa_dense_decode(const saga_shape *shape, const void *q,
                             const void *K, const void *V,
                             const int32_t *l_kv, float *out, void *ws,
                             size_t ws_bytes, saga_stream_t stream);

/*
 * Full-attention decode with SAGA's asymmetric heads (SAGA Architecture;
 * Eq. 2-4 over every t < l_kv[b], query head j reading key head
 * floor(j*h_k/h_q) and value head floor(j*h_v/h_q)): the "SAGA, full
 * attention" arm of the paper's ablation of key merging and Atop-N, and,
 * with h_k == h_v, the same result as gqa_dense_decode.
 *   Arguments, layouts, ownership and workspace as for gqa_dense_decode;
 *   out [B][h_q][d] fp32 is written.
 *   Supported: h_v / h_k == 1 with h_q / h_k <= 16, or h_v / h_k in {2, 4}
 *   with h_q / h_k in {4, 8, 12, 16}; other shapes return
 *   SAGA_ERR_UNSUPPORTED and nothing is enqueued.
 */
saga_status saga_dense_decode(const saga_shape *shape, const void *q,
                              const void *K, const void *V,
                              const int32_t *l_kv, float *out, void *ws,
                              size_t ws_bytes, saga_stream_t stream);

/*
 * KV-cache append, the input side of a decode step (Background on
 * autoregressive decoding: each generated token's key and value join the
 * cache before the next attention): for every sequence b, the new key rows
 * k_new[b][0..h_k-1][0..d-1] and value rows v_new[b][0..h_v-1][0..d-1]
 * (contiguous, the cache dtype) are written at position l_kv[b] of every
 * head of K and V, then l_kv[b] grows by one, all on the device and in
 * stream order, so a following step or refresh attends over l_kv[b] + 1
 * positions.
 *   K, V      the caches described by `shape`, written at one position per head.
 *   l_kv      [B] int32, read and incremented on the device.
 *   ws        a workspace (only its error word is used; >= 256 bytes).
 * A sequence whose l_kv[b] is already >= cap (or negative) is left as it is
 * and the workspace's error word receives SAGA_DEVERR_LKV_TOO_LONG (or
 * _NEGATIVE). Steps plan with shape->max_l_kv, so callers that grow the
 * context set max_l_kv to the longest length they will reach.
 */
saga_status saga_append_kv(const saga_shape *shape, const void *k_new,
                           const void *v_new, void *K, void *V, int32_t *l_kv,
                           void *ws, size_t ws_bytes, saga_stream_t stream);

/*
 * saga_decode_step without a workspace argument, for callers that cannot
 * allocate device memory (for example code running inside an allocator's
 * own callbacks, or a runtime that only hands out its preallocated pools and
 * forbids cudaMalloc after start-up). It does exactly what saga_decode_step
 * does with sel_mask = NULL, but keeps its scratch (error word and per-split
 * softmax states) in one fixed array of SAGA_NOALLOC_SCRATCH_BYTES compiled
 * into the library; every GPU that loads the library holds that array until
 * the process exits. The paper has no counterpart to this entry point.
 *   - On the tensor-core path the step needs, each part rounded up to 256
 *     bytes: 256 bytes of error and abort words; 4*B*h_q*SB*(d+4) bytes of
 *     per-split softmax states, SB being the gather splits of a (b, query
 *     head) row the library plans (at most max_l_kv/2048, and no more than
 *     4736/(B*h_q) when that is larger than one); and 132*B*h_q*nblk bytes of
 *     per-head kept lists, nblk = ceil(max_l_kv/32) (a 32-bit mask and 32
 *     fp32 kept scores per 32-position block). A shape needing more than
 *     SAGA_NOALLOC_SCRATCH_BYTES is rejected with SAGA_ERR_WORKSPACE, an
 *     invalid one with SAGA_ERR_INVALID_ARG, and nothing is enqueued then.
 *     (The 16-layer batch-8 128K Llama-3.2-1B workload, h_q = 32, needs
 *     about 140 MB per layer call; batch-1 128K Qwen2.5-1.5B, h_q = 12,
 *     about 6.9 MB.)
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - The first call on each device looks up the array's device address
 *     with that device current; make that first call before any stream
 *     capture on the device.
 *   - All calls on a device share the one array, which keeps the previous
 *     call's contents: calls that can overlap on the GPU (different streams
 *     without ordering) race on it and must be serialised by the caller.
 *   - The device error word lives in that array and cannot be read back;
 *     out-of-range lengths are still clamped exactly as in saga_decode_step.
 *     A step kernel that gives up a bounded wait (the error that
 *     saga_decode_step would report as SAGA_DEVERR_TIMEOUT) cannot report
 *     it here either: instead it poisons its output, every out[b][j][:] of
 *     the call NaN and every sel_count -1, so that the caller sees the
 *     failure in the results.
 */
#define SAGA_NOALLOC_SCRATCH_BYTES (160u << 20)
saga_status saga_decode_step_noalloc(const saga_shape *shape, const void *q,
                                     const void *K, const void *V,
                                     const int32_t *l_kv, const float *tau,
                                     float *out, int32_t *sel_count,
                                     saga_stream_t stream);

/*
 * Write the fp32 score rows A[b][j][t], t < l_kv[b], into
 * scores [B][h_q][max_l_kv], with the same arithmetic as every other entry
 * point. For checking. Uses the workspace's error word only.
 */
saga_status saga_debug_scores(const saga_shape *shape, const void *q,
                              const void *K, const int32_t *l_kv,
                              float *scores, void *ws, size_t ws_bytes,
                              saga_stream_t stream);

/*
 * Synchronise `stream`, copy the device error word to *flags and clear it.
 * Returns SAGA_ERR_DEVICE if it was non-zero, SAGA_OK otherwise.
 */
saga_status saga_read_device_error(void *ws, saga_stream_t stream,
                                   int32_t *flags);

/* Static description of a status code. */
const char *saga_status_string(saga_status status);

/* The last CUDA failure seen by a call of this library on the calling
 * thread, as "<launch or call>: <CUDA error name> (<description>)", or the
 * empty string if there was none. Every call that returns SAGA_ERR_CUDA
 * records it first; a later success does not clear it. The string belongs
 * to the library and stays valid until the thread's next failing call. */
const char *saga_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGA_H_ */
