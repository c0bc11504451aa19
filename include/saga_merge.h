/*
 * saga_merge.h -- C ABI of the closed-form GQA-to-SAGA key-head merge on
 * NVIDIA B200 (sm_100a).
 *
 * Source of the operation: "More Value per Key: Asymmetric Sparse Attention
 * for Faster LLM Decoding" (the SAGA paper), as summarised on its pages,
 * GQA-to-SAGA Conversion, Stage 1: Closed-Form Initialization:
 *   - Eq. (13): merging teacher key heads a and b into one key projection M
 *     costs L_{a,b}(M) = sum over the query heads j of a of
 *     ||Q^j (X M)^T - Q^j (X W_K^a)^T||_F^2, plus the same sum over the query
 *     heads of b against W_K^b;
 *   - Eq. (15), Lemma 4.1: the minimising M is
 *     (W_K^a S_a + W_K^b S_b)(S_a + S_b)^+, S_r = sum_{j of r} Q^j^T Q^j,
 *     + the Moore-Penrose pseudoinverse;
 *   - Eq. (14), Theorem 4.2: the pairing of the teacher's key heads is a
 *     minimum-weight perfect matching of the complete graph whose edge (a, b)
 *     weighs w(a, b) = L_{a,b} at the Eq. (15) optimum.
 *
 * What one call computes, from calibration hidden states X, the teacher's key
 * projection and calibration queries:
 *   w[a][b]   = L_{a,b}(Eq. 15 optimum) for every a != b (w[a][a] = 0);
 *   pairs     = the minimum-weight perfect matching, h_k / 2 pairs (a, b) with
 *               a < b, sorted by a; merged key head i comes from pairs[i];
 *   W_S       = the student's key projection: rows i*d .. i*d+d hold M^T of
 *               pairs[i] (the linear layer's weight layout).
 * The loss is evaluated without forming any T x T logit matrix: with
 * K_r = X W_K^r, D = (K_a - K_b)^T (K_a - K_b) and H = S_a (S_a + S_b)^+ S_b,
 * Eq. (13) at the Eq. (15) optimum equals trace(D H) (the two sums of Eq. 13
 * become (K_b - K_a) S_b S^+ and (K_a - K_b) S_a S^+ seen through S_a and
 * S_b, which add up to H).
 *
 * Conventions: as for saga.h. Device pointers owned by the caller, nothing
 * allocated, asynchronous on `stream`, host-side argument checks that
 * enqueue nothing on failure, bounded on-chip waits that set the device
 * error word instead of hanging.
 */
#ifndef SAGA_MERGE_H_
#define SAGA_MERGE_H_

#include <stddef.h>
#include <stdint.h>

#include "saga.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Shapes and layouts (row-major, last index contiguous, bf16 inputs):
 *   X      [T][d_model]         calibration hidden states, one token per row
 *   W_K    [h_k * d][d_model]   teacher key projection (linear-layer weight):
 *                               key head r's keys are X W_K[r*d:(r+1)*d]^T
 *   Q      [T][h_q * d]         calibration queries; Q^j = columns j*d..j*d+d
 *   Query head j belongs to teacher key head floor(j * h_k / h_q).
 * Requirements (SAGA_ERR_INVALID_ARG otherwise): T >= 128 and T % 8 == 0;
 * d_model >= 64 and d_model % 8 == 0 (row strides and tile boxes of the
 * TMA copies); h_k even, h_k >= 2; h_q % h_k == 0. Supported
 * (SAGA_ERR_UNSUPPORTED otherwise): d in {64, 128}; h_k <= 16;
 * T <= 2^21; d_model <= 2^20; h_q * d <= 2^20. X, W_K and Q 16-byte aligned.
 */
typedef struct saga_merge_shape {
  int32_t T, d_model, h_q, h_k, d;
} saga_merge_shape;

/*
 * Bytes of device workspace saga_merge_keys needs (256-byte aligned base;
 * 0 if the shape is invalid). Holds the transposed queries, the teacher's
 * keys as bf16 hi/lo pairs, the Gram partial sums, per-pair matrices, the
 * matching table and the device error word. Zero it once with
 * saga_workspace_init after allocation.
 */
size_t saga_merge_workspace_size(const saga_merge_shape *shape);

/*
 * The closed-form merge stage.
 *   X, W_K, Q  bf16 inputs as above.
 *   rcond      pseudoinverse cutoff: eigenvalues of S_a + S_b with
 *              |lambda| <= rcond * max |lambda| count as zero. The Gram
 *              matrices are accumulated in fp32, so exactly singular
 *              directions carry noise near 1e-7 of the largest eigenvalue:
 *              1e-6 is a sensible value. Must be >= 0.
 *   w          [h_k][h_k] float64, written (symmetric, zero diagonal).
 *   pairs      [h_k / 2][2] int32, written.
 *   total      nullable [1] float64: the matching's summed weight.
 *   W_S        [h_k / 2 * d][d_model] float32, written.
 * Errors: SAGA_ERR_INVALID_ARG for null or misaligned pointers, a bad shape
 * or rcond; SAGA_ERR_UNSUPPORTED for a shape outside the supported sizes;
 * SAGA_ERR_WORKSPACE for a missing, misaligned or short workspace;
 * SAGA_ERR_CUDA if a launch fails.
 */
saga_status saga_merge_keys(const saga_merge_shape *shape, const void *X,
                            const void *W_K, const void *Q, double rcond,
                            double *w, int32_t *pairs, double *total,
                            float *W_S, void *ws, size_t ws_bytes,
                            saga_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGA_MERGE_H_ */
