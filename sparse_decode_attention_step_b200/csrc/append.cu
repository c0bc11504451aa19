// KV-cache append: each sequence's new key rows (every key head) and value
// rows (every value head) go to position l_kv[b] of the caches, then
// l_kv[b] grows by one. One CTA per sequence; rows are copied in 16-byte
// words. A full cache (or a negative length) writes nothing and sets the
// device error word.
#include "common.cuh"
#include "kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, uint4 *K, uint4 *V,
              int32_t *l_kv, int32_t *err, int h_k, int h_v, int row_words, int64_t k_sb,
              int64_t k_sh, int64_t v_sb, int64_t v_sh, int64_t cap) {
  const int b = blockIdx.x;
  const int64_t t = l_kv[b];                 // read by every thread before the update below
  if (t < 0 || t >= cap) {
    if (threadIdx.x == 0) atomicOr(err, t < 0 ? SAGA_DEVERR_LKV_NEGATIVE : SAGA_DEVERR_LKV_TOO_LONG);
    return;
  }
  // strides arrive in 16-byte words
  for (int i = threadIdx.x; i < h_k * row_words; i += kThreads) {
    const int hh = i / row_words, w = i % row_words;
    K[b * k_sb + hh * k_sh + t * row_words + w] = k_new[(static_cast<int64_t>(b) * h_k + hh) * row_words + w];
  }
  for (int i = threadIdx.x; i < h_v * row_words; i += kThreads) {
    const int hh = i / row_words, w = i % row_words;
    V[b * v_sb + hh * v_sh + t * row_words + w] = v_new[(static_cast<int64_t>(b) * h_v + hh) * row_words + w];
  }
  __syncthreads();
  if (threadIdx.x == 0) l_kv[b] = static_cast<int32_t>(t + 1);
}

}  // namespace

cudaError_t launch_append(const void *k_new, const void *v_new, void *K, void *V, int32_t *l_kv,
                          int32_t *err, int B, int h_k, int h_v, int d, int esz, int64_t k_sb,
                          int64_t k_sh, int64_t v_sb, int64_t v_sh, int64_t cap,
                          cudaStream_t st) {
  const int row_words = d * esz / 16;
  const int64_t wpe = 16 / esz;              // elements per 16-byte word
  append_kernel<<<B, kThreads, 0, st>>>(
      static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
      static_cast<uint4 *>(K), static_cast<uint4 *>(V), l_kv, err, h_k, h_v, row_words,
      k_sb / wpe, k_sh / wpe, v_sb / wpe, v_sh / wpe, cap);
  return cudaGetLastError();
}

}  // namespace saga
