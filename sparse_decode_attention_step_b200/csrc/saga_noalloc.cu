// A plain Atop-N decode step for callers that cannot allocate device memory.
//
// Some hosts run this step where cudaMalloc is off limits: inside a custom
// allocator's own callbacks, in a runtime that hands out only its own
// preallocated pools, or in a process whose memory budget is frozen after
// start-up. For them this entry point keeps its scratch (the device error
// word and the per-split softmax states) in one fixed array compiled into the
// library, instead of a caller-provided workspace. Every GPU that loads the
// library holds that array until the process exits.
//
// The caller still passes q, K, V, l_kv, tau and out (and optionally
// sel_count), exactly as for saga_decode_step; the same checks and kernels
// do the work.
#include <mutex>

#include "kernels.h"
#include "saga.h"

namespace {

constexpr size_t kScratchBytes = SAGA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Shared by every call on a device; keeps the previous call's contents.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void *g_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device, resolved once per
// device (host code cannot use the symbol itself as a device pointer).
saga_status scratch_for_current_device(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return saga::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return saga::cuda_fail(cudaErrorInvalidDevice, "device index");
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return saga::cuda_fail(e, "cudaGetSymbolAddress (no-alloc scratch)");
    if (p == nullptr) return saga::cuda_fail(cudaErrorInvalidSymbol, "cudaGetSymbolAddress (no-alloc scratch)");
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return SAGA_OK;
}

}  // namespace

extern "C" saga_status saga_decode_step_noalloc(const saga_shape *shape, const void *q,
                                                const void *K, const void *V,
                                                const int32_t *l_kv, const float *tau,
                                                float *out, int32_t *sel_count,
                                                saga_stream_t stream) {
  if (saga_workspace_size(shape, 1) == 0) return SAGA_ERR_INVALID_ARG;   // invalid shape
  if (saga::plain_step_scratch_bytes(*shape) > kScratchBytes) return SAGA_ERR_WORKSPACE;
  void *scratch = nullptr;
  saga_status r = scratch_for_current_device(&scratch);
  if (r != SAGA_OK) return r;
  // Nothing in the scratch needs clearing between calls: every per-split
  // state the step reads was written earlier in the same step, and the error
  // word at its head is only ever OR-ed into, never read back here.
  return saga::plain_step_with_scratch(shape, q, K, V, l_kv, tau, out, sel_count, scratch,
                                       kScratchBytes, reinterpret_cast<cudaStream_t>(stream));
}
