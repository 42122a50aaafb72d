// noalloc.cu — hstu_layer_fwd_noalloc: one HSTU layer for callers that
// cannot allocate device memory (a host runtime whose allocator is owned by
// someone else, a process that must not call cudaMalloc after start-up, code
// already running inside a memory-capped sandbox).  Its scratch space is a
// fixed, file-scope device array instead of a caller-provided workspace.
#include <mutex>

#include "hstu_internal.h"

namespace {

// The scratch every call of hstu_layer_fwd_noalloc uses.  Every device that
// loads this library holds it (HSTU_NOALLOC_SCRATCH_BYTES) until the process
// exits.  In host code this name is only a handle: its device address comes
// from cudaGetSymbolAddress, once per device.
__device__ __align__(256) uint8_t g_noalloc_scratch[HSTU_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device (first use: the
// symbol lookup, with that device current).  Null on failure.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" hstu_status hstu_layer_fwd_noalloc(const hstu_layer_desc* desc, int64_t B,
                                              int64_t total_tokens, int64_t max_len,
                                              const int64_t* offsets, const void* X,
                                              const hstu_layer_weights* weights,
                                              const int64_t* timestamps, void* out,
                                              void* stream) {
  const size_t need = hstu_workspace_size(desc, 1, B, total_tokens, max_len, 0, 0, 0);
  if (need == 0) return HSTU_ERR_INVALID_ARG;
  if (need > (size_t)HSTU_NOALLOC_SCRATCH_BYTES) return HSTU_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return HSTU_ERR_CUDA;
  return hstu_layer_fwd(desc, B, total_tokens, max_len, offsets, X, weights, timestamps, out,
                        scratch, (size_t)HSTU_NOALLOC_SCRATCH_BYTES, stream);
}
