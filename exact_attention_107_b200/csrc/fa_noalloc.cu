// fa_noalloc.cu -- fa_bwd_noalloc: the backward pass for callers that cannot allocate.
//
// fa_bwd and fa_bwd_deterministic need a device workspace that the caller allocates.
// Some callers cannot: code that is handed only its input and output buffers by a host
// framework which plans all device memory up front and gives an operator neither a
// workspace nor access to an allocator.  For them this entry point runs the three-stage
// backward of fa_bwd_deterministic (whose workspace is only the per-row statistics:
// -lse * log2(e) and delta = rowsum(dO * O)) on a fixed scratch array that lives in the
// library's own device memory instead.
//
// The scratch is a file-scope __device__ array of FA_NOALLOC_SCRATCH_BYTES.  Every
// GPU that loads the library holds it until the process exits.  In host code the
// array's name is only a host-side stand-in, never a device address, so its device
// address is looked up (cudaGetSymbolAddress, with that device current) by the first
// call that runs on the device, and that address is what the kernels receive.  Only a
// successful lookup is kept; after a failed one the error is cleared and the next call
// on that device tries again.  Nothing in the scratch has to start at zero: the
// preprocess kernel writes every value the later kernels read, so stale contents from
// an earlier call are never used.  All calls share the one array, so two calls whose
// work overlaps on the GPU (different streams, no ordering between them) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (looked up on first use).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();   // clear the (non-sticky) error so that a later call can retry
      return FA_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return FA_OK;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                              const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int D,
                              float scale, int causal, void* stream) {
  const size_t need = fa_bwd_deterministic_workspace_size(B, H, N, D);
  if (need == 0) {
    // Unsupported shape: let the backward report the precise reason (it returns before any launch).
    return fa_bwd_deterministic(q, k, v, o, dO, lse, dq, dk, dv, nullptr, 0, B, H, N, D, scale, causal, stream);
  }
  if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_NOALLOC_CAPACITY;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != FA_OK) return st;
  return fa_bwd_deterministic(q, k, v, o, dO, lse, dq, dk, dv, scratch, FA_NOALLOC_SCRATCH_BYTES, B, H, N, D, scale,
                              causal, stream);
}
