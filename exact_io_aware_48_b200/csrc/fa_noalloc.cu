// fa_noalloc.cu -- fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point where they run the backward: for
// example code hosted inside a framework or plugin host that owns all device memory and forbids allocation while
// it executes, or a latency-sensitive loop that cannot afford cudaMalloc's implicit device synchronisation.  Such
// a caller still owns and passes q, k, v, o, dO, lse and dq, dk, dv; this entry point supplies the scratch that
// fa_bwd otherwise takes as `workspace` from a fixed file-scope device array of FA_NOALLOC_SCRATCH_BYTES.
//
// The array lives in every GPU that loads the library until the process exits.  In host code its name is only a
// host-side stand-in, not a device address, so the device address is fetched with cudaGetSymbolAddress once per
// device (with that device current) on the first call made on that device, and passed on as the workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "fa.h"

namespace {

// Backward scratch shared by every fa_bwd_noalloc call on a device.  Its contents persist between calls; fa_bwd
// rewrites everything it reads from it (it zeroes the dQ accumulator itself), so nothing needs clearing here.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                              float softmax_scale, int causal, const int32_t* key_lens, const uint8_t* block_mask,
                              int dtype, void* stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d, block_mask != nullptr);
  if (need == 0) return (d != 32 && d != 64 && d != 96 && d != 128 && B >= 1 && H >= 1 && N >= 1) ? FA_ERR_UNSUPPORTED
                                                                             : FA_ERR_INVALID_ARG;
  if (need > (size_t)FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;  // problem too large for the fixed array
  void* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal, key_lens, block_mask, scratch,
                (size_t)FA_NOALLOC_SCRATCH_BYTES, dtype, stream);
}
