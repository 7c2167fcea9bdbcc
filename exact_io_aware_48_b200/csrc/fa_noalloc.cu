// fa_noalloc.cu -- fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point where they run the backward: for
// example code hosted inside a framework or plugin host that owns all device memory and forbids allocation while
// it executes, or a latency-sensitive loop that cannot afford cudaMalloc's implicit device synchronisation.  Such
// a caller still owns and passes q, k, v, o, dO, lse and dq, dk, dv; this entry point supplies the scratch that
// fa_bwd otherwise takes as `workspace` from a fixed file-scope device array of FA_NOALLOC_SCRATCH_BYTES.
//
// The array lives in every GPU whose context loads this file's module, until the context is destroyed.  In host
// code its name is only a host-side stand-in, not a device address, so the device address is fetched with
// cudaGetSymbolAddress at set-up: once per device (with that device current), on the first call made on that
// device, and again only if that device's context has been replaced since (after cudaDeviceReset a new context
// loads the module again and the array may sit at a new address).  A context is recognised by its process-unique
// id (cuCtxGetId), so the check costs two driver queries and no allocation.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_abi_checks.h"

namespace {

// Backward scratch shared by every fa_bwd_noalloc call on a device.  Its contents persist between calls; fa_bwd
// rewrites everything it reads from it (it zeroes the dQ accumulator and rebuilds the per-row LSE / D values and the
// block-mask lists itself), so nothing needs clearing here.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const DriverFns& driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

// Id of the context current on this thread, or 0 if there is none (or the driver cannot say).
unsigned long long current_context_id() {
  const DriverFns& f = driver_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct DeviceSlot {
  unsigned long long ctx_id = 0;  // context the address below belongs to (0: not set up)
  void* ptr = nullptr;
};

std::mutex g_mu;
DeviceSlot g_slots[kMaxDevices];

// Device address of the scratch array in the current device's context: looked up at set-up and cached.
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceSlot& s = g_slots[dev];
  if (id != 0 && s.ctx_id == id && s.ptr != nullptr) {
    *out = s.ptr;
    return cudaSuccess;
  }
  // Set-up: the first call on this device, or its context changed.  cudaGetSymbolAddress also makes the device's
  // primary context current on this thread if no runtime call has done so yet; it allocates nothing beyond
  // loading the module that holds the array.
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  s.ptr = p;
  s.ctx_id = current_context_id();  // 0 if unknown: the next call looks the address up again
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                              float softmax_scale, int causal, const int32_t* key_lens, const uint8_t* block_mask,
                              int dtype, void* stream) {
  // the same argument checks as fa_bwd, in the same order, so both calls report the same status
  const int rc = fa_abi::bwd_check_args(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, key_lens,
                                        block_mask, dtype);
  if (rc != FA_OK) return rc;
  const size_t need = fa_bwd_workspace_size(B, H, N, d, block_mask != nullptr);
  if (need == 0) return FA_ERR_INVALID_ARG;                              // not reached after the checks above
  if (need > (size_t)FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;  // problem too large for the fixed array
  void* scratch = nullptr;
  const cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal, key_lens, block_mask, scratch,
                (size_t)FA_NOALLOC_SCRATCH_BYTES, dtype, stream);
}
