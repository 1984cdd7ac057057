// frnnt_fwd_bwd_noalloc: frnnt_fwd_bwd with its workspace in a fixed,
// library-owned device array instead of caller-provided memory.
//
// Who needs it: callers that cannot call cudaMalloc (or any allocator) at
// the point where they run the loss -- for example code running inside a
// host framework whose allocator owns all device memory and hands out only
// the input/output tensors, plug-ins that must not grow the process's memory
// footprint at run time, or code paths that must not call into an allocator
// because doing so could synchronise the device.  They still pass every
// input and output buffer; only the scratch memory is supplied here.
//
// The scratch is one file-scope __device__ array of FRNNT_NOALLOC_MAX_BYTES.
// Every GPU that loads this file's module holds it until the process exits.
// With lazy module loading (the CUDA 12 default) the driver loads the module,
// and reserves the array, inside the first cudaGetSymbolAddress on a device,
// i.e. during the first call there: callers make that call at start-up.
#include <atomic>

#include "frnnt_common.cuh"
#include "frnnt_internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)FRNNT_NOALLOC_MAX_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress (once per device, with that device current).
// Threads racing on a device's first call each look the address up (the
// same value) and store it atomically.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FRNNT_ERR_CUDA;
  }
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();   // e.g. out of memory while the module loads: leave no sticky error behind
      return FRNNT_ERR_CUDA;
    }
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return FRNNT_OK;
}

}  // namespace

extern "C" FRNNT_API int frnnt_fwd_bwd_noalloc(const frnnt_dims* d, const void* f, const void* g, const void* W_f,
                                               const void* W_g, const void* W_o, const void* b_o,
                                               const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                                               const float* grad_loss, float* loss, void* df, void* dg, void* dW_f,
                                               void* dW_g, void* dW_o, void* db_o, int32_t* status, void* stream) {
  size_t need = 0;
  int rc = frnnt_workspace_size(d, &need);
  if (rc != FRNNT_OK) return rc;
  if (need > kScratchBytes) return FRNNT_ERR_WORKSPACE;   // larger than the fixed scratch array
  void* scratch = nullptr;
  rc = scratch_for_current_device(&scratch);
  if (rc != FRNNT_OK) return rc;
  // frnnt_fwd_bwd clears on the stream every workspace region it accumulates
  // into, so the previous call's leftovers in the shared array are harmless.
  return frnnt_fwd_bwd(d, f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, loss, df, dg, dW_f, dW_g, dW_o,
                       db_o, scratch, kScratchBytes, status, stream);
}
