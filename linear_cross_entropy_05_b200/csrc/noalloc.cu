// Allocation-free variant of cce_forward.
//
// Some callers cannot allocate device memory at the point where they need the
// loss: code running under an allocator that is locked or exhausted, plugins
// and inference hooks handed only their input and output buffers, or a
// runtime that forbids cudaMalloc inside its step.  cce_forward_noalloc
// serves them: its scratch (the status block and the per-split (max, sum)
// partials the forward kernel writes) lives in the file-scope device array
// below, which the CUDA module reserves on every GPU that loads this library
// and keeps until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/cce.h"

namespace {

// Maximum scratch: enough for N x splits x 8 bytes of partials plus the
// 256-byte status block on the workloads up to N = 32768 tokens (see
// cce_forward_workspace_size for the exact need of a given size).
constexpr size_t kNoallocScratchBytes = size_t(8) << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the array, looked up once per device and CUDA context.
// The name g_noalloc_scratch is only a host-side stand-in in host code: a
// kernel given &g_noalloc_scratch would fault (or, where the GPU can reach
// host memory, silently use the wrong memory), so the address comes from
// cudaGetSymbolAddress with the device current.  The cached address belongs
// to the context the module was loaded into: when the device's current
// context is another one (after cudaDeviceReset, or a context the caller
// created), the module is loaded anew there and the address is looked up
// again.
struct ScratchSlot {
  std::mutex mu;
  void* ctx = nullptr;  // context the cached address belongs to
  void* ptr = nullptr;
};
constexpr int kMaxDevices = 64;
ScratchSlot g_slots[kMaxDevices];

typedef int (*CtxGetCurrentFn)(void**);  // CUresult cuCtxGetCurrent(CUcontext*)

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

cce_status_t device_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CCE_ERR_CUDA;
  // make the device's primary context current (cudaSetDevice initialises
  // it if needed), then identify it
  if (cudaSetDevice(dev) != cudaSuccess) return CCE_ERR_CUDA;
  CtxGetCurrentFn get = ctx_get_current();
  void* ctx = nullptr;
  if (!get || get(&ctx) != 0 || ctx == nullptr) return CCE_ERR_CUDA;
  ScratchSlot& s = g_slots[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (s.ptr == nullptr || s.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CCE_ERR_CUDA;
    s.ptr = p;
    s.ctx = ctx;
  }
  *out = s.ptr;
  return CCE_OK;
}

}  // namespace

extern "C" cce_status_t cce_forward_noalloc(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D,
                                            int64_t V, int64_t ignore_index, float* loss, float* lse,
                                            void* stream) {
  const size_t need = cce_forward_workspace_size(N, D, V);
  if (need == 0) return CCE_ERR_INVALID_ARG;
  if (need > kNoallocScratchBytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const cce_status_t st = device_scratch(&scratch);
  if (st != CCE_OK) return st;
  return cce_forward(E, C, y, N, D, V, ignore_index, loss, lse, scratch, kNoallocScratchBytes, stream);
}
