// gbsa_static_scratch.cu -- gbsa_forward_static_scratch(): the forward
// pass for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) when they
// run the attention: a serving engine that hands out a fixed device-memory
// budget at start-up and forbids allocation afterwards, or code that runs
// inside an allocator or a framework hook, where allocating again could
// deadlock or break the budget.  For them the split-KV scratch (fp32 partial
// outputs and log-sum-exps, the only memory the forward needs beyond its
// inputs and outputs) lives in the file-scope array below, which the CUDA
// module creates on every GPU that loads this library and keeps until the
// process exits.  The caller still passes the inputs, the outputs and the
// metadata buffer.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/gbsa.h"

namespace {

constexpr size_t kScratchBytes = GBSA_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Split-KV scratch shared by every call on a device.
static __device__ __align__(256) uint8_t g_static_scratch[kScratchBytes];

// The address is a property of the context that loaded the module: after
// cudaDeviceReset the primary context (and the module in it) is created
// anew, and a caller may make another context of the same device current.
// So the cache of each device remembers the unique id of the context it was
// filled in, and the set-up runs again when the current context differs.
struct Cached {
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_lock;
Cached g_cache[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return reinterpret_cast<Fn>(ptr);
}

// Unique id of the context current on this thread (made current by the
// runtime call before it); 0 if it cannot be read.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_static_scratch in the current context.  The set-up
// (cudaGetSymbolAddress, which also loads the module holding the array on
// first use) runs once per device and context; later calls read the cache.
gbsa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GBSA_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return GBSA_ERR_NO_DEVICE;
  // 0 when no context is current yet (the runtime makes the device's primary
  // context current in the set-up below)
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> guard(g_lock);
  Cached& c = g_cache[dev];
  if (!c.ptr || ctx == 0 || c.ctx_id != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      c = Cached{0, nullptr};
      return GBSA_ERR_CUDA;
    }
    c = Cached{current_context_id(), ptr};
  }
  *out = c.ptr;
  return GBSA_OK;
}

}  // namespace

extern "C" gbsa_status gbsa_forward_static_scratch(const gbsa_problem* problem,
                                                   const gbsa_tensors* tensors, void* meta,
                                                   int32_t* dev_status, void* stream) {
  size_t need = 0;
  gbsa_status st = gbsa_workspace_size(problem, &need);
  if (st != GBSA_OK) return st;
  if (need > kScratchBytes) return GBSA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != GBSA_OK) return st;
  return gbsa_forward(problem, tensors, meta, scratch, kScratchBytes, dev_status, stream);
}
