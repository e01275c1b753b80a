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
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/gbsa.h"

namespace {

constexpr size_t kScratchBytes = GBSA_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Split-KV scratch shared by every call on a device.
static __device__ __align__(256) uint8_t g_static_scratch[kScratchBytes];

std::mutex g_lock;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once
// per device (the host-side symbol is not a device address).
gbsa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GBSA_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return GBSA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return GBSA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return GBSA_OK;
}

}  // namespace

extern "C" gbsa_status gbsa_forward_static_scratch(const gbsa_problem* problem,
                                                   const gbsa_tensors* tensors, const void* meta,
                                                   int32_t* dev_status, void* stream) {
  size_t need = 0;
  gbsa_status st = gbsa_workspace_size(problem, &need);
  if (st != GBSA_OK) return st;
  if (need > kScratchBytes) return GBSA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != GBSA_OK) return st;
  return gbsa_forward(problem, tensors, meta, scratch, kScratchBytes, dev_status, stream);
}
