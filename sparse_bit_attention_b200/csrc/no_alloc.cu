// Forward without any caller-provided or library-allocated device memory.
//
// Some callers cannot allocate device memory at all: a host integration that only hands over
// the input and output buffers, code running inside a memory pool that may not grow, or a
// process where cudaMalloc is forbidden once the model is loaded. For them,
// sagesla_forward_no_alloc runs the ordinary forward with its scratch (the workspace) placed
// in a fixed device array that is part of this library: every GPU that loads the library
// holds these SAGESLA_NO_ALLOC_SCRATCH_BYTES until the process exits.
//
// In host code the array's name only stands in for it; a kernel handed that name would fault
// (or, where the GPU can reach host memory, quietly use the wrong memory). The device address
// is therefore looked up with cudaGetSymbolAddress once per device, with that device current,
// on the first call made on the device, and kept for the life of the process. A
// cudaDeviceReset unloads the module and makes that address stale; the library does not see
// the reset, so this entry point must not be used on a device after it was reset.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace sagesla {
namespace {

static __device__ __align__(256) unsigned char g_no_alloc_scratch[SAGESLA_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
sagesla_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGESLA_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return SAGESLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_no_alloc_scratch) != cudaSuccess || !ptr)
      return SAGESLA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return SAGESLA_OK;
}

}  // namespace
}  // namespace sagesla

extern "C" sagesla_status sagesla_forward_no_alloc(const sagesla_tensor* q,
                                                   const sagesla_tensor* k,
                                                   const sagesla_tensor* v, double topk_ratio,
                                                   int block, sagesla_tensor* out,
                                                   void* stream) {
  if (!q || !k || !v || !out) return SAGESLA_ERR_INVALID_ARG;
  const size_t need = sagesla_workspace_size(q->B, q->H, q->N, q->D, topk_ratio, block);
  if (need == 0) {
    if (q->D != sagesla::kHeadDim || block != sagesla::kBlock) return SAGESLA_ERR_UNSUPPORTED;
    return SAGESLA_ERR_INVALID_ARG;
  }
  if (need > SAGESLA_NO_ALLOC_SCRATCH_BYTES) return SAGESLA_ERR_WORKSPACE;
  // Same device check, and so the same status, as sagesla_forward before the symbol lookup
  // (on a device that is not sm_100 the module cannot load and the lookup would fail).
  sagesla_status st = sagesla::require_b200();
  if (st != SAGESLA_OK) return st;
  void* scratch = nullptr;
  st = sagesla::scratch_address(&scratch);
  if (st != SAGESLA_OK) return st;
  // The forward clears the only scratch word it reads before writing (its status word) at the
  // start of every call; everything else it writes before reading.
  return sagesla_forward(q, k, v, topk_ratio, block, out, scratch,
                         SAGESLA_NO_ALLOC_SCRATCH_BYTES, stream);
}
