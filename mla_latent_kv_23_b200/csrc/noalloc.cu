// mla_decode_noalloc: mla_decode with its scratch space in a fixed device
// array that belongs to the library, for callers that cannot allocate
// device memory themselves.
//
// Some hosts own every byte of device memory (a serving engine that carves
// a fixed pool at start-up, a plugin interface that hands kernels only
// their inputs and outputs) and give a kernel library no way to obtain a
// workspace.  For them this entry point uses the array below instead of a
// caller-provided workspace.  It calls no cudaMalloc, cudaFree or any other
// allocating routine.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoallocScratchBytes for it until the process exits.  All
// calls on a device share it, so two calls whose work overlaps on the GPU
// (different streams without ordering between them) race on it; order
// them.  Nothing in it needs to start at zero: every word the decode reads
// from its scratch is written earlier in the same call.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "mla.h"

namespace mla {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// In host code `g_noalloc_scratch` names a host-side stand-in, not device
// memory, so the kernels get the device address looked up per device.
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

mla_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace
}  // namespace mla

extern "C" mla_status mla_decode_noalloc(const mla_decode_params* p, void* stream) {
  if (p == nullptr) return MLA_ERR_INVALID_ARG;
  if (p->B == 0) return mla_decode(p, nullptr, 0, stream);
  size_t need = 0;
  mla_status st = mla_decode_workspace_size(p, &need);
  if (st != MLA_OK) return st;
  if (need > mla::kNoallocScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if ((st = mla::scratch_for_current_device(&scratch)) != MLA_OK) return st;
  return mla_decode(p, scratch, mla::kNoallocScratchBytes, stream);
}
