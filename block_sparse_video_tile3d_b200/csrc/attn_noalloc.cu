// Scratch memory for block_sparse_attn_fwd_noalloc: the attention kernel's device scratch (the
// counter of its work queue) held in a fixed array of the library instead of a caller's workspace,
// for callers that may not allocate device memory themselves.
//
// The array is a file-scope __device__ variable, so every GPU on which the library is loaded
// holds its kNoAllocScratchBytes bytes until the process exits. In host code its name only stands
// for the variable: the device address comes from cudaGetSymbolAddress, taken once per device
// (with that device current) on the first call and cached.
#include <mutex>

#include "kernels.h"

namespace t3d {
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace t3d
