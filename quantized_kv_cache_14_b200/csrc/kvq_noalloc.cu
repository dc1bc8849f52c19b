// kvq_noalloc.cu -- fixed scratch for kvq_decode_attn_noalloc.
//
// Some callers cannot allocate device memory at the time they decode: a
// runtime that hands this library a pre-sized arena, a process whose
// allocations must all happen at start-up, or a host that forbids allocation
// on its serving path.  For them, decode's scratch (the split-K partials, the
// per-row tile prefix and the device error word) lives in one file-scope
// device array instead of handle-owned memory.  Every GPU that loads the
// library keeps this array until the process exits.
#include <cstddef>
#include <mutex>

#include <cuda_runtime.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device

__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the scratch array on the current device.  The first call
// on a device looks it up with cudaGetSymbolAddress (host code cannot use the
// array's name as a device address); later calls reuse the cached pointer.
cudaError_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace kvq
