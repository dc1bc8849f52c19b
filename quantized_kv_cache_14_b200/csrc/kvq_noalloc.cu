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

#include <cuda_runtime.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device

__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the scratch array in the current context.  Host code
// cannot use the array's name as a device address, so every call looks it up
// with cudaGetSymbolAddress: the lookup is cheap, and it stays right when the
// context is torn down and rebuilt (the module then loads again and the array
// may move).
cudaError_t noalloc_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace kvq
