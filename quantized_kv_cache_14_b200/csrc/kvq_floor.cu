// kvq_floor.cu -- measurement kernels: the HBM read floor of a decode pass.
//
// Decode attention over a compressed cache is meant to be bound by memory
// traffic (llmdaily.org day-65, "Why compression may also improve speed"), so
// the floor of one decode call is the time a single launch needs just to read
// the bytes the call must read.  These kernels read a list of chunks and do
// nothing with them but fold one word per chunk into a checksum; their time is
// that floor for a given way of reading:
//
//  * bulk: the decode kernel's scheme.  A persistent grid of CTAs of four
//    warps; each CTA takes a contiguous share of the chunk list and each warp
//    every fourth unit (`per_unit` chunks) of it, filling `stages` shared-memory
//    stages per warp with bulk asynchronous copies (cp.async.bulk) that
//    complete on one mbarrier per stage, and re-issuing a stage as soon as it
//    has landed.  The chunk list is either a contiguous buffer or the page
//    chunks a decode call stages (offsets computed from the block table).
//  * stream: plain 128-bit non-coherent loads of a contiguous buffer by every
//    thread, eight in flight per thread.
//
// Every offset is checked against the buffer's size before it is read; a bad
// one, or a wait that gives up after 2 s, sets sink[1] instead of faulting.
#include <cstdint>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kFloorWarps = 4;
constexpr uint64_t kFloorWaitNs = 2000000000ull;

struct FloorArgs {
  const uint8_t* base;
  const int64_t* offsets;   // null: chunk i starts at base + i * chunk_bytes
  int64_t n_chunks;
  int64_t span;             // bytes readable from base
  int32_t chunk_bytes;      // multiple of 16
  int32_t per_unit;         // chunks per unit, <= 32
  int32_t stages;           // stages per warp
  int32_t stage_bytes;      // per_unit * chunk_bytes rounded up to 128
  uint32_t* sink;           // [0] checksum, [1] error flag
};

__global__ void __launch_bounds__(kFloorWarps * 32) floor_bulk_kernel(const __grid_constant__ FloorArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int S = a.stages;
  const uint32_t stage0 = smem_addr(smem) + uint32_t(warp * S) * uint32_t(a.stage_bytes);
  const uint32_t bar0 = smem_addr(smem) + uint32_t(kFloorWarps * S) * uint32_t(a.stage_bytes) + 8u * uint32_t(warp * S);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFloorWarps * S; ++s)
      mbar_init(smem_addr(smem) + uint32_t(kFloorWarps * S) * uint32_t(a.stage_bytes) + 8u * s, 1);
    mbar_init_fence();
  }
  __syncthreads();
  const int64_t units = (a.n_chunks + a.per_unit - 1) / a.per_unit;
  const int64_t u0 = int64_t(blockIdx.x) * units / gridDim.x;
  const int64_t u1 = int64_t(blockIdx.x + 1) * units / gridDim.x;
  const int64_t K = u1 - u0 > warp ? (u1 - u0 - warp + kFloorWarps - 1) / kFloorWarps : 0;

  // the chunk of unit k this lane copies (or -1), checked against the span
  auto src_of = [&](int64_t k, int& nc) -> int64_t {
    const int64_t c0 = (u0 + warp + kFloorWarps * k) * a.per_unit;
    nc = int(min(int64_t(a.per_unit), a.n_chunks - c0));
    if (lane >= nc) return -1;
    const int64_t off = a.offsets ? a.offsets[c0 + lane] : (c0 + lane) * int64_t(a.chunk_bytes);
    const bool ok = off >= 0 && (off & 15) == 0 && off + a.chunk_bytes <= a.span;
    return ok ? off : -2;
  };
  auto issue = [&](int64_t k, int s) {
    int nc = 0;
    const int64_t off = src_of(k, nc);
    const bool bad = __any_sync(0xffffffffu, off == -2);
    fence_proxy_async();
    const uint32_t bar = bar0 + 8u * s;
    if (bad) {   // copy nothing; the stage completes empty
      if (lane == 0) {
        atomicOr(&a.sink[1], 1u);
        mbar_arrive_expect_tx(bar, 0);
      }
      return;
    }
    if (lane == 0) mbar_arrive_expect_tx(bar, uint32_t(nc) * uint32_t(a.chunk_bytes));
    __syncwarp();
    if (off >= 0) bulk_g2s(stage0 + uint32_t(s * a.stage_bytes + lane * a.chunk_bytes), a.base + off,
                           uint32_t(a.chunk_bytes), bar);
  };

  int64_t issued = 0;
  for (; issued < K && issued < S; ++issued) issue(issued, int(issued));
  uint32_t acc = 0;
  int64_t k = 0;
  for (; k < K; ++k) {
    const int s = int(k % S);
    const bool ok = mbar_wait_bounded(bar0 + 8u * s, uint32_t((k / S) & 1), kFloorWaitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) atomicOr(&a.sink[1], 2u);
      break;
    }
    int nc = 0;
    (void)src_of(k, nc);
    if (lane < nc)
      acc ^= *reinterpret_cast<const uint32_t*>(smem + size_t(warp * S + s) * a.stage_bytes + size_t(lane) * a.chunk_bytes);
    __syncwarp();
    if (issued < K) {
      issue(issued, s);
      ++issued;
    }
  }
  // after a timeout, wait (bounded) for this warp's copies still in flight
  for (int64_t j = k; j < issued; ++j)
    (void)mbar_wait_bounded(bar0 + 8u * int(j % S), uint32_t((j / S) & 1), kFloorWaitNs);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0 && acc) atomicXor(&a.sink[0], acc);
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__global__ void __launch_bounds__(256) floor_stream_kernel(const uint4* p, int64_t n16, uint32_t* sink) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 7 * stride < n16; i += 8 * stride) {
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = ldg_stream(p + i + j * stride);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc ^= v[j].x ^ v[j].y ^ v[j].z ^ v[j].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ldg_stream(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0 && acc) atomicXor(&sink[0], acc);
}

}  // namespace

size_t floor_smem_bytes(int chunk_bytes, int per_unit, int stages) {
  const size_t stage = (size_t(per_unit) * size_t(chunk_bytes) + 127) / 128 * 128;
  return size_t(kFloorWarps) * size_t(stages) * (stage + 8);
}

cudaError_t launch_floor(const void* base, const int64_t* offsets, int64_t n_chunks, int64_t span,
                         int chunk_bytes, int mode, int ctas, int stages, int per_unit, uint32_t* sink,
                         cudaStream_t s) {
  if (mode == 1) {
    const int64_t n16 = span / 16;
    floor_stream_kernel<<<ctas, 256, 0, s>>>(static_cast<const uint4*>(base), n16, sink);
    return cudaGetLastError();
  }
  FloorArgs a{};
  a.base = static_cast<const uint8_t*>(base);
  a.offsets = offsets;
  a.n_chunks = n_chunks;
  a.span = span;
  a.chunk_bytes = chunk_bytes;
  a.per_unit = per_unit;
  a.stages = stages;
  a.stage_bytes = int((int64_t(per_unit) * chunk_bytes + 127) / 128 * 128);
  a.sink = sink;
  const size_t smem = floor_smem_bytes(chunk_bytes, per_unit, stages);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = raise_smem_limit(dev, reinterpret_cast<const void*>(&floor_bulk_kernel), smem);
  if (e != cudaSuccess) return e;
  floor_bulk_kernel<<<ctas, kFloorWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
