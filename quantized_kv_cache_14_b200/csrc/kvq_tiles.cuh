// kvq_tiles.cuh -- register fragments of packed 16-token sub-tiles for the
// mma.sync m16n8k16 products of the attention kernels (decode and chunked
// prefill), and the small metadata / splitting helpers they share.
//
// A key sub-tile is 16 rows of packed codes; lane (gq = lane / 4, tq = lane %
// 4) holds the words of rows gq and gq + 8 at byte slice tq of the row.  Its
// k-step j (16 of the 128 channels) pairs k = 2tq, 2tq + 1 with channels
// 32tq + 4j + {0, 1} and k = 2tq + 8, 2tq + 9 with channels 32tq + 4j + {2, 3};
// the other operand of a score product must use the same channel order.  A
// value sub-tile is a lane record: channel tile i (16 channels) x the lane's
// tokens 2tq, 2tq + 1, 2tq + 8, 2tq + 9.  Codes become exact small integers in
// fp16 (see the *_pair_h helpers of kvq_device.cuh).
#pragma once
#include <cstdint>

#include "kvq_device.cuh"

namespace kvq {
namespace {

// Key words of rows gq and gq + 8 of a packed 16-token sub-tile.
template <int BITS>
__device__ __forceinline__ void load_key_words(const uint8_t* ksub, int gq, int tq, uint32_t (&wa)[BITS],
                                               uint32_t (&wb)[BITS]) {
  constexpr int row = kD * BITS / 8, slice = 4 * BITS;
  const uint8_t* pa = ksub + gq * row + tq * slice;
  const uint8_t* pb = pa + 8 * row;
  if (BITS == 2) {
    const uint2 x = *reinterpret_cast<const uint2*>(pa);
    const uint2 y = *reinterpret_cast<const uint2*>(pb);
    wa[0] = x.x; wa[1 % BITS] = x.y; wb[0] = y.x; wb[1 % BITS] = y.y;
  } else {
#pragma unroll
    for (int v = 0; v < BITS / 4; ++v) {
      const uint4 x = reinterpret_cast<const uint4*>(pa)[v];
      const uint4 y = reinterpret_cast<const uint4*>(pb)[v];
      wa[4 * v] = x.x; wa[4 * v + 1] = x.y; wa[4 * v + 2] = x.z; wa[4 * v + 3] = x.w;
      wb[4 * v] = y.x; wb[4 * v + 1] = y.y; wb[4 * v + 2] = y.z; wb[4 * v + 3] = y.w;
    }
  }
}

// One operand register from two codes: fp16 (H) or bf16.
template <bool SGN, bool H>
__device__ __forceinline__ uint32_t nib2(uint32_t w, int x) {
  return H ? nib_pair_h<SGN>(w, x) : nib_pair<SGN>(w, x);
}
template <bool SGN, bool H>
__device__ __forceinline__ uint32_t crumb2(uint32_t w, int x) {
  return H ? crumb_pair_h<SGN>(w, x) : crumb_pair<SGN>(w, x);
}
template <bool SGN, bool H>
__device__ __forceinline__ uint32_t byte2(uint32_t w, int x) {
  return H ? byte_pair_h<SGN>(w, x) : byte_pair<SGN>(w, x);
}

// A operand (rows gq / gq+8, k-step j) of the score product from key words.
template <int BITS, bool SGN, bool H>
__device__ __forceinline__ void key_frag(const uint32_t (&wa)[BITS], const uint32_t (&wb)[BITS], int j,
                                         uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  if (BITS == 4) {
    const int jj = j >> 1, x = 2 * (j & 1);
    a0 = nib2<SGN, H>(wa[jj], x);
    a1 = nib2<SGN, H>(wb[jj], x);
    a2 = nib2<SGN, H>(wa[jj], x + 1);
    a3 = nib2<SGN, H>(wb[jj], x + 1);
  } else if (BITS == 2) {
    const int jj = j >> 2, x = 2 * (j & 3);
    a0 = crumb2<SGN, H>(wa[jj], x);
    a1 = crumb2<SGN, H>(wb[jj], x);
    a2 = crumb2<SGN, H>(wa[jj], x + 1);
    a3 = crumb2<SGN, H>(wb[jj], x + 1);
  } else {
    a0 = byte2<SGN, H>(wa[j], 0);
    a1 = byte2<SGN, H>(wb[j], 0);
    a2 = byte2<SGN, H>(wa[j], 1);
    a3 = byte2<SGN, H>(wb[j], 1);
  }
}

// A operand of the value product for channel tile i from a lane record.
template <int BITS, bool SGN, bool H>
__device__ __forceinline__ void value_frag(const uint32_t (&w)[2 * BITS], int i, uint32_t& a0, uint32_t& a1,
                                           uint32_t& a2, uint32_t& a3) {
  if (BITS == 4) {
    a0 = nib2<SGN, H>(w[i], 0);
    a1 = nib2<SGN, H>(w[i], 1);
    a2 = nib2<SGN, H>(w[i], 2);
    a3 = nib2<SGN, H>(w[i], 3);
  } else if (BITS == 2) {
    const int b = 2 * (i & 1);
    a0 = crumb2<SGN, H>(w[i >> 1], b);
    a1 = crumb2<SGN, H>(w[i >> 1], b + 1);
    a2 = crumb2<SGN, H>(w[i >> 1], b + 4);
    a3 = crumb2<SGN, H>(w[i >> 1], b + 5);
  } else {
    a0 = byte2<SGN, H>(w[2 * i], 0);
    a1 = byte2<SGN, H>(w[2 * i], 1);
    a2 = byte2<SGN, H>(w[2 * i + 1], 0);
    a3 = byte2<SGN, H>(w[2 * i + 1], 1);
  }
}

template <int BITS>
__device__ __forceinline__ void load_value_words(const uint8_t* vsub, int lane, uint32_t (&w)[2 * BITS]) {
  const uint4* p = reinterpret_cast<const uint4*>(vsub + lane * (8 * BITS));
#pragma unroll
  for (int v = 0; v < BITS / 2; ++v) {
    const uint4 x = p[v];
    w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
  }
}

__device__ __forceinline__ float meta_at(const uint8_t* base, int idx, int es) {
  return es == 4 ? reinterpret_cast<const float*>(base)[idx]
                 : __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(base)[idx]));
}

// Four consecutive metadata entries starting at a multiple of 4.
__device__ __forceinline__ void meta4(const uint8_t* base, int idx, int es, float (&v)[4]) {
  if (es == 4) {
    const float4 x = *reinterpret_cast<const float4*>(base + idx * 4);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    const uint2 x = *reinterpret_cast<const uint2*>(base + idx * 2);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&x.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&x.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
}

// Both bf16 parts of an fp32 pair: hi = bf16_rn(x), lo = bf16_rn(x - hi).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const __nv_bfloat162 l =
      __floats2bfloat162_rn(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xFFFF0000u));
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Both fp16 parts of an fp32 pair: hi = f16_rn(x), lo = f16_rn(x - hi).
__device__ __forceinline__ void split2h(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float(uint32_t(e + 127) << 23); }

}  // namespace
}  // namespace kvq
