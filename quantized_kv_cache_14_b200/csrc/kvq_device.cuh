// kvq_device.cuh -- device helpers of the kvq kernels: the storage format's
// word packing, code unpacking to bf16 operand pairs, the quantizer, and thin
// wrappers over PTX (mma.sync, ldmatrix, mbarrier, bulk async copies).
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kvq_internal.h"

namespace kvq {

// ---------------------------------------------------------------------------
// Format rules (the storage contract; see the format notes).
// ---------------------------------------------------------------------------

// Key rows list channels in mma-operand order: position f = 32 t + 4 j + e
// holds channel 16 j + 2 t + (e & 1) + 8 (e >> 1).
__host__ __device__ constexpr int key_channel(int f) {
  return 16 * ((f >> 2) & 7) + 2 * (f >> 5) + (f & 1) + 8 * ((f >> 1) & 1);
}

// Element l of a word of n elements occupies field (l >> 1) + (n / 2)(l & 1):
// even elements take the low half-word, odd elements the high half-word.
__host__ __device__ constexpr int word_field(int l, int n) { return (l >> 1) + (n >> 1) * (l & 1); }

// bf16 bit pattern of an exactly representable float (compile time).
__host__ __device__ constexpr uint32_t bf16x2_of(float x) {
  return (__builtin_bit_cast(uint32_t, x) >> 16) * 0x10001u;
}

// fp16 bit pattern, twice, of a float exactly representable as a normal fp16
// (compile time).
__host__ __device__ constexpr uint32_t f16x2_of(float x) {
  const uint32_t b = __builtin_bit_cast(uint32_t, x);
  const uint32_t h = ((b >> 16) & 0x8000u) | ((((b >> 23) & 0xFFu) - 112u) << 10) | ((b >> 13) & 0x3FFu);
  return (x == 0.0f ? 0u : h) * 0x10001u;
}

// ---------------------------------------------------------------------------
// Debug-build checks.  With KVQ_DEBUG set (libkvq_debug.so) dcheck sets `bit`
// in the device error word and returns false when `ok` fails, and the caller
// skips the access; in the release build it is the constant true and compiles
// away.
// ---------------------------------------------------------------------------
#ifndef KVQ_DEBUG
#define KVQ_DEBUG 0
#endif

__device__ __forceinline__ bool dcheck(bool ok, uint32_t* err, uint32_t bit) {
  if (KVQ_DEBUG && !ok) {
    atomicOr(err, bit);
    return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// PTX wrappers.
// ---------------------------------------------------------------------------

// r = (a & mask) ^ k  (one LOP3).
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t mask, uint32_t k) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(a), "r"(mask), "r"(k));
  return r;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Two FP8 E4M3 values in the low 16 bits of v (low byte first) -> fp16x2,
// exactly (every E4M3 value is an fp16 value).
__device__ __forceinline__ uint32_t fp8x2_to_h2(uint32_t v) {
  const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(__nv_fp8x2_storage_t(v & 0xFFFFu), __NV_E4M3);
  return uint32_t(r.x) | (uint32_t(r.y) << 16);
}

// D += A * B, m16n8k16, fp16 operands, fp32 accumulation.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A * B, m16n8k16, bf16 operands, fp32 accumulation.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}

// One arrival (release at CTA scope) on a barrier that counts thread arrivals.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bulk (TMA, non-tensor) copy global -> shared, completing on an mbarrier.
// dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same buffer.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Wait for a phase, letting the hardware suspend the thread (up to `hint_ns`
// per try) instead of spinning: true when complete.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase: true when complete, false once `limit_ns`
// of wall time has passed or `*abort_flag` (if given) became non-zero; the
// caller then records a timeout and stops issuing work.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                                  const volatile int32_t* abort_flag = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (abort_flag && *abort_flag) return false;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// ---------------------------------------------------------------------------
// Unpacking codes into bf16x2 operand registers.
//
// A bf16 with exponent field 0x86 holds 128 + m for a 7-bit integer m in its
// mantissa bits, so OR-ing a small field into the mantissa of 0x4300 gives
// 128 + field exactly; one bf16x2 FMA then removes the 128 (and a signed code's
// offset) and undoes any left shift of the field.  Two's complement fields are
// turned into offset binary by flipping their top bit in the same LOP3.
// ---------------------------------------------------------------------------

// 4-bit fields at bit 4x (low half) and 16 + 4x (high half) -> bf16x2.
template <bool SIGNED>
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int x) {
  const uint32_t v = x ? (w >> (4 * x)) : w;
  const uint32_t r = and_xor(v, 0x000F000Fu, SIGNED ? 0x43084308u : 0x43004300u);
  return bf2_fma(r, bf16x2_of(1.0f), SIGNED ? bf16x2_of(-136.0f) : bf16x2_of(-128.0f));
}

// 2-bit fields at bit 2x and 16 + 2x, x in [0, 8).
template <bool SIGNED>
__device__ __forceinline__ uint32_t crumb_pair(uint32_t w, int x) {
  // fields 0..2 read from w, 3..5 from w >> 6, 6..7 from w >> 12, at local
  // position y (bits 2y..2y+1 of each half, all inside the 7 mantissa bits)
  const int shift = x < 3 ? 0 : (x < 6 ? 6 : 12);
  const int y = x - (x < 3 ? 0 : (x < 6 ? 3 : 6));
  const uint32_t v = shift ? (w >> shift) : w;
  const uint32_t m = 0x00030003u << (2 * y);
  const uint32_t k = 0x43004300u | (SIGNED ? (0x00020002u << (2 * y)) : 0u);
  const uint32_t r = and_xor(v, m, k);
  // r = 128 + 4^y c  ->  c - offset = r / 4^y - 128 / 4^y - offset
  const float off = SIGNED ? 2.0f : 0.0f;
  const uint32_t mul = y == 0 ? bf16x2_of(1.0f) : (y == 1 ? bf16x2_of(0.25f) : bf16x2_of(0.0625f));
  const uint32_t add = y == 0 ? bf16x2_of(-128.0f - off)
                              : (y == 1 ? bf16x2_of(-32.0f - off) : bf16x2_of(-8.0f - off));
  return bf2_fma(r, mul, add);
}

// 8-bit fields at byte x and byte x + 2 (x in {0, 1}) -> bf16x2, built from
// the two nibble planes: code = low nibble (unsigned) + 16 * high nibble.
template <bool SIGNED>
__device__ __forceinline__ uint32_t byte_pair(uint32_t w, int x) {
  const uint32_t vlo = x ? (w >> 8) : w;
  const uint32_t vhi = x ? (w >> 12) : (w >> 4);
  const uint32_t lo = bf2_fma(and_xor(vlo, 0x000F000Fu, 0x43004300u), bf16x2_of(1.0f),
                              bf16x2_of(-128.0f));
  const uint32_t hr = and_xor(vhi, 0x000F000Fu, SIGNED ? 0x43084308u : 0x43004300u);
  const uint32_t hi16 = bf2_fma(hr, bf16x2_of(16.0f), SIGNED ? bf16x2_of(-2176.0f) : bf16x2_of(-2048.0f));
  return bf2_fma(lo, bf16x2_of(1.0f), hi16);
}

// ---------------------------------------------------------------------------
// Unpacking codes into fp16x2 operand registers.
//
// An fp16 with exponent field 25 holds 1024 + m for a 10-bit integer m in its
// mantissa bits, so OR-ing a field that sits anywhere inside the low 10 bits of
// each half into 0x6400 gives 1024 + field * 2^pos exactly; one fp16x2 FMA
// scales by 2^-pos and removes the 1024 (and a signed code's offset).  A
// nibble at bit 4 or a byte at bit 0 therefore needs no shift, which leaves one
// shift per word of nibbles or bytes.  Two's complement fields become offset
// binary by flipping their top bit in the same LOP3.
// ---------------------------------------------------------------------------

// 4-bit fields at bit 4x (low half) and 16 + 4x (high half) -> fp16x2.
template <bool SIGNED>
__device__ __forceinline__ uint32_t nib_pair_h(uint32_t w, int x) {
  const uint32_t v = x >= 2 ? (w >> 8) : w;
  const int y = x & 1;   // field at bit 4y of v
  const uint32_t r = and_xor(v, 0x000F000Fu << (4 * y), 0x64006400u | (SIGNED ? (0x00080008u << (4 * y)) : 0u));
  // r = 1024 + 16^y f', f' the field (top bit flipped when signed)
  return h2_fma(r, y ? f16x2_of(0.0625f) : f16x2_of(1.0f),
                y ? f16x2_of(SIGNED ? -72.0f : -64.0f) : f16x2_of(SIGNED ? -1032.0f : -1024.0f));
}

// 2-bit fields at bit 2x and 16 + 2x, x in [0, 8) -> fp16x2.
template <bool SIGNED>
__device__ __forceinline__ uint32_t crumb_pair_h(uint32_t w, int x) {
  // fields 0..4 read from w, 5..7 from w >> 10, at local position y
  const uint32_t v = x >= 5 ? (w >> 10) : w;
  const int y = x >= 5 ? x - 5 : x;
  const uint32_t m = 0x00030003u << (2 * y);
  const uint32_t k = 0x64006400u | (SIGNED ? (0x00020002u << (2 * y)) : 0u);
  const uint32_t r = and_xor(v, m, k);
  // r = 1024 + 4^y c'  ->  c - offset = r / 4^y - 1024 / 4^y - offset
  const float off = SIGNED ? 2.0f : 0.0f;
  const float inv = y == 0 ? 1.0f : y == 1 ? 0.25f : y == 2 ? 0.0625f : y == 3 ? 0.015625f : 0.00390625f;
  return h2_fma(r, f16x2_of(inv), f16x2_of(-1024.0f * inv - off));
}

// 8-bit fields at byte x and byte x + 2 (x in {0, 1}) -> fp16x2.
template <bool SIGNED>
__device__ __forceinline__ uint32_t byte_pair_h(uint32_t w, int x) {
  const uint32_t v = x ? (w >> 8) : w;
  const uint32_t r = and_xor(v, 0x00FF00FFu, SIGNED ? 0x64806480u : 0x64006400u);
  return h2_fma(r, f16x2_of(1.0f), f16x2_of(SIGNED ? -1152.0f : -1024.0f));
}

// ---------------------------------------------------------------------------
// hi/lo bf16 split of fp32 values for a two-column tensor-core product:
// hi = bf16_rn(x), lo = bf16_rn(x - hi); hi + lo carries x with relative error
// <= 2^-16.  Returns the pair (x0, x1) as packed hi parts, or as packed lo
// parts when `lo` is set.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t split_pack(float x0, float x1, bool lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);   // .x = x0 (low half)
  const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
  const float h0 = __uint_as_float(hb << 16);
  const float h1 = __uint_as_float(hb & 0xFFFF0000u);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - h0, x1 - h1);
  const uint32_t lb = *reinterpret_cast<const uint32_t*>(&l);
  return lo ? lb : hb;
}

// ---------------------------------------------------------------------------
// The quantizer (IEEE fp32 division, round half to even, stored scale).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float stored_value(float s, int scale_fp32) {
  if (scale_fp32) return s;
  float r = __half2float(__float2half_rn(s));
  if (isinf(r)) r = r > 0.0f ? 65504.0f : -65504.0f;
  return r;
}

__device__ __forceinline__ int quant_sym(float x, float sh, int Q) {
  if (sh == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(x, sh));
  return q < -Q ? -Q : (q > Q ? Q : q);
}

__device__ __forceinline__ int quant_asym(float x, float sh, float zh, int Qa) {
  if (sh == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(__fsub_rn(x, zh), sh));
  return q < 0 ? 0 : (q > Qa ? Qa : q);
}

// The same codes through a multiply by inv = RN(1 / sh) (__frcp_rn, once per
// scale).  y = fl(x * inv) is within (2^-23 + 2^-24) |x / sh| of the IEEE
// quotient fl(x / sh) (each of the reciprocal, the product and the quotient
// is one rounding, relative error <= 2^-24).  For |y| < 256 that is below
// 2^-13.4, so when y lies farther than 2^-13 from the half-integer between
// its two neighbouring integers, y and fl(x / sh) round to the same integer;
// |y| >= 256 clips to +-Q either way (Q <= 255).  Only the rare y near a
// half-integer, a zero scale, or a non-finite product (NaN, or an infinite
// reciprocal of a tiny fp32 scale) takes the exact division.
// The exact fallbacks of the fast quantizers below, out of line so that the
// rare call stays a branch instead of being computed for every element.
static __device__ __noinline__ int quant_sym_exact(float x, float sh, int Q) { return quant_sym(x, sh, Q); }
static __device__ __noinline__ int quant_asym_exact(float x, float sh, float zh, int Qa) { return quant_asym(x, sh, zh, Qa); }

__device__ __forceinline__ int quant_sym_fast(float x, float sh, float inv, int Q) {
  const float y = x * inv;
  const float ay = fabsf(y);
  if (ay >= 256.0f) return y > 0.0f ? Q : -Q;   // infinite y included
  const float f = y - floorf(y);                 // exact for |y| < 2^23
  if (sh != 0.0f && fabsf(f - 0.5f) > 0.0001220703125f) {
    const int q = __float2int_rn(y);
    return q < -Q ? -Q : (q > Q ? Q : q);
  }
  return quant_sym_exact(x, sh, Q);
}

__device__ __forceinline__ int quant_asym_fast(float x, float sh, float inv, float zh, int Qa) {
  const float y = __fsub_rn(x, zh) * inv;
  const float ay = fabsf(y);
  if (ay >= 256.0f) return y > 0.0f ? Qa : 0;
  const float f = y - floorf(y);
  if (sh != 0.0f && fabsf(f - 0.5f) > 0.0001220703125f) {
    const int q = __float2int_rn(y);
    return q < 0 ? 0 : (q > Qa ? Qa : q);
  }
  return quant_asym_exact(x, sh, zh, Qa);
}

// Branch-free form of the fast quantizers for bulk work: the code of y =
// x * inv (or (x - zh) * inv) clipped to [lo, hi], and `tie` set when y lies
// within 2^-13 of a half-integer, or is NaN or infinite -- then the caller
// must take quant_sym / quant_asym instead (exact, and rare).  For |y| < 256
// the fast code is right whenever `tie` is clear; beyond, the code clips
// either way.  With a zero scale inv is 0, so y = 0 and the code 0 (the exact
// quantizer's zero group) for every finite x.
__device__ __forceinline__ int quant_code_nb(float y, int lo, int hi, bool& tie) {
  const float r = rintf(y);
  tie = !(fabsf(y - r) <= 0.4998779296875f);   // 0.5 - 2^-13; NaN and inf included
  const int q = __float2int_rn(r);
  return q < lo ? lo : (q > hi ? hi : q);
}

// RN(1 / sh) for the fast quantizers (0 for a zero scale: those codes are 0).
__device__ __forceinline__ float quant_inv(float sh) { return sh != 0.0f ? __frcp_rn(sh) : 0.0f; }

__device__ __forceinline__ void store_meta(uint8_t* p, float v, int scale_fp32) {
  if (scale_fp32) *reinterpret_cast<float*>(p) = v;
  else *reinterpret_cast<uint16_t*>(p) = __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ float load_meta(const uint8_t* p, int scale_fp32) {
  if (scale_fp32) return *reinterpret_cast<const float*>(p);
  return __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(p)));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(uint32_t(b) << 16);
}

}  // namespace kvq
