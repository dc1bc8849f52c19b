// kvq_prefill_tc.cu -- chunked-prefill attention of the INT4 KIVI format (keys
// per channel G = 64, values per token G = 64, fp16 scales, page 16, BF16
// window 64, 4 query heads per kv head) on the fifth-generation tensor cores:
// tcgen05.mma with operands in shared and tensor memory, accumulators in tensor
// memory.
//
// The attention is that of kvq_decode_attn for every query token of a chunk
// over its causal prefix (oh-bug.com "KV Cache Quantization in Practice",
// "Go-Live Checklist"; llmdaily.org day-65, "Why the KV cache grows so
// quickly").  Many query tokens of one sequence make it a dense contraction:
//
//  * A CTA (four warps, 128 threads) takes one task of the prefill plan: a
//    block of up to 32 query tokens of one sequence, one kv head and a range
//    of key units.  Its 128 rows (token-major, the kv head's 4 query heads
//    per token) are the mma M dimension; thread r owns row r, which is also
//    tensor-memory lane r.
//  * Q, scaled per row by a power of two into fp16 range, is the A tile, its
//    columns in key-list order (the order the key codes are stored in).  Each
//    64-token unit is dequantized once: K^ = s (c - 8) is not exact in fp16,
//    so it goes to two B tiles, hi = f16(K^) and lo = f16(K^ - hi), and the
//    scores are Q K^hi^T + Q K^lo^T (16 products of K = 16 into 64 fp32
//    columns of tensor memory).  Values become one fp16 tile V^T (rounding a
//    value element moves the output by 2^-12 of it at most, below the
//    attention tolerance).
//  * Each thread reads its row of scores from tensor memory, masks it
//    causally, and takes an online-softmax step whose running max only moves
//    when a score passes it by more than 8 (log2): p = 2^(s - m) <= 256 stays
//    in fp16, and the accumulator in tensor memory is rescaled only then.
//    P (fp16) replaces the scores in tensor memory and O += P V^ is 4 more
//    products (A from tensor memory) into 128 columns.  BF16 window tiles (16
//    tokens) take the same path with N = 16.
//  * The score block is double-buffered in tensor memory, so the products
//    overlap the CUDA-core work: an item's scores run while its values are
//    dequantized, its P V while the next item's keys are.
//  * Thread 0 stages units and window tiles with cp.async.bulk into a
//    2-stage ring and issues the tensor-core products; tcgen05.commit
//    signals their completion on mbarriers.  Every wait is bounded (an error
//    bit, then the CTA drains and leaves); the tensor memory is freed on
//    every exit path.
//  * With one split the CTA writes the output; with several it writes (o, m,
//    l) records that prefill_merge_kernel combines, as the mma.sync kernel's;
//    the merge is a programmatic dependent launch, scheduled once every CTA
//    has left its item loop.
//
// Shared-memory tiles use the 128-byte swizzle of the tensor-core operand
// descriptors: a tile is 8-row groups of 128-byte rows (64 fp16 along K),
// the 16-byte chunk j of row r stored at chunk j ^ (r mod 8); K beyond 64
// takes a second such block.
#include <algorithm>
#include <cstdint>

#include "kvq_device.cuh"

namespace kvq {
namespace {

// Geometry of the format (the host checks it field by field).
constexpr int kTcChunk = 2176;          // bytes per (page, head): K codes | V codes | V scales | K-scale slice
constexpr int kTcOffV = 1024, kTcOffVm = 2048, kTcOffKm = 2112;
constexpr int kTcKslice = 32;           // key-list positions whose scales a page holds
constexpr int kTcThreads = 128;
constexpr int kTcRows = 128;            // 32 query tokens x 4 heads
constexpr int kTcStages = 2;
constexpr int kTcStageBytes = 4 * kTcChunk;   // >= a window tile's 2 x 4096 bytes
constexpr uint64_t kTcWaitNs = 2000000000ull;
constexpr int kTcCols = 256;            // tensor-memory columns: O at 0, two score blocks at 128 and 192
constexpr int kTcColO = 0;
constexpr int kTcColS = 128;

struct TcSmem {
  int q, kh, kl, vt, stages, blk, bars, misc, total;
};

__host__ __device__ constexpr TcSmem tc_smem() {
  TcSmem L{};
  L.q = 0;                                  // A: [2 K-blocks][128 rows][128 B]
  L.kh = L.q + 2 * kTcRows * 128;           // B: [2][64 rows][128 B], hi parts
  L.kl = L.kh + 2 * 64 * 128;               // lo parts
  L.vt = L.kl + 2 * 64 * 128;               // B of P V: [128 rows (channels)][128 B (64 tokens)]
  L.stages = L.vt + kD * 128;
  L.blk = L.stages + kTcStages * kTcStageBytes;
  L.bars = L.blk + kPrefillMaxPages * 4;    // stage barriers, then S and O barriers
  L.misc = L.bars + (kTcStages + 2) * 8;    // tensor-memory base, abort flag
  L.total = L.misc + 16;
  return L;
}

// ---- tcgen05 wrappers (one instruction each, from the PTX ISA) ------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// D[tmem] (+)= A[smem] B[smem]^T, fp16 inputs, fp32 accumulate; accumulate
// when `acc` is set, else overwrite.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// D[tmem] (+)= A[tmem] B[smem]^T: A's rows are the tensor-memory lanes, two
// fp16 elements of K per 32-bit column (the lower K index in the low half).
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// Arrive on an mbarrier once every earlier tcgen05.mma of this thread is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
// This warp's 32 lanes x 32 consecutive columns: v[i] = column col + i of the
// thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
  tmem_st32(taddr, f);
}

// Shared-memory operand descriptor of a K-major tile with the 128-byte
// swizzle: start address (16-byte units), leading offset 1 (unused by this
// layout), stride offset 1024 bytes (one 8-row group), version 1, layout 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) |
         (uint64_t(2) << 61);
}
// Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, M x N.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N) {
  return (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
// Byte offset of 16-byte chunk `ch` (0..7) of row r inside a swizzled block.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch) { return uint32_t(r * 128 + ((ch ^ (r & 7)) << 4)); }


__global__ void __launch_bounds__(kTcThreads, 2) prefill_tc_kernel(const __grid_constant__ PrefillArgs a) {
  constexpr int D = kD;
  constexpr TcSmem L = tc_smem();
  const Geo& g = a.g;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles want 1024-byte alignment (the launch adds that slack)
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_addr(smem);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t bar_st = sb + L.bars, bar_s = bar_st + 8 * kTcStages, bar_o = bar_s + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int32_t* abort_flag = reinterpret_cast<int32_t*>(smem + L.misc + 4);
  int32_t* sblk = reinterpret_cast<int32_t*>(smem + L.blk);

  // ---- once per CTA: barriers, tensor memory ------------------------------------
  if (tid == 0) {
    for (int b = 0; b < kTcStages + 2; ++b) mbar_init(bar_st + 8 * b, 1);
    mbar_init_fence();
    *abort_flag = 0;
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), kTcCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t trow_addr = tmem + (uint32_t(warp * 32) << 16);   // this warp's 32 lanes

  // ---- the task: a block of query tokens, a kv head, a range of key units ----
  const int32_t* task = a.plan + a.off_tasks + 5 * blockIdx.x;
  const int bi = task[0], h = task[1], split = task[2], u0 = task[3], u1 = task[4];
  const int32_t* binfo = a.plan + a.off_blocks + 4 * bi;
  const int seq = binfo[0], nrow = binfo[2], Lq = binfo[3];
  const int32_t* rows = a.plan + a.off_rows + 2 * binfo[1];   // (row, position), positions ascending
  const int bmax = rows[2 * (nrow - 1) + 1];
  const int qa = min(bmax + 1, Lq);
  const int nu = u1 - u0;
  const int nw = split == a.splits - 1 ? (max(0, bmax + 1 - Lq) + 15) >> 4 : 0;
  const int K = nu + nw;
  const int tok = tid >> 2, hd = tid & 3;              // this thread's row: token tok of the block, head hd
  const int pos = tok < nrow ? rows[2 * tok + 1] : -1;

  // ---- setup: block ids, Q --------------------------------------------------------
  const int page0 = u0 * 4;                            // 4 pages per 64-token unit
  const int qg = ((qa + 63) >> 6) << 6;                // every page of each key group touched
  const int npages = min(nu * 4, (qg >> 4) - page0);
  const int32_t* trow = a.table + int64_t(seq) * a.table_stride;
  for (int i = tid; i < npages; i += kTcThreads) sblk[i] = trow[page0 + i];
  float cs;   // the row's score scale (log2 domain, with its power of two)
  {
    uint32_t qw[64];
    if (tok < nrow) {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + (int64_t(rows[2 * tok]) * g.h_q + h * 4 + hd) * D);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = src[c];
        qw[4 * c] = v.x; qw[4 * c + 1] = v.y; qw[4 * c + 2] = v.z; qw[4 * c + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) qw[c] = 0u;
    }
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 64; ++c)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(qw[c] << 16)), fabsf(__uint_as_float(qw[c] & 0xFFFF0000u))));
    // 2^-ex puts the row's max |q| in [1/2, 1): every element lands in fp16 range
    const int ex = amax > 0.0f ? min(max(int((__float_as_uint(amax) >> 23) & 0xFF) - 126, -100), 100) : 0;
    const float down = __uint_as_float(uint32_t(127 - ex) << 23);
    cs = a.qk_scale * __uint_as_float(uint32_t(127 + ex) << 23);
    // chunk c holds key-list positions 8c .. 8c + 7: channels 16 j + 2 t + {0, 1, 8, 9}
    // for j = 2 (c mod 4) + {0, 1}, t = c / 4 (u32 pairs 8 j + t and 8 j + t + 4)
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      uint32_t hw[4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int j = 2 * (c & 3) + jj;
        const uint32_t w01 = qw[8 * j + (c >> 2)], w89 = qw[8 * j + (c >> 2) + 4];
        const __half2 x = __floats2half2_rn(__uint_as_float(w01 << 16) * down, __uint_as_float(w01 & 0xFFFF0000u) * down);
        const __half2 y = __floats2half2_rn(__uint_as_float(w89 << 16) * down, __uint_as_float(w89 & 0xFFFF0000u) * down);
        hw[2 * jj] = *reinterpret_cast<const uint32_t*>(&x);
        hw[2 * jj + 1] = *reinterpret_cast<const uint32_t*>(&y);
      }
      *reinterpret_cast<uint4*>(smem + L.q + (c >> 3) * (kTcRows * 128) + sw128_off(tid, c & 7)) =
          make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- staging (thread 0) ---------------------------------------------------------
  int issued = 0;
  auto issue = [&](int k) {
    ++issued;
    const int sidx = k % kTcStages;
    const uint32_t dst = sb + L.stages + sidx * kTcStageBytes, bar = bar_st + 8 * sidx;
    fence_proxy_async();   // earlier generic reads of the stage come before the copies
    if (k < nu) {
      bool bad = false;
      for (int p = 0; p < 4; ++p) {
        const int32_t b = sblk[k * 4 + p];
        bad |= b < 0 || b >= g.num_blocks;
      }
      if (bad) {
        atomicOr(a.err, KVQ_DEVERR_BLOCK_ID);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      mbar_arrive_expect_tx(bar, 4 * kTcChunk);
      for (int p = 0; p < 4; ++p)
        bulk_g2s(dst + p * kTcChunk, a.pool + int64_t(sblk[k * 4 + p]) * g.block_bytes + int64_t(h) * g.chunk_bytes,
                 kTcChunk, bar);
    } else {
      const int64_t base = ((int64_t(seq) * g.h_kv + h) * g.R + 16 * (k - nu)) * D;
      mbar_arrive_expect_tx(bar, 2 * 16 * D * 2);
      bulk_g2s(dst, a.kres + base, 16 * D * 2, bar);
      bulk_g2s(dst + 16 * D * 2, a.vres + base, 16 * D * 2, bar);
    }
  };
  if (tid == 0)
    for (int k = 0; k < K && k < kTcStages; ++k) issue(k);

  // ---- items: quantized units, then window tiles -------------------------------------
  float m_run = -INFINITY, l_run = 0.0f;
  int consumed = 0, s_commits = 0, o_commits = 0;   // consumed: this thread's completed stage waits
  bool aborted = false;
  auto raise_abort = [&]() {
    atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
    *abort_flag = 1;
  };
  for (int k = 0; k < K; ++k) {
    const int sidx = k % kTcStages;
    // A wait that gives up raises the abort flag and carries on; the CTA
    // leaves together at the next barrier (steps 1 and 4 end in one).
    if (mbar_wait_bounded(bar_st + 8 * sidx, uint32_t((k / kTcStages) & 1), kTcWaitNs, abort_flag)) ++consumed;
    else raise_abort();
    const uint8_t* stg = smem + L.stages + sidx * kTcStageBytes;
    const bool quant = k < nu;
    const int T0 = quant ? (u0 + k) * 64 : Lq + 16 * (k - nu);   // position of the item's first key
    const int nt = quant ? 64 : 16;                               // its keys (N of the score product)
    const uint32_t s_col = kTcColS + uint32_t(k & 1) * 64;       // its scores, then its P

    // 1. keys: K^ hi and lo tiles [keys][key-list positions] (their last
    //    reader, the previous item's score product, was waited for)
    if (quant) {
      const int w = tid & 15;   // word w of a key row: positions 8w .. 8w + 7, scales on page w / 4
      const uint4 sr = *reinterpret_cast<const uint4*>(stg + (w >> 2) * kTcChunk + kTcOffKm + ((8 * w) & 31) * 2);
      const uint32_t sw[4] = {sr.x, sr.y, sr.z, sr.w};   // scale pairs of elements (2e, 2e + 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = (tid >> 4) + 8 * i;   // key 0..63 of the unit: page t / 16, row t % 16
        const uint32_t word = *reinterpret_cast<const uint32_t*>(stg + (t >> 4) * kTcChunk + (t & 15) * 64 + 4 * w);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // elements 2e, 2e + 1 of the word sit at bit 4e of each half: the
          // two's complement nibble with its top bit flipped, OR-ed into the
          // mantissa of 1024, is 1032 + c exactly; then hi = f16(c s) and lo =
          // f16(c s - hi) (the FMA's residual is exact)
          const uint32_t r = and_xor(e ? (word >> (4 * e)) : word, 0x000F000Fu, 0x64086408u);
          const __half2 c2 = __hsub2(*reinterpret_cast<const __half2*>(&r), __float2half2_rn(1032.0f));
          const __half2 s2 = *reinterpret_cast<const __half2*>(&sw[e]);
          const __half2 hh = __hmul2(c2, s2);
          const __half2 ll = __hfma2(c2, s2, __hneg2(hh));
          hi[e] = *reinterpret_cast<const uint32_t*>(&hh);
          lo[e] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        const uint32_t off = (w >> 3) * (64 * 128) + sw128_off(t, w & 7);
        *reinterpret_cast<uint4*>(smem + L.kh + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(smem + L.kl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    } else {
      // a window tile: 16 natural bf16 key rows; (key t, chunk c) per item
#pragma unroll
      for (int it2 = 0; it2 < 2; ++it2) {
        const int it = tid + kTcThreads * it2, t = it >> 4, c = it & 15;
        const uint32_t* kr = reinterpret_cast<const uint32_t*>(stg + t * D * 2);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * (c & 3) + jj;
          const uint32_t pr[2] = {kr[8 * j + (c >> 2)], kr[8 * j + (c >> 2) + 4]};
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float x0 = __uint_as_float(pr[u] << 16), x1 = __uint_as_float(pr[u] & 0xFFFF0000u);
            const __half2 hh = __floats2half2_rn(x0, x1);
            const float2 hf = __half22float2(hh);
            const __half2 ll = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
            hi[2 * jj + u] = *reinterpret_cast<const uint32_t*>(&hh);
            lo[2 * jj + u] = *reinterpret_cast<const uint32_t*>(&ll);
          }
        }
        const uint32_t off = (c >> 3) * (64 * 128) + sw128_off(t, c & 7);
        *reinterpret_cast<uint4*>(smem + L.kh + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(smem + L.kl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    fence_proxy_async();   // the tiles' generic writes before the tensor core's reads
    tc_fence_before();
    if (__syncthreads_or(*abort_flag != 0)) {
      aborted = true;
      break;
    }
    // 2. the scores S = Q K^T into this item's column block; they run while
    //    the values are dequantized
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = tc_idesc(kTcRows, nt);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t bt = sb + (part ? L.kl : L.kh);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {   // K = 128 positions in steps of 16 (32 bytes)
          const uint32_t oa = (ks >> 2) * (kTcRows * 128) + (ks & 3) * 32;
          const uint32_t ob = (ks >> 2) * (64 * 128) + (ks & 3) * 32;
          tc_mma_f16(tmem + s_col, sw128_desc(sb + L.q + oa), sw128_desc(bt + ob), idesc, (part | ks) != 0);
        }
      }
      tc_commit(bar_s);
    }
    ++s_commits;
    // 3. values: V^T tile [channels][keys], once the previous item's P V
    //    product (their last reader) is done
    if (k > 0 && !mbar_wait_bounded(bar_o, uint32_t((k - 1) & 1), kTcWaitNs, abort_flag)) raise_abort();
    if (quant) {
      // lane record (sub-tile st, lane gq * 4 + tq): word i holds channel tile i,
      // register x (x = 0..3) the channel 16 i + gq + 8 (x % 2) for keys
      // 2 tq + 8 (x / 2) and + 1 (fields x and x + 4)
      const int st = tid >> 5, lam = tid & 31, gq = lam >> 2, tq = lam & 3;
      const uint8_t* page = stg + st * kTcChunk;
      const uint4 va = reinterpret_cast<const uint4*>(page + kTcOffV + 32 * lam)[0];
      const uint4 vb = reinterpret_cast<const uint4*>(page + kTcOffV + 32 * lam)[1];
      const uint32_t vw[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
      // scales [key][group]: keys 2tq, 2tq + 1 and 2tq + 8, 2tq + 9 of the page
      const uint16_t* vm = reinterpret_cast<const uint16_t*>(page + kTcOffVm);
      const uint2 sa = *reinterpret_cast<const uint2*>(vm + 4 * tq), sbv = *reinterpret_cast<const uint2*>(vm + 4 * tq + 16);
      // scale pairs (key t, key t + 1) of group gv for keys 2tq (+ 8 when hi8)
      uint32_t sp[2][2];
#pragma unroll
      for (int gv = 0; gv < 2; ++gv) {
        const uint32_t sel = gv ? 0x7632u : 0x5410u;
        sp[0][gv] = __byte_perm(sa.x, sa.y, sel);
        sp[1][gv] = __byte_perm(sbv.x, sbv.y, sel);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int gv = i >> 2;   // value group of channel tile i (64 channels each)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int d = 16 * i + gq + 8 * (x & 1);
          const int t = 16 * st + 2 * tq + 8 * (x >> 1);
          // fields x and x + 4: keys t and t + 1 of channel d, as 1032 + c in fp16
          const uint32_t r = and_xor(x ? (vw[i] >> (4 * x)) : vw[i], 0x000F000Fu, 0x64086408u);
          const __half2 c2 = __hsub2(*reinterpret_cast<const __half2*>(&r), __float2half2_rn(1032.0f));
          const __half2 pv = __hmul2(c2, *reinterpret_cast<const __half2*>(&sp[x >> 1][gv]));
          *reinterpret_cast<uint32_t*>(smem + L.vt + sw128_off(d, t >> 3) + (t & 7) * 2) =
              *reinterpret_cast<const uint32_t*>(&pv);
        }
      }
    } else {
      // window values: channel tid of the 16 natural bf16 rows
      const uint16_t* vr = reinterpret_cast<const uint16_t*>(stg + 16 * D * 2);
#pragma unroll
      for (int t = 0; t < 16; t += 2) {
        const __half2 pv = __floats2half2_rn(__uint_as_float(uint32_t(vr[t * D + tid]) << 16),
                                             __uint_as_float(uint32_t(vr[(t + 1) * D + tid]) << 16));
        *reinterpret_cast<uint32_t*>(smem + L.vt + sw128_off(tid, t >> 3) + (t & 7) * 2) =
            *reinterpret_cast<const uint32_t*>(&pv);
      }
    }
    // 4. this row's scores, masked causally; online softmax with a lazy max
    if (!mbar_wait_bounded(bar_s, uint32_t(k & 1), kTcWaitNs, abort_flag)) raise_abort();
    tc_fence_after();
    float sv[64];
    {
      float h32[32];
      tmem_ld32(trow_addr + s_col, h32);
#pragma unroll
      for (int j = 0; j < 32; ++j) sv[j] = h32[j];
      if (nt == 64) {
        tmem_ld32(trow_addr + s_col + 32, h32);
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[32 + j] = h32[j];
      } else {
#pragma unroll
        for (int j = 32; j < 64; ++j) sv[j] = 0.0f;
      }
    }
    // raw scores; the row scale cs > 0 goes into the exponent's FMA below.
    // A unit wholly before every position of the warp's rows needs no mask.
    float mx = -INFINITY;
    if (__all_sync(0xffffffffu, nt == 64 && T0 + 63 <= pos)) {
#pragma unroll
      for (int j = 0; j < 64; ++j) mx = fmaxf(mx, sv[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        sv[j] = (j < nt && T0 + j <= pos) ? sv[j] : -INFINITY;
        mx = fmaxf(mx, sv[j]);
      }
    }
    mx = mx == -INFINITY ? mx : mx * cs;
    const bool raise = mx > m_run + 8.0f || (m_run == -INFINITY && mx != -INFINITY);
    float alpha = 1.0f;
    if (raise) {
      alpha = m_run == -INFINITY ? 0.0f : fast_exp2(m_run - mx);
      l_run *= alpha;
      m_run = mx;
    }
    if (k > 0 && __any_sync(0xffffffffu, raise)) {
      // rescale the accumulator rows of this warp (complete: the previous P V was waited for)
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float ov[32];
        tmem_ld32(trow_addr + kTcColO + 32 * c4, ov);
#pragma unroll
        for (int j = 0; j < 32; ++j) ov[j] *= alpha;
        tmem_st32(trow_addr + kTcColO + 32 * c4, ov);
      }
    }
    {
      // p = 2^(s cs - m): a masked score is -inf and gives 0 (as does a row
      // with nothing attended, m = -inf, whose scores are all -inf); l sums
      // the fp32 p (its fp16 rounding moves the sum by 2^-12 at most).  P
      // (fp16 pairs, key 2c in the low half of column c) replaces the scores
      // in tensor memory, the A operand of the P V product.
      uint32_t pw[32];
      const float nm = m_run == -INFINITY ? 0.0f : -m_run;
      float lsum = 0.0f;
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const float p0 = fast_exp2(fmaf(sv[j], cs, nm));
        const float p1 = fast_exp2(fmaf(sv[j + 1], cs, nm));
        const __half2 ph = __floats2half2_rn(p0, p1);
        lsum += p0 + p1;
        pw[j >> 1] = *reinterpret_cast<const uint32_t*>(&ph);
      }
      l_run += lsum;
      tmem_st32u(trow_addr + s_col, pw);
    }
    fence_proxy_async();   // the V^T tile's generic writes before the tensor core's reads
    tc_fence_before();
    if (__syncthreads_or(*abort_flag != 0)) {
      aborted = true;
      break;
    }
    // 5. the stage is consumed: its next item; O += P V^ (the item's keys in
    //    steps of 16, P from tensor memory); it runs while the next keys are
    //    dequantized
    if (tid == 0) {
      if (k + kTcStages < K) issue(k + kTcStages);
      tc_fence_after();
      const uint32_t idesc = tc_idesc(kTcRows, D);
      for (int ks = 0; ks < nt / 16; ++ks)
        tc_mma_f16_ts(tmem + kTcColO, tmem + s_col + 8 * ks, sw128_desc(sb + L.vt + ks * 32), idesc,
                      (k > 0 || ks > 0) ? 1u : 0u);
      tc_commit(bar_o);
    }
    ++o_commits;
  }

  // the merge grid may be scheduled now (it waits on the device for this grid)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  if (aborted) {
    // bounded: the copies in flight land, the committed products finish
    if (tid == 0)
      for (int j = consumed; j < issued; ++j)
        (void)mbar_wait_bounded(bar_st + 8 * (j % kTcStages), uint32_t((j / kTcStages) & 1), kTcWaitNs);
    if (s_commits > 0) (void)mbar_wait_bounded(bar_s, uint32_t((s_commits - 1) & 1), kTcWaitNs);
    if (o_commits > 0) (void)mbar_wait_bounded(bar_o, uint32_t((o_commits - 1) & 1), kTcWaitNs);
  } else if (K > 0) {
    const bool oko = mbar_wait_bounded(bar_o, uint32_t((K - 1) & 1), kTcWaitNs);
    if (!oko && tid == 0) atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
    tc_fence_after();
    float o[128];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      float ov[32];
      tmem_ld32(trow_addr + kTcColO + 32 * c4, ov);
#pragma unroll
      for (int j = 0; j < 32; ++j) o[32 * c4 + j] = ov[j];
    }
    if (tok < nrow) {
      const int64_t row = int64_t(rows[2 * tok]) * g.h_q + h * 4 + hd;
      if (a.splits == 1) {
        const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
        float4* dst = reinterpret_cast<float4*>(a.out + row * D);
#pragma unroll
        for (int c = 0; c < 32; ++c) dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
      } else {
        float* rec = a.part + (row * a.splits + split) * (D + 2);
        float2* dst = reinterpret_cast<float2*>(rec);
#pragma unroll
        for (int c = 0; c < 64; ++c) dst[c] = make_float2(o[2 * c], o[2 * c + 1]);
        rec[D] = m_run;
        rec[D + 1] = l_run;
      }
    }
  } else if (tok < nrow) {
    // nothing attended in this split
    const int64_t row = int64_t(rows[2 * tok]) * g.h_q + h * 4 + hd;
    if (a.splits == 1) {
      for (int c = 0; c < D; ++c) a.out[row * D + c] = 0.0f;
    } else {
      float* rec = a.part + (row * a.splits + split) * (D + 2);
      for (int c = 0; c < D; ++c) rec[c] = 0.0f;
      rec[D] = -INFINITY;
      rec[D + 1] = 0.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTcCols);
}

}  // namespace

// The tensor-core prefill covers the INT4 KIVI geometry with 4 query heads
// per kv head exactly (field by field).
bool prefill_tc_supported(const Geo& g) {
  return g.bits == 4 && g.asym == 0 && g.k_axis == 1 && g.g_k == 64 && g.g_v == 64 && g.scale_fp32 == 0 &&
         g.R == 64 && g.P == 16 && g.G == 4 && !g.fp8 && g.chunk_used == kTcChunk && g.off_V == kTcOffV &&
         g.off_Vm == kTcOffVm && g.off_Km == kTcOffKm && g.kslice == kTcKslice && g.row_bytes == 64;
}

size_t prefill_tc_smem_bytes() { return size_t(tc_smem().total) + 1024; }

int prefill_tc_stage_bytes() { return kTcStageBytes; }

// Resident CTAs per SM from the kernel's own resources: shared memory (with the
// per-CTA reservation), registers (allocated per warp in units of 256), and
// tensor memory (512 columns per SM, kTcCols per CTA).  The occupancy API
// reports one CTA for this kernel where its resources allow two.
int prefill_tc_ctas_per_sm() {
  int dev = 0, per_sm = 0, reserved = 0, regs_sm = 0;
  cudaFuncAttributes fa{};
  if (cudaGetDevice(&dev) != cudaSuccess || cudaFuncGetAttributes(&fa, prefill_tc_kernel) != cudaSuccess ||
      cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess)
    return 1;
  const int by_smem = per_sm / (int(prefill_tc_smem_bytes()) + reserved);
  const int warp_regs = (fa.numRegs * 32 + 255) / 256 * 256;
  const int by_regs = regs_sm / (warp_regs * (kTcThreads / 32));
  const int n = std::min(std::min(by_smem, by_regs), 512 / kTcCols);
  return n > 0 ? n : 1;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches) {
  const int smem = int(prefill_tc_smem_bytes());
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = raise_smem_limit(dev, reinterpret_cast<const void*>(&prefill_tc_kernel), size_t(smem));
  if (e != cudaSuccess) return e;
  prefill_tc_kernel<<<a.n_tasks, kTcThreads, smem, s>>>(a);
  ++*launches;
  e = cudaGetLastError();
  if (e != cudaSuccess || a.splits == 1) return e;
  return launch_prefill_merge(a, n_rows, s, launches);
}

}  // namespace kvq
