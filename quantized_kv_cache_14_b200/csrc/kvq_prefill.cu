// kvq_prefill.cu -- chunked-prefill attention over the packed cache, with
// every staged tile shared by a block of query rows.
//
// kvq_prefill_attn gives each query token of a chunk the attention of
// kvq_decode_attn over its causal prefix (oh-bug.com "KV Cache Quantization in
// Practice", "Go-Live Checklist": a quantized cache has to keep serving
// chunked prefill; llmdaily.org day-65, "Why the KV cache grows so quickly",
// for the attention itself).  Several query tokens of one sequence make the
// work a small dense contraction, so here the rows take the mma M dimension
// (flash-attention style) instead of the columns as in decode:
//
//  * A CTA is four warps over one (block of query tokens, kv head, split of
//    the key range).  Warp w owns 16 rows: 16 / g query tokens x the g query
//    heads of the kv head.  All four warps consume the same staged tiles, so
//    a tile is read from memory once for up to 64 rows.
//  * Thread 0 stages whole page chunks of units (whole key groups, 64 tokens
//    or one group when longer) and 16-row tiles of the BF16 window with
//    cp.async.bulk into a 2-stage ring that completes on mbarriers; the CTA
//    frees a stage with one barrier per item.  The task's block ids are read
//    into shared memory once.  Up to three CTAs (12 warps) fit on an SM (two
//    with 128-token units): the context is mostly in L2, so more warps hide
//    latency better than a deeper ring would.
//  * Scores S = Q' C^T: the codes C are exact small integers in fp16 (the B
//    operand, from the packed words exactly as in decode) and Q' = q s_key of
//    the key group, split into fp16 hi + lo parts kept in shared memory and
//    read per k-step with ldmatrix (two A operands).  Each row's q is first
//    scaled by a power of two (max |q| in [1/2, 1)) so that Q' stays inside
//    the fp16 range; the power goes back into the row's score scale.  Window
//    tiles multiply q and the bf16 rows directly (exact).
//  * Online softmax per 16-token sub-tile in the log2 domain with the exact
//    running max (p <= 1); P' = p s_value of each value group as fp16 hi + lo
//    A operands against the value codes.  Zero-points enter as a per-row key
//    bias and a p-weighted value sum.
//  * A single split writes the output; several splits write (m, l, o)
//    records that prefill_merge_kernel combines by log-sum-exp in split order.
#include <algorithm>
#include <cstdint>

#include "kvq_device.cuh"
#include "kvq_tiles.cuh"

namespace kvq {
namespace {

constexpr int kPfWarps = 4;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfStages = 2;
constexpr uint64_t kPfWaitNs = 2000000000ull;   // give up on a copy after 2 s
constexpr uint32_t kFull = 0xffffffffu;

struct PfSmem {
  int stages, qs, qp, cs, dn, blk, bars, flag, total;
};

__host__ __device__ inline PfSmem pf_smem(int stage_bytes) {
  PfSmem L;
  L.stages = 0;
  L.qs = kPfStages * stage_bytes;                   // bf16 q rows, 16-byte chunks swizzled by row
  L.qp = L.qs + kPfWarps * 16 * kD * 2;             // Q' hi and lo tiles per warp, swizzled likewise
  L.cs = L.qp + kPfWarps * 2 * 16 * kD * 2;         // per-row score scale
  L.dn = L.cs + kPfWarps * 16 * 4;                  // per-row q scaling 2^-e
  L.blk = L.dn + kPfWarps * 16 * 4;                 // the task's block ids
  L.bars = L.blk + kPrefillMaxPages * 4;
  L.flag = L.bars + kPfStages * 8;
  L.total = L.flag + 16;
  return L;
}

// An fp16 pair of q times a pair of key scales: hi = f16(q s), lo = f16(q s -
// hi) (the FMA's residual is exact, so hi + lo = q s unless a part underflows).
__device__ __forceinline__ void qs_split(uint32_t q2, uint32_t s2, uint32_t& hi, uint32_t& lo) {
  const __half2 q = *reinterpret_cast<const __half2*>(&q2);
  const __half2 s = *reinterpret_cast<const __half2*>(&s2);
  const __half2 h = __hmul2(q, s);
  const __half2 l = __hfma2(q, s, __hneg2(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// p' = p s for a pair split as (ph, pl) in fp16: hi = f16(ph s), lo =
// f16(pl s + the exact residual of ph s).
__device__ __forceinline__ void ps_split(uint32_t ph, uint32_t pl, uint32_t s2, uint32_t& hi, uint32_t& lo) {
  const __half2 a = *reinterpret_cast<const __half2*>(&ph), b = *reinterpret_cast<const __half2*>(&pl);
  const __half2 s = *reinterpret_cast<const __half2*>(&s2);
  const __half2 h = __hmul2(a, s);
  const __half2 l = __hfma2(b, s, __hfma2(a, s, __hneg2(h)));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <int BITS, int ASYM>
__global__ void __launch_bounds__(kPfThreads, 3) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  constexpr int D = kD;
  constexpr bool SGN = !ASYM;
  const Geo& g = a.g;
  extern __shared__ __align__(128) uint8_t smem[];
  const PfSmem L = pf_smem(a.stage_bytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;

  const int32_t* task = a.plan + a.off_tasks + 5 * blockIdx.x;
  const int bi = task[0], h = task[1], split = task[2], u0 = task[3], u1 = task[4];
  const int32_t* binfo = a.plan + a.off_blocks + 4 * bi;
  const int seq = binfo[0], nrow = binfo[2], Lq = binfo[3];
  const int32_t* rows = a.plan + a.off_rows + 2 * binfo[1];   // (row, position), positions ascending
  const int G = g.G;
  const int lg_G = G == 4 ? 2 : G == 2 ? 1 : 0;
  const int PW = 16 >> lg_G;                      // query tokens per warp
  const int wt0 = warp * PW;
  const int wn = max(0, min(PW, nrow - wt0));     // this warp's query tokens
  const int bmax = rows[2 * (nrow - 1) + 1];
  const int wmax = wn > 0 ? rows[2 * (wt0 + wn - 1) + 1] : -1;
  const int slot_a = gq >> lg_G, slot_b = (gq + 8) >> lg_G;
  const int pos_a = slot_a < wn ? rows[2 * (wt0 + slot_a) + 1] : -1;
  const int pos_b = slot_b < wn ? rows[2 * (wt0 + slot_b) + 1] : -1;
  const int qa = min(bmax + 1, Lq);               // quantized positions any row attends
  const int nu = u1 - u0;
  const int nw = split == a.splits - 1 ? (max(0, bmax + 1 - Lq) + 15) >> 4 : 0;
  const int K = nu + nw;

  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs) + warp * 16 * D;
  __half* qph = reinterpret_cast<__half*>(smem + L.qp) + warp * 2 * 16 * D;
  __half* qpl = qph + 16 * D;
  float* cs = reinterpret_cast<float*>(smem + L.cs) + warp * 16;
  float* dn = reinterpret_cast<float*>(smem + L.dn) + warp * 16;
  int32_t* sblk = reinterpret_cast<int32_t*>(smem + L.blk);
  volatile int32_t* abort_flag = reinterpret_cast<int32_t*>(smem + L.flag);
  const uint32_t stage0 = smem_addr(smem + L.stages);
  const uint32_t bar0 = smem_addr(smem + L.bars);

  // ---- setup: barriers, block ids, q rows -----------------------------------
  if (tid == 0) {
    for (int s = 0; s < kPfStages; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
    *abort_flag = 0;
  }
  const int ppu = a.sup >> g.lg_P;                // pages per unit
  const int page0 = (u0 << a.lg_sup) >> g.lg_P;
  // every page of each key group touched: a group's key scales are spread over its pages
  const int qg = ((qa + g.g_k - 1) >> g.lg_gk) << g.lg_gk;
  const int npages = min(nu * ppu, (qg >> g.lg_P) - page0);
  const int32_t* trow = a.table + int64_t(seq) * a.table_stride;
  for (int i = tid; i < npages; i += kPfThreads) sblk[i] = trow[page0 + i];
  {
    // lane pair (2r, 2r + 1) loads row r: 64 channels each
    const int r = lane >> 1, half = lane & 1;
    const int slot = r >> lg_G, head = r & (G - 1);
    uint4 v[8];
    if (slot < wn) {
      const uint4* src = reinterpret_cast<const uint4*>(
          a.q + (int64_t(rows[2 * (wt0 + slot)]) * g.h_q + h * G + head) * D + 64 * half);
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = src[c];
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = make_uint4(0, 0, 0, 0);
    }
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
    }
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    // 2^-ex puts max |q| in [1/2, 1)
    const int ex = amax > 0.0f ? min(max(int((__float_as_uint(amax) >> 23) & 0xFF) - 126, -126), 126) : 0;
    const float down = __uint_as_float(uint32_t(127 - ex) << 23);
    if (half == 0) {
      cs[r] = a.qk_scale * __uint_as_float(uint32_t(127 + ex) << 23);
      dn[r] = down;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int ch = 8 * half + c;   // 16-byte chunk of the row
      *reinterpret_cast<uint4*>(qs + r * D + 8 * (ch ^ (r & 7))) = v[c];
    }
  }
  __syncthreads();
  const float cs_a = cs[gq], cs_b = cs[gq + 8];

  // ---- staging ----------------------------------------------------------------
  int issued = 0;   // thread 0: items whose copies are issued
  auto issue = [&](int k) {
    ++issued;
    const int sidx = k % kPfStages;
    const uint32_t dst = stage0 + sidx * a.stage_bytes, bar = bar0 + 8 * sidx;
    fence_proxy_async();   // earlier generic reads of the stage come before the copies
    if (k < nu) {
      const int T0 = (u0 + k) << a.lg_sup;
      const int valid = min(a.sup, qa - T0);
      const int ncopy = ((valid + g.g_k - 1) >> g.lg_gk) << (g.lg_gk - g.lg_P);
      bool bad = false;
      for (int p = 0; p < ncopy; ++p) {
        const int32_t b = sblk[k * ppu + p];
        bad |= b < 0 || b >= g.num_blocks;
      }
      if (bad) {
        atomicOr(a.err, KVQ_DEVERR_BLOCK_ID);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      mbar_arrive_expect_tx(bar, uint32_t(ncopy * g.chunk_used));
      for (int p = 0; p < ncopy; ++p) {
        const uint8_t* chunk = a.pool + int64_t(sblk[k * ppu + p]) * g.block_bytes + int64_t(h) * g.chunk_bytes;
        bulk_g2s(dst + p * g.chunk_used, chunk, uint32_t(g.chunk_used), bar);
      }
    } else {
      const int64_t base = ((int64_t(seq) * g.h_kv + h) * g.R + 16 * (k - nu)) * D;
      mbar_arrive_expect_tx(bar, 2 * 16 * D * 2);
      bulk_g2s(dst, a.kres + base, 16 * D * 2, bar);
      bulk_g2s(dst + 16 * D * 2, a.vres + base, 16 * D * 2, bar);
    }
  };
  if (tid == 0)
    for (int k = 0; k < min(K, kPfStages); ++k) issue(k);

  // ---- per-lane state: rows gq (a) and gq + 8 (b) of the warp ----------------
  float o[16][4];
#pragma unroll
  for (int d = 0; d < 16; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.0f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
  float za[4] = {0.0f, 0.0f, 0.0f, 0.0f}, zb[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // value zero sums per group
  float bias_a = 0.0f, bias_b = 0.0f;
  const int vg_shift = g.g_v == 32 ? 1 : g.g_v == 64 ? 2 : 3;   // channel tiles per value group, log2

  // online softmax over one sub-tile's scores x[4] (row a: x[0..1] tokens
  // 2tq, 2tq+1 and x[2..3] tokens 8+2tq, 9+2tq; row b likewise) -> p in place
  auto softmax = [&](float (&xa)[4], float (&xb)[4]) {
    float ma = fmaxf(fmaxf(xa[0], xa[1]), fmaxf(xa[2], xa[3]));
    float mb = fmaxf(fmaxf(xb[0], xb[1]), fmaxf(xb[2], xb[3]));
    ma = fmaxf(ma, __shfl_xor_sync(kFull, ma, 1));
    ma = fmaxf(ma, __shfl_xor_sync(kFull, ma, 2));
    mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, 1));
    mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, 2));
    if (__any_sync(kFull, ma > m_a || mb > m_b)) {
      const float aa = ma > m_a ? fast_exp2(m_a - ma) : 1.0f;
      const float ab = mb > m_b ? fast_exp2(m_b - mb) : 1.0f;
      m_a = fmaxf(m_a, ma);
      m_b = fmaxf(m_b, mb);
      l_a *= aa;
      l_b *= ab;
#pragma unroll
      for (int d = 0; d < 16; ++d) {
        o[d][0] *= aa; o[d][1] *= aa;
        o[d][2] *= ab; o[d][3] *= ab;
      }
      if (ASYM) {
#pragma unroll
        for (int v = 0; v < 4; ++v) { za[v] *= aa; zb[v] *= ab; }
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      xa[e] = m_a == -INFINITY ? 0.0f : fast_exp2(xa[e] - m_a);
      xb[e] = m_b == -INFINITY ? 0.0f : fast_exp2(xb[e] - m_b);
      l_a += xa[e];
      l_b += xb[e];
    }
  };

  // Q' = q s of key group gi (of the unit in `stg`) for the warp's 16 rows,
  // written as fp16 hi and lo tiles in natural channel order (16-byte chunks
  // swizzled by row, as qs) for ldmatrix.  The lane covers channels 16j + 2tq
  // + {0, 1, 8, 9} of rows gq and gq + 8: the k indices 2tq, 2tq + 1, 2tq + 8,
  // 2tq + 9 of k-step j, whose scales sit at key-row positions 32tq + 4j +
  // {0..3}.  With zero-points, also the rows' key bias.
  auto qprime = [&](const uint8_t* stg, int gi) {
    const int lg_ppg = g.lg_gk - g.lg_P;
    const float dna = dn[gq], dnb = dn[gq + 8];
    const int sw = gq & 7;   // rows gq and gq + 8 share their swizzle
    float da = 0.0f, db = 0.0f;
    auto scaled = [](uint32_t w, float d, float& x0, float& x1) {
      x0 = __uint_as_float(w << 16) * d;
      x1 = __uint_as_float(w & 0xFFFF0000u) * d;
      const __half2 h = __floats2half2_rn(x0, x1);
      return *reinterpret_cast<const uint32_t*>(&h);
    };
    __syncwarp();   // the previous group's tiles are no longer read
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int f = 32 * tq + 4 * j;
      const uint8_t* km = stg + ((gi << lg_ppg) + (f >> g.lg_kslice)) * g.chunk_used + g.off_Km;
      const int off = f & (g.kslice - 1);
      const uint2 s = *reinterpret_cast<const uint2*>(km + 2 * off);
      const int e0 = 8 * ((2 * j) ^ sw) + 2 * tq, e1 = 8 * ((2 * j + 1) ^ sw) + 2 * tq;
      float x[8];
      const uint32_t qa0 = scaled(*reinterpret_cast<const uint32_t*>(qs + gq * D + e0), dna, x[0], x[1]);
      const uint32_t qa1 = scaled(*reinterpret_cast<const uint32_t*>(qs + gq * D + e1), dna, x[2], x[3]);
      const uint32_t qb0 = scaled(*reinterpret_cast<const uint32_t*>(qs + (gq + 8) * D + e0), dnb, x[4], x[5]);
      const uint32_t qb1 = scaled(*reinterpret_cast<const uint32_t*>(qs + (gq + 8) * D + e1), dnb, x[6], x[7]);
      uint32_t hi, lo;
      qs_split(qa0, s.x, hi, lo);
      *reinterpret_cast<uint32_t*>(qph + gq * D + e0) = hi;
      *reinterpret_cast<uint32_t*>(qpl + gq * D + e0) = lo;
      qs_split(qa1, s.y, hi, lo);
      *reinterpret_cast<uint32_t*>(qph + gq * D + e1) = hi;
      *reinterpret_cast<uint32_t*>(qpl + gq * D + e1) = lo;
      qs_split(qb0, s.x, hi, lo);
      *reinterpret_cast<uint32_t*>(qph + (gq + 8) * D + e0) = hi;
      *reinterpret_cast<uint32_t*>(qpl + (gq + 8) * D + e0) = lo;
      qs_split(qb1, s.y, hi, lo);
      *reinterpret_cast<uint32_t*>(qph + (gq + 8) * D + e1) = hi;
      *reinterpret_cast<uint32_t*>(qpl + (gq + 8) * D + e1) = lo;
      if (ASYM) {
        const uint2 z = *reinterpret_cast<const uint2*>(km + 2 * (g.kslice + off));
        const float2 z0 = __half22float2(*reinterpret_cast<const __half2*>(&z.x));
        const float2 z1 = __half22float2(*reinterpret_cast<const __half2*>(&z.y));
        da += x[0] * z0.x + x[1] * z0.y + x[2] * z1.x + x[3] * z1.y;
        db += x[4] * z0.x + x[5] * z0.y + x[6] * z1.x + x[7] * z1.y;
      }
    }
    __syncwarp();   // the tiles are complete before any lane reads them
    if (ASYM) {
      da += __shfl_xor_sync(kFull, da, 1);
      da += __shfl_xor_sync(kFull, da, 2);
      db += __shfl_xor_sync(kFull, db, 1);
      db += __shfl_xor_sync(kFull, db, 2);
      bias_a = cs_a * da;
      bias_b = cs_b * db;
    }
  };

  // one 16-token sub-tile of a quantized unit at token offset tok0 (absolute T)
  auto quant_sub = [&](const uint8_t* stg, int tok0, int T) {
    const uint8_t* cb = stg + (tok0 >> g.lg_P) * g.chunk_used;
    const int us = (tok0 & (g.P - 1)) >> 4;
    uint32_t wa[BITS], wb[BITS];
    load_key_words<BITS>(cb + us * g.sub_bytes, gq, tq, wa, wb);
    // four independent accumulator chains (n-tile x {hi, lo}) keep the mma
    // dependency chains short
    float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float r0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, r1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // ldmatrix row addresses of the Q' tiles: lane L gives row (L & 7) + 8 ((L >> 3) & 1)
    // of chunk 2j + (L >> 4)
    const int lr = (lane & 7) + 8 * ((lane >> 3) & 1), lc = lane >> 4;
    const uint32_t qh_base = smem_addr(qph) + lr * D * 2, ql_base = smem_addr(qpl) + lr * D * 2;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t off = 16 * (((2 * j + lc) ^ (lr & 7)));
      uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
      ldsm_x4(qh_base + off, h0, h1, h2, h3);
      ldsm_x4(ql_base + off, l0, l1, l2, l3);
      uint32_t k0, k1, k2, k3;
      key_frag<BITS, SGN, true>(wa, wb, j, k0, k1, k2, k3);
      mma_f16(s0, h0, h1, h2, h3, k0, k2);
      mma_f16(s1, h0, h1, h2, h3, k1, k3);
      mma_f16(r0, l0, l1, l2, l3, k0, k2);
      mma_f16(r1, l0, l1, l2, l3, k1, k3);
    }
    const int t0 = T + 2 * tq;
    float xa[4] = {s0[0] + r0[0], s0[1] + r0[1], s1[0] + r1[0], s1[1] + r1[1]};
    float xb[4] = {s0[2] + r0[2], s0[3] + r0[3], s1[2] + r1[2], s1[3] + r1[3]};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = t0 + (e & 1) + 8 * (e >> 1);
      xa[e] = t <= pos_a ? fmaf(xa[e], cs_a, bias_a) : -INFINITY;
      xb[e] = t <= pos_b ? fmaf(xb[e], cs_b, bias_b) : -INFINITY;
    }
    softmax(xa, xb);
    // A operands of P: rows a / b x tokens (2tq, 2tq+1) and (8+2tq, 9+2tq)
    uint32_t ph[4], pl[4];
    split2h(xa[0], xa[1], ph[0], pl[0]);
    split2h(xb[0], xb[1], ph[1], pl[1]);
    split2h(xa[2], xa[3], ph[2], pl[2]);
    split2h(xb[2], xb[3], ph[3], pl[3]);
    uint32_t vw[2 * BITS];
    load_value_words<BITS>(cb + g.off_V + us * g.sub_bytes, lane, vw);
    const uint16_t* vms = reinterpret_cast<const uint16_t*>(cb + g.off_Vm) + 16 * us * g.nvg;
    const uint16_t* vmz = vms + g.P * g.nvg;
    uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0, l0 = 0, l1 = 0, l2 = 0, l3 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & ((1 << vg_shift) - 1)) == 0) {
        const int gv = i >> vg_shift, n = g.nvg;
        const uint32_t s01 = uint32_t(vms[(2 * tq) * n + gv]) | (uint32_t(vms[(2 * tq + 1) * n + gv]) << 16);
        const uint32_t s89 = uint32_t(vms[(2 * tq + 8) * n + gv]) | (uint32_t(vms[(2 * tq + 9) * n + gv]) << 16);
        ps_split(ph[0], pl[0], s01, h0, l0);
        ps_split(ph[1], pl[1], s01, h1, l1);
        ps_split(ph[2], pl[2], s89, h2, l2);
        ps_split(ph[3], pl[3], s89, h3, l3);
        if (ASYM) {
          const float z0 = __half2float(__ushort_as_half(vmz[(2 * tq) * n + gv]));
          const float z1 = __half2float(__ushort_as_half(vmz[(2 * tq + 1) * n + gv]));
          const float z8 = __half2float(__ushort_as_half(vmz[(2 * tq + 8) * n + gv]));
          const float z9 = __half2float(__ushort_as_half(vmz[(2 * tq + 9) * n + gv]));
          const float dza = xa[0] * z0 + xa[1] * z1 + xa[2] * z8 + xa[3] * z9;
          const float dzb = xb[0] * z0 + xb[1] * z1 + xb[2] * z8 + xb[3] * z9;
#pragma unroll
          for (int v = 0; v < 4; ++v) {   // register-resident select of group gv
            za[v] += v == gv ? dza : 0.0f;
            zb[v] += v == gv ? dzb : 0.0f;
          }
        }
      }
      uint32_t v0, v1, v2, v3;
      value_frag<BITS, SGN, true>(vw, i, v0, v1, v2, v3);
      mma_f16(o[2 * i], h0, h1, h2, h3, v0, v2);
      mma_f16(o[2 * i], l0, l1, l2, l3, v0, v2);
      mma_f16(o[2 * i + 1], h0, h1, h2, h3, v1, v3);
      mma_f16(o[2 * i + 1], l0, l1, l2, l3, v1, v3);
    }
  };

  // one 16-row tile of the BF16 window (tokens T .. T + 15)
  auto window_tile = [&](const uint8_t* stg, int T) {
    const uint32_t kaddr = smem_addr(stg), vaddr = kaddr + 16 * D * 2;
    const uint32_t qaddr = smem_addr(qs);
    const int mi = lane >> 3, rr = lane & 7;
    float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
      const int qr = rr + 8 * (mi & 1), qc = 2 * j + (mi >> 1);
      ldsm_x4(qaddr + (qr * D + 8 * (qc ^ (qr & 7))) * 2, a0, a1, a2, a3);
      const int kr = rr + 8 * (mi >> 1), kc = 16 * j + 8 * (mi & 1);
      ldsm_x4(kaddr + (kr * D + kc) * 2, b0, b1, b2, b3);
      mma_bf16(s0, a0, a1, a2, a3, b0, b1);
      mma_bf16(s1, a0, a1, a2, a3, b2, b3);
    }
    const int t0 = T + 2 * tq;
    const float cw = a.qk_scale;
    float xa[4] = {s0[0], s0[1], s1[0], s1[1]}, xb[4] = {s0[2], s0[3], s1[2], s1[3]};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = t0 + (e & 1) + 8 * (e >> 1);
      xa[e] = t <= pos_a ? xa[e] * cw : -INFINITY;
      xb[e] = t <= pos_b ? xb[e] * cw : -INFINITY;
    }
    softmax(xa, xb);
    uint32_t ph[4], pl[4];
    split2(xa[0], xa[1], ph[0], pl[0]);
    split2(xb[0], xb[1], ph[1], pl[1]);
    split2(xa[2], xa[3], ph[2], pl[2]);
    split2(xb[2], xb[3], ph[3], pl[3]);
#pragma unroll
    for (int d2 = 0; d2 < 8; ++d2) {
      uint32_t v0, v1, v2, v3;
      const int vr = rr + 8 * (mi & 1), vc = 16 * d2 + 8 * (mi >> 1);
      ldsm_x4_t(vaddr + (vr * D + vc) * 2, v0, v1, v2, v3);
      mma_bf16(o[2 * d2], ph[0], ph[1], ph[2], ph[3], v0, v1);
      mma_bf16(o[2 * d2], pl[0], pl[1], pl[2], pl[3], v0, v1);
      mma_bf16(o[2 * d2 + 1], ph[0], ph[1], ph[2], ph[3], v2, v3);
      mma_bf16(o[2 * d2 + 1], pl[0], pl[1], pl[2], pl[3], v2, v3);
    }
  };

  // ---- main loop: every warp consumes every item --------------------------------
  bool aborted = false;
  int consumed = K;   // items whose copies this CTA has waited for
  for (int k = 0; k < K; ++k) {
    const int sidx = k % kPfStages;
    if (!aborted) {
      const bool ok = mbar_wait_bounded(bar0 + 8 * sidx, uint32_t((k / kPfStages) & 1), kPfWaitNs, abort_flag);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) {
          atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        aborted = true;
        consumed = k;
      }
    }
    if (!aborted && wn > 0) {
      const uint8_t* stg = smem + L.stages + sidx * a.stage_bytes;
      if (k < nu) {
        const int T0 = (u0 + k) << a.lg_sup;
        const int valid = min(a.sup, qa - T0);
        int cur = -1;
        for (int tok0 = 0; tok0 < valid && T0 + tok0 <= wmax; tok0 += 16) {
          const int gi = tok0 >> g.lg_gk;
          if (gi != cur) {
            cur = gi;
            qprime(stg, gi);
          }
          quant_sub(stg, tok0, T0 + tok0);
        }
      } else {
        const int T = Lq + 16 * (k - nu);
        if (T <= wmax) window_tile(stg, T);
      }
    }
    __syncthreads();   // every warp is done with stage sidx
    if (tid == 0 && !aborted && !*abort_flag && k + kPfStages < K) issue(k + kPfStages);
  }
  if (aborted || *abort_flag) {
    // let the copies in flight land before the CTA exits (bounded)
    if (tid == 0)
      for (int k = consumed; k < issued; ++k)
        (void)mbar_wait_bounded(bar0 + 8 * (k % kPfStages), uint32_t((k / kPfStages) & 1), kPfWaitNs);
    return;
  }

  // ---- emit ---------------------------------------------------------------------
  l_a += __shfl_xor_sync(kFull, l_a, 1);
  l_a += __shfl_xor_sync(kFull, l_a, 2);
  l_b += __shfl_xor_sync(kFull, l_b, 1);
  l_b += __shfl_xor_sync(kFull, l_b, 2);
  if (ASYM) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      za[v] += __shfl_xor_sync(kFull, za[v], 1);
      za[v] += __shfl_xor_sync(kFull, za[v], 2);
      zb[v] += __shfl_xor_sync(kFull, zb[v], 1);
      zb[v] += __shfl_xor_sync(kFull, zb[v], 2);
    }
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      const int gv = (8 * d) >> (vg_shift + 4);
      const float zav = gv == 0 ? za[0] : gv == 1 ? za[1] : gv == 2 ? za[2] : za[3];
      const float zbv = gv == 0 ? zb[0] : gv == 1 ? zb[1] : gv == 2 ? zb[2] : zb[3];
      o[d][0] += zav; o[d][1] += zav;
      o[d][2] += zbv; o[d][3] += zbv;
    }
  }
  auto emit_row = [&](int slot, int head, float m, float l, int c01) {
    const int hq = h * G + head;
    const int64_t row = int64_t(rows[2 * (wt0 + slot)]) * g.h_q + hq;
    if (a.splits == 1) {
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;
      float2* dst = reinterpret_cast<float2*>(a.out + row * D + 2 * tq);
#pragma unroll
      for (int d = 0; d < 16; ++d) dst[4 * d] = make_float2(o[d][c01] * inv, o[d][c01 + 1] * inv);
    } else {
      float* rec = a.part + (row * a.splits + split) * (D + 2);
      float2* dst = reinterpret_cast<float2*>(rec + 2 * tq);
#pragma unroll
      for (int d = 0; d < 16; ++d) dst[4 * d] = make_float2(o[d][c01], o[d][c01 + 1]);
      if (tq == 0) {
        rec[D] = m;
        rec[D + 1] = l;
      }
    }
  };
  if (slot_a < wn) emit_row(slot_a, gq & (G - 1), m_a, l_a, 0);
  if (slot_b < wn) emit_row(slot_b, (gq + 8) & (G - 1), m_b, l_b, 2);
}

// out[row][hq] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the
// splits in order (records of splits that saw no position have m = -inf).
// One row of a split prefill: the records (o[D], m, l) of its `splits` key
// ranges, back to back, combined by log-sum-exp in split order into
// out[D] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s (M the largest m_s;
// a record with m = -inf saw no position).  Called by a whole warp: lane c
// holds channels 4c .. 4c + 3.  The loads of up to 8 records are in flight
// together (one round trip for 8 splits or fewer; beyond that the running
// sums are rescaled to each batch's max).  The loads go through L2 only:
// the attention grid wrote the records.
__device__ __forceinline__ void prefill_merge_row(const float* rec, int splits, int lane, float* out) {
  constexpr int kBatch = 8;
  float M = -INFINITY, den = 0.0f;
  float4 num = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int s0 = 0; s0 < splits; s0 += kBatch) {
    float m[kBatch], l[kBatch];
    float2 x0[kBatch], x1[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (s0 + i < splits) {
        const float* r = rec + (s0 + i) * (kD + 2);
        m[i] = __ldcg(r + kD);
        l[i] = __ldcg(r + kD + 1);
        x0[i] = __ldcg(reinterpret_cast<const float2*>(r + 4 * lane));
        x1[i] = __ldcg(reinterpret_cast<const float2*>(r + 4 * lane + 2));
      } else {
        m[i] = -INFINITY;
        l[i] = 0.0f;
        x0[i] = x1[i] = make_float2(0.0f, 0.0f);
      }
    }
    float Mb = M;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) Mb = fmaxf(Mb, m[i]);
    if (Mb == -INFINITY) continue;
    const float c = M == -INFINITY ? 0.0f : fast_exp2(M - Mb);
    num = make_float4(num.x * c, num.y * c, num.z * c, num.w * c);
    den *= c;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const float w = m[i] == -INFINITY ? 0.0f : fast_exp2(m[i] - Mb);
      num.x = fmaf(w, x0[i].x, num.x);
      num.y = fmaf(w, x0[i].y, num.y);
      num.z = fmaf(w, x1[i].x, num.z);
      num.w = fmaf(w, x1[i].y, num.w);
      den = fmaf(w, l[i], den);
    }
    M = Mb;
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  reinterpret_cast<float4*>(out)[lane] = make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
}

// One warp per (row, query head): lane c holds channels 4c .. 4c + 3.
constexpr int kMergeRowsPerCta = 4;
__global__ void __launch_bounds__(32 * kMergeRowsPerCta) prefill_merge_kernel(const float* __restrict__ part,
                                                                             float* __restrict__ out, int splits,
                                                                             int64_t items) {
  // a programmatic dependent launch: the records are complete once the
  // attention grid is (a no-op after a plain launch)
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t item = int64_t(blockIdx.x) * kMergeRowsPerCta + (threadIdx.x >> 5);
  if (item >= items) return;
  prefill_merge_row(part + item * splits * (kD + 2), splits, lane, out + item * kD);
}

template <int BITS, int ASYM>
cudaError_t launch_prefill_t(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches) {
  const int smem = pf_smem(a.stage_bytes).total;
  auto kern = prefill_kernel<BITS, ASYM>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = raise_smem_limit(dev, reinterpret_cast<const void*>(kern), size_t(smem));
  if (e != cudaSuccess) return e;
  kern<<<a.n_tasks, kPfThreads, smem, s>>>(a);
  ++*launches;
  e = cudaGetLastError();
  if (e != cudaSuccess || a.splits == 1) return e;
  return launch_prefill_merge(a, n_rows, s, launches);
}

}  // namespace

cudaError_t launch_prefill_merge(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches) {
  const int64_t items = n_rows * a.g.h_q;
  // a programmatic dependent launch: scheduled while the attention grid
  // finishes, waiting for it on the device
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned((items + kMergeRowsPerCta - 1) / kMergeRowsPerCta));
  cfg.blockDim = dim3(32 * kMergeRowsPerCta);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_merge_kernel, static_cast<const float*>(a.part), a.out,
                                           int(a.splits), items);
  if (e == cudaSuccess) ++*launches;
  return e;
}

bool prefill_supported(const Geo& g) {
  return g.k_axis == 1 && g.R == g.g_k && !g.fp8 && g.bits != 16 && !g.scale_fp32;
}

int prefill_stage_bytes(const Geo& g, int sup) {
  return std::max((sup / g.P) * g.chunk_used, 2 * 16 * kD * 2);
}

size_t prefill_smem_bytes(int stage_bytes) { return size_t(pf_smem(stage_bytes).total); }

int prefill_ctas_per_sm(const Geo& g, int stage_bytes) {
  const int smem = pf_smem(stage_bytes).total;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  auto occ = [&](auto kern) {
    int n = 0;
    if (raise_smem_limit(dev, reinterpret_cast<const void*>(kern), size_t(smem)) != cudaSuccess) return 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kPfThreads, smem) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
  };
  if (g.bits == 4) return g.asym ? occ(prefill_kernel<4, 1>) : occ(prefill_kernel<4, 0>);
  if (g.bits == 2) return g.asym ? occ(prefill_kernel<2, 1>) : occ(prefill_kernel<2, 0>);
  return g.asym ? occ(prefill_kernel<8, 1>) : occ(prefill_kernel<8, 0>);
}

cudaError_t launch_prefill(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches) {
  const Geo& g = a.g;
  if (g.bits == 4) return g.asym ? launch_prefill_t<4, 1>(a, n_rows, s, launches) : launch_prefill_t<4, 0>(a, n_rows, s, launches);
  if (g.bits == 2) return g.asym ? launch_prefill_t<2, 1>(a, n_rows, s, launches) : launch_prefill_t<2, 0>(a, n_rows, s, launches);
  return g.asym ? launch_prefill_t<8, 1>(a, n_rows, s, launches) : launch_prefill_t<8, 0>(a, n_rows, s, launches);
}

}  // namespace kvq
