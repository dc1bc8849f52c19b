// kvq_append.cu -- kernels of kvq_append: quantize new K/V tokens into the
// paged cache.
//
//  * apply: zero newly allocated blocks that this call does not fill, and
//    write block-table / length updates of the host planner.
//  * quant_token (token-axis keys, no residual window): one warp per (token,
//    head) quantizes the key row per g_k channels and the value row per g_v
//    channels (chipfoundryservices.com "KV Cache Quantization", per-token
//    quantization; llmdaily.org day-65, "From BF16 to INT8, INT4, or even
//    fewer bits", symmetric quantizer and asymmetric zero-points).
//  * flush (channel-axis keys): once a sequence's BF16 residual window holds a
//    whole key group of R = g_k tokens, one CTA per (group, head) quantizes
//    keys per channel over the g_k tokens and values per token over g_v
//    channels and writes the group's pages (day-65, "Why some systems keep a
//    full-precision window"; oh-bug.com "KV Cache Quantization in Practice",
//    KIVI: keys per channel, values per token).  Tokens of the group appended
//    in this call are read straight from the input, earlier ones from the
//    window; the bytes equal those of appending one token at a time.
//  * residual: copy the tokens that stay in the window to their slots.
#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "kvq_device.cuh"

namespace kvq {
namespace {

// Every launch of this file fits the classic 4 KB kernel-parameter space.
static_assert(sizeof(Geo) + sizeof(DevState) + sizeof(PlanView) + 3 * sizeof(void*) + 16 <= 4096,
              "append kernel parameters exceed 4 KB");

// The bulk flush gives up on its row copies after 2 s (a device error bit).
constexpr uint64_t kFlushWaitNs = 2000000000ull;
// Row stride (bf16 elements) of the bulk flush's gathered K and V rows: 16
// bytes of padding per 256-byte row move consecutive rows by four banks (and
// keep every row 16-byte aligned for its bulk copy).
constexpr int kFlushRowStride = kD + 8;

// A decode launched right after an append is a programmatic dependent launch:
// letting it be scheduled at the start of every append kernel hides its launch
// behind the append (it waits for this grid on the device before it reads).
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// The plan's entries: inline in the launch parameters or uploaded.
__device__ __forceinline__ const int32_t* plan_of(const PlanView& p) { return p.plan ? p.plan : p.inl; }

// Debug build: the indices of one flush entry (sequence, page blocks, window
// slots of the group's rows) lie inside their buffers.  Every thread of the
// CTA reads the same entry, so the answer is uniform over the CTA.
__device__ __forceinline__ bool flush_entry_ok(const Geo& g, const DevState& d, const int32_t* ent,
                                               const int32_t* srcs) {
  if (!KVQ_DEBUG) return true;
  bool ok = ent[0] >= 0 && ent[0] < g.max_seqs && ent[2] >= 1 && ent[2] <= kFlushEntryInts - 3;
  for (int j = 0; ok && j < ent[2]; ++j) ok = ent[3 + j] >= 0 && ent[3 + j] < g.num_blocks;
  for (int r = 0; ok && r < g.R; ++r) ok = srcs[r] >= -g.R;
  if (!ok && threadIdx.x == 0) atomicOr(d.err, KVQ_DEVERR_INDEX);
  return ok;
}

// ---------------------------------------------------------------------------
// Table and length updates and zeroing of new partial blocks, done by threads
// tid, tid + nthr, ...; with `kin` given it also copies the plan's window rows
// into the BF16 window (a call whose window writes touch no slot that a flush
// of the same call reads).
__device__ __forceinline__ void apply_body(const Geo& g, const DevState& d, const PlanView& p,
                                           const uint16_t* kin, const uint16_t* vin, int64_t tid,
                                           int64_t nthr) {
  const int32_t* plan = plan_of(p);
  if (kin) {
    constexpr int D = kD;
    const int64_t total = int64_t(p.n_res) * g.h_kv * 2 * (D / 8);
    for (int64_t idx = tid; idx < total; idx += nthr) {
      const int c8 = int(idx % (D / 8));
      int64_t rest = idx / (D / 8);
      const int which = int(rest % 2);
      rest /= 2;
      const int h = int(rest % g.h_kv);
      const int e = int(rest / g.h_kv);
      const int32_t src = plan[p.off_res + 3 * e];
      const int32_t seq = plan[p.off_res + 3 * e + 1];
      const int32_t slot = plan[p.off_res + 3 * e + 2];
      if (!dcheck(src >= 0 && seq >= 0 && seq < g.max_seqs && slot >= 0 && slot < g.R, d.err, KVQ_DEVERR_INDEX))
        continue;
      const uint16_t* s = (which ? vin : kin) + (int64_t(src) * g.h_kv + h) * D;
      uint16_t* dst = (which ? d.vres : d.kres) + ((int64_t(seq) * g.h_kv + h) * g.R + slot) * D;
      reinterpret_cast<uint4*>(dst)[c8] = reinterpret_cast<const uint4*>(s)[c8];
    }
  }
  // zero whole blocks (16-byte stores)
  const int64_t per_block = g.block_bytes / 16;
  const int64_t zero_items = int64_t(p.n_zero) * per_block;
  for (int64_t i = tid; i < zero_items; i += nthr) {
    const int32_t blk = plan[p.off_zero + i / per_block];
    if (!dcheck(blk >= 0 && blk < g.num_blocks, d.err, KVQ_DEVERR_INDEX)) continue;
    reinterpret_cast<uint4*>(d.pool + int64_t(blk) * g.block_bytes)[i % per_block] =
        make_uint4(0, 0, 0, 0);
  }
  for (int64_t i = tid; i < p.n_tab; i += nthr) {
    const int32_t ti = plan[p.off_tab + 2 * i], tv = plan[p.off_tab + 2 * i + 1];
    if (!dcheck(ti >= 0 && int64_t(ti) < int64_t(g.max_seqs) * g.mbps && tv >= -1 && tv < g.num_blocks, d.err,
                KVQ_DEVERR_INDEX))
      continue;
    d.table[ti] = tv;
  }
  for (int64_t i = tid; i < p.n_len; i += nthr) {
    const int32_t li = plan[p.off_len + 2 * i];
    if (!dcheck(li >= 0 && li < g.max_seqs, d.err, KVQ_DEVERR_INDEX)) continue;
    d.len[li] = plan[p.off_len + 2 * i + 1];
  }
}

// Threads an apply body needs for a plan (window rows copied or not).
inline int64_t apply_work(const Geo& g, const PlanView& p, bool copy_rows) {
  int64_t work = std::max<int64_t>(int64_t(p.n_zero) * (g.block_bytes / 16), std::max(p.n_tab, p.n_len));
  if (copy_rows) work = std::max<int64_t>(work, int64_t(p.n_res) * g.h_kv * 2 * (kD / 8));
  return work;
}

__global__ void apply_kernel(const Geo g, const DevState d, const __grid_constant__ PlanView p,
                             const uint16_t* kin, const uint16_t* vin) {
  launch_dependents();
  apply_body(g, d, p, kin, vin, int64_t(blockIdx.x) * blockDim.x + threadIdx.x,
             int64_t(gridDim.x) * blockDim.x);
}

// ---------------------------------------------------------------------------
// Per-token quantization: one warp per (token, head); lane l holds channels
// 4l .. 4l+3.
template <int BITS, int ASYM>
__global__ void __launch_bounds__(256) quant_token_kernel(const Geo g, const DevState d,
                                                          const __grid_constant__ PlanView p, const uint16_t* kin,
                                                          const uint16_t* vin) {
  launch_dependents();
  constexpr int D = kD;
  constexpr int N = 32 / BITS;                 // codes per word
  constexpr int Q = ASYM ? (1 << BITS) - 1 : (1 << (BITS - 1)) - 1;
  __shared__ int8_t s_codes[8][D];             // per warp: codes by channel
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t item = int64_t(blockIdx.x) * 8 + wib;
  if (item >= int64_t(p.n_tok) * g.h_kv) return;
  const int e = int(item / g.h_kv), h = int(item % g.h_kv);
  const int32_t src = plan_of(p)[p.off_tok + 3 * e];
  const int32_t blk = plan_of(p)[p.off_tok + 3 * e + 1];
  const int32_t tok = plan_of(p)[p.off_tok + 3 * e + 2];
  if (!dcheck(src >= 0 && blk >= 0 && blk < g.num_blocks && tok >= 0 && tok < g.P, d.err, KVQ_DEVERR_INDEX))
    return;   // the warp's item, uniform over the warp
  uint8_t* chunk = d.pool + int64_t(blk) * g.block_bytes + int64_t(h) * g.chunk_bytes;
  const int sub = tok >> 4, r = tok & 15;

  for (int which = 0; which < 2; ++which) {      // 0: key row, 1: value row
    const uint16_t* row = (which ? vin : kin) + (int64_t(src) * g.h_kv + h) * D;
    const uint2 raw = *reinterpret_cast<const uint2*>(row + 4 * lane);
    float x[4] = {bf16_bits_to_float(raw.x & 0xFFFF), bf16_bits_to_float(raw.x >> 16),
                  bf16_bits_to_float(raw.y & 0xFFFF), bf16_bits_to_float(raw.y >> 16)};
    const int gsz = which ? g.g_v : g.g_k;
    const int ng = which ? g.nvg : g.nkg;
    const int lanes_per_group = gsz / 4;
    float a = 0.0f, mn = x[0], mx = x[0];
    for (int i = 0; i < 4; ++i) {
      a = fmaxf(a, fabsf(x[i]));
      mn = fminf(mn, x[i]);
      mx = fmaxf(mx, x[i]);
    }
    for (int off = 1; off < lanes_per_group; off <<= 1) {
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    float sh, zh = 0.0f;
    if (ASYM) {
      zh = stored_value(mn, g.scale_fp32);
      sh = stored_value(__fdiv_rn(__fsub_rn(mx, mn), float(Q)), g.scale_fp32);
    } else {
      sh = stored_value(__fdiv_rn(a, float(Q)), g.scale_fp32);
    }
    const float inv = quant_inv(sh);
    for (int i = 0; i < 4; ++i)
      s_codes[wib][4 * lane + i] =
          int8_t(ASYM ? quant_asym_fast(x[i], sh, inv, zh, Q) : quant_sym_fast(x[i], sh, inv, Q));
    const int gi = (4 * lane) / gsz;
    if ((4 * lane) % gsz == 0) {
      const int off_meta = which ? g.off_Vm : g.off_Km;
      uint8_t* m = chunk + off_meta + (int64_t(tok) * ng + gi) * g.es;
      store_meta(m, sh, g.scale_fp32);
      if (ASYM) store_meta(m + int64_t(g.P) * ng * g.es, zh, g.scale_fp32);
    }
    __syncwarp();
    if (which == 0) {
      // key row: D*BITS/32 words, element l of word w is list position w*N + l
      if (lane < D * BITS / 32) {
        uint32_t word = 0;
        for (int l = 0; l < N; ++l) {
          const int c = key_channel(lane * N + l);
          word |= (uint32_t(s_codes[wib][c]) & ((1u << BITS) - 1)) << (BITS * word_field(l, N));
        }
        *reinterpret_cast<uint32_t*>(chunk + sub * g.sub_bytes + r * g.row_bytes + 4 * lane) = word;
      }
    } else {
      // value codes: this token owns whole bytes of its sub-tile
      const int tau = r, tq = (tau & 7) >> 1, hi = tau & 1, second = tau >> 3;
      uint8_t* vsub = chunk + g.off_V + sub * g.sub_bytes;
      constexpr int bytes_per_token = D * BITS / 8;
      for (int bi = lane; bi < bytes_per_token; bi += 32) {
        uint32_t byte = 0;
        int gq, word, bsel;
        if (BITS == 4) {
          gq = bi >> 3;
          const int i = bi & 7;
          word = i;
          bsel = 2 * hi + second;
          byte = (uint32_t(s_codes[wib][16 * i + gq]) & 15u) |
                 ((uint32_t(s_codes[wib][16 * i + gq + 8]) & 15u) << 4);
        } else if (BITS == 2) {
          gq = bi >> 2;
          const int i2 = bi & 3;
          word = i2;
          bsel = 2 * hi + second;
          const int cs[4] = {32 * i2 + gq, 32 * i2 + gq + 8, 32 * i2 + 16 + gq, 32 * i2 + 24 + gq};
          for (int m = 0; m < 4; ++m) byte |= (uint32_t(s_codes[wib][cs[m]]) & 3u) << (2 * m);
        } else {
          gq = bi >> 4;
          const int rest = bi & 15, i = rest >> 1, half = rest & 1;
          word = 2 * i + second;
          bsel = 2 * hi + half;
          byte = uint32_t(s_codes[wib][16 * i + gq + 8 * half]) & 255u;
        }
        const int lam = 4 * gq + tq;
        vsub[lam * (8 * BITS) + 4 * word + bsel] = uint8_t(byte);
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Per-channel key flush: one CTA per (flushed group, head, 16-token sub-tile).
// Every CTA gathers the group's R key rows and computes all channel scales
// (they need every row), then writes only its own sub-tile's key and value
// codes, value scales, and -- when its sub-tile starts a page -- that page's
// slice of the key scales.  CTAs with blockIdx.x >= n_flush run the plan's
// apply body instead (with the window copy when `fuse_rows` is set), so a
// decode-sized append is one launch.
template <int BITS, int ASYM>
__global__ void __launch_bounds__(kFlushThreads) flush_kernel(const Geo g, const DevState d,
                                                              const __grid_constant__ PlanView p,
                                                              const uint16_t* kin,
                                                              const uint16_t* vin, int fuse_rows) {
  launch_dependents();
  if (int(blockIdx.x) >= p.n_flush) {
    const int64_t cta =
        (int64_t(blockIdx.x - p.n_flush) * gridDim.y + blockIdx.y) * gridDim.z + blockIdx.z;
    const int64_t ctas = int64_t(gridDim.x - p.n_flush) * gridDim.y * gridDim.z;
    apply_body(g, d, p, fuse_rows ? kin : nullptr, vin, cta * blockDim.x + threadIdx.x, ctas * blockDim.x);
    return;
  }
  constexpr int D = kD;
  constexpr int N = 32 / BITS;
  constexpr int Q = ASYM ? (1 << BITS) - 1 : (1 << (BITS - 1)) - 1;
  extern __shared__ __align__(16) uint8_t smem[];
  const int R = g.R;
  uint16_t* kt = reinterpret_cast<uint16_t*>(smem);                  // [R][D] bf16
  uint16_t* vt = kt + R * D;                                         // [R][D]
  float* ksc = reinterpret_cast<float*>(vt + R * D);                 // [D]
  float* kzp = ksc + D;                                              // [D]
  float* vsc = kzp + D;                                              // [R][nvg]
  float* vzp = vsc + R * g.nvg;                                      // [R][nvg]
  float* kinv = vzp + R * g.nvg;                                     // [D] RN(1 / key scale)
  float* vinv = kinv + D;                                            // [R][nvg]

  const int e = blockIdx.x, h = blockIdx.y, zs = blockIdx.z, tid = threadIdx.x;
  const int r_lo = 16 * zs;   // this CTA's rows [r_lo, r_lo + 16)
  const int32_t* ent = plan_of(p) + p.off_flush + e * kFlushEntryInts;
  const int seq = ent[0];
  const int npg = ent[2];
  const int32_t* srcs = plan_of(p) + p.off_src + int64_t(e) * R;
  if (!flush_entry_ok(g, d, ent, srcs)) return;

  // 1. gather the group's K rows and this sub-tile's V rows (bf16) into
  //    shared memory
  for (int idx = tid; idx < R * (D / 8) * 2; idx += blockDim.x) {
    const int which = idx / (R * (D / 8));
    const int rem = idx % (R * (D / 8));
    const int r = rem / (D / 8), c8 = rem % (D / 8);
    if (which && (r < r_lo || r >= r_lo + 16)) continue;
    const int32_t s = srcs[r];
    const uint16_t* src;
    if (s >= 0) src = (which ? vin : kin) + (int64_t(s) * g.h_kv + h) * D;
    else src = (which ? d.vres : d.kres) + ((int64_t(seq) * g.h_kv + h) * R + (-1 - s)) * D;
    reinterpret_cast<uint4*>((which ? vt : kt) + r * D)[c8] = reinterpret_cast<const uint4*>(src)[c8];
  }
  __syncthreads();

  // 2. statistics: key channels (threads 0..127), value (token, group) rows
  if (tid < D) {
    const int c = tid;
    float a = 0.0f, mn = bf16_bits_to_float(kt[c]), mx = mn;
    for (int r = 0; r < R; ++r) {
      const float x = bf16_bits_to_float(kt[r * D + c]);
      a = fmaxf(a, fabsf(x));
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    if (ASYM) {
      kzp[c] = stored_value(mn, g.scale_fp32);
      ksc[c] = stored_value(__fdiv_rn(__fsub_rn(mx, mn), float(Q)), g.scale_fp32);
    } else {
      ksc[c] = stored_value(__fdiv_rn(a, float(Q)), g.scale_fp32);
      kzp[c] = 0.0f;
    }
    kinv[c] = quant_inv(ksc[c]);
  } else {
    const int w = (tid - D) >> 5, lane = tid & 31;
    const int lanes_per_group = g.g_v / 4;
    for (int r = r_lo + w; r < r_lo + 16; r += (blockDim.x - D) / 32) {
      float x[4];
      for (int i = 0; i < 4; ++i) x[i] = bf16_bits_to_float(vt[r * D + 4 * lane + i]);
      float a = 0.0f, mn = x[0], mx = x[0];
      for (int i = 0; i < 4; ++i) {
        a = fmaxf(a, fabsf(x[i]));
        mn = fminf(mn, x[i]);
        mx = fmaxf(mx, x[i]);
      }
      for (int off = 1; off < lanes_per_group; off <<= 1) {
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      }
      if ((4 * lane) % g.g_v == 0) {
        const int gi = (4 * lane) / g.g_v;
        if (ASYM) {
          vzp[r * g.nvg + gi] = stored_value(mn, g.scale_fp32);
          vsc[r * g.nvg + gi] = stored_value(__fdiv_rn(__fsub_rn(mx, mn), float(Q)), g.scale_fp32);
        } else {
          vsc[r * g.nvg + gi] = stored_value(__fdiv_rn(a, float(Q)), g.scale_fp32);
          vzp[r * g.nvg + gi] = 0.0f;
        }
        vinv[r * g.nvg + gi] = quant_inv(vsc[r * g.nvg + gi]);
      }
    }
  }
  __syncthreads();

  auto chunk_of = [&](int page) -> uint8_t* {
    return d.pool + int64_t(ent[3 + page]) * g.block_bytes + int64_t(h) * g.chunk_bytes;
  };
  const int lg_gv = __ffs(g.g_v) - 1;
  auto kcode = [&](int r, int c) -> uint32_t {
    const float x = bf16_bits_to_float(kt[r * D + c]);
    const int q = ASYM ? quant_asym_fast(x, ksc[c], kinv[c], kzp[c], Q) : quant_sym_fast(x, ksc[c], kinv[c], Q);
    return uint32_t(q) & ((1u << BITS) - 1);
  };
  auto vcode = [&](int r, int c) -> uint32_t {
    const float x = bf16_bits_to_float(vt[r * D + c]);
    const int m = r * g.nvg + (c >> lg_gv);
    const int q = ASYM ? quant_asym_fast(x, vsc[m], vinv[m], vzp[m], Q) : quant_sym_fast(x, vsc[m], vinv[m], Q);
    return uint32_t(q) & ((1u << BITS) - 1);
  };
  const int lg_spp = g.lg_P - 4, spp_mask = (1 << lg_spp) - 1;   // 16-token sub-tiles per page (a power of two)

  // 3. key codes: word W of the group -> (sub-tile, row, word in row)
  const int row_words = D * BITS / 32;
  const int k_words = 16 * row_words;
  for (int W = tid; W < k_words; W += blockDim.x) {
    const int rowi = r_lo + W / row_words, w = W % row_words;   // rowi = token in group
    uint32_t word = 0;
    for (int l = 0; l < N; ++l) word |= kcode(rowi, key_channel(w * N + l)) << (BITS * word_field(l, N));
    const int sub = rowi >> 4, rr = rowi & 15;
    uint8_t* dst = chunk_of(sub >> lg_spp) + (sub & spp_mask) * g.sub_bytes +
                   rr * g.row_bytes + 4 * w;
    *reinterpret_cast<uint32_t*>(dst) = word;
  }

  // 4. value codes: word W -> (sub-tile, lane record, word in record); the
  //    record of lane (4 gq + tq) packs mma operand registers a0..a3 of each
  //    16-channel tile i: a0 = (ch 16i+gq, tok 2tq | 2tq+1), a1 = ch + 8,
  //    a2 = tokens + 8, a3 = both.
  const int rec_words = 2 * BITS;
  const int v_words = 32 * rec_words;
  for (int W = tid; W < v_words; W += blockDim.x) {
    const int sub = zs, rem = W;
    const int lam = rem / rec_words, w = rem % rec_words;
    const int gq = lam >> 2, tq = lam & 3;
    uint32_t word = 0;
    for (int x = 0; x < N / 2; ++x) {
      int i, reg;
      if (BITS == 8) { i = w >> 1; reg = 2 * (w & 1) + x; }
      else if (BITS == 4) { i = w; reg = x; }
      else { i = 2 * w + ((x >> 1) & 1); reg = 2 * (x >> 2) + (x & 1); }
      const int c = 16 * i + gq + 8 * (reg & 1);
      const int t0 = 16 * sub + 2 * tq + 8 * (reg >> 1);
      word |= vcode(t0, c) << (BITS * x);
      word |= vcode(t0 + 1, c) << (BITS * (x + N / 2));
    }
    uint8_t* dst = chunk_of(sub >> lg_spp) + g.off_V + (sub & spp_mask) * g.sub_bytes +
                   lam * (8 * BITS) + 4 * w;
    *reinterpret_cast<uint32_t*>(dst) = word;
  }

  // 5. metadata: key scales in list order, striped over the group's pages
  //    (the CTA of a page's first sub-tile writes that page's slice); value
  //    scales of this sub-tile's rows
  //    (page and nvg are powers of two)
  if ((r_lo & (g.P - 1)) == 0) {
    const int page = r_lo >> g.lg_P;
    for (int off = tid; off < g.kslice; off += blockDim.x) {
      const int c = key_channel(page * g.kslice + off);
      uint8_t* km = chunk_of(page) + g.off_Km;
      store_meta(km + off * g.es, ksc[c], g.scale_fp32);
      if (ASYM) store_meta(km + (g.kslice + off) * g.es, kzp[c], g.scale_fp32);
    }
  }
  const int lg_nvg = __ffs(g.nvg) - 1;
  for (int idx = r_lo * g.nvg + tid; idx < (r_lo + 16) * g.nvg; idx += blockDim.x) {
    const int r = idx >> lg_nvg, gi = idx & (g.nvg - 1);
    const int page = r >> g.lg_P, rp = r & (g.P - 1);
    uint8_t* vm = chunk_of(page) + g.off_Vm;
    store_meta(vm + (rp * g.nvg + gi) * g.es, vsc[idx], g.scale_fp32);
    if (ASYM) store_meta(vm + (g.P * g.nvg + rp * g.nvg + gi) * g.es, vzp[idx], g.scale_fp32);
  }
  (void)npg;
}

// ---------------------------------------------------------------------------
// Per-channel key flush for calls that flush many groups (bulk prefill): one
// CTA per (flushed group, head).  The group's R key and value rows are
// gathered once, the channel statistics use every thread, every code is
// quantized once into shared memory, and the packing passes then write all
// of the group's pages.  The bytes are those of flush_kernel.
template <int BITS, int ASYM>
__global__ void __launch_bounds__(kFlushThreads) flush_group_kernel(const Geo g, const DevState d,
                                                                    const __grid_constant__ PlanView p,
                                                                    const uint16_t* kin, const uint16_t* vin,
                                                                    int fuse_rows) {
  launch_dependents();
  if (int(blockIdx.x) >= p.n_flush) {
    const int64_t cta = int64_t(blockIdx.x - p.n_flush) * gridDim.y + blockIdx.y;
    const int64_t ctas = int64_t(gridDim.x - p.n_flush) * gridDim.y;
    apply_body(g, d, p, fuse_rows ? kin : nullptr, vin, cta * blockDim.x + threadIdx.x, ctas * blockDim.x);
    return;
  }
  constexpr int D = kD;
  constexpr int N = 32 / BITS;
  constexpr int Q = ASYM ? (1 << BITS) - 1 : (1 << (BITS - 1)) - 1;
  constexpr uint32_t MASK = (1u << BITS) - 1;
  extern __shared__ __align__(16) uint8_t smem[];
  const int R = g.R;
  constexpr int RS = kFlushRowStride;
  uint16_t* kt = reinterpret_cast<uint16_t*>(smem);                 // [R][RS] bf16 (D used)
  uint16_t* vt = kt + R * RS;                                       // [R][RS] bf16
  float* ksc = reinterpret_cast<float*>(vt + R * RS);               // [D]
  float* kzp = ksc + D;                                             // [D]
  float* vsc = kzp + D;                                             // [R][nvg]
  float* vzp = vsc + R * g.nvg;                                     // [R][nvg]
  float* kinv = vzp + R * g.nvg;                                    // [D] RN(1 / key scale)
  float* vinv = kinv + D;                                           // [R][nvg]
  float* part = vinv + R * g.nvg;                                   // [3][3][D] key statistics of row quarters 1-3
  int32_t* ssrc = reinterpret_cast<int32_t*>(part + 9 * D);         // [R]
  const uint32_t gbar = smem_addr(ssrc + ((R + 1) & ~1));           // 8-byte mbarrier of the row copies

  const int e = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, T = blockDim.x;
  const int32_t* ent = plan_of(p) + p.off_flush + e * kFlushEntryInts;
  const int seq = ent[0];
  const int32_t* srcs = plan_of(p) + p.off_src + int64_t(e) * R;
  if (!flush_entry_ok(g, d, ent, srcs)) return;
  for (int r = tid; r < R; r += T) ssrc[r] = srcs[r];
  if (tid == 0) {
    mbar_init(gbar, 1);
    mbar_init_fence();
    mbar_arrive_expect_tx(gbar, uint32_t(2 * R * D * 2));
  }
  __syncthreads();

  // 1. the group's K and V rows (bf16, 256 bytes each) from the input, or the
  //    window for rows appended earlier: one bulk copy per row, all 2R in
  //    flight at once on one mbarrier (R <= 128, so one row per thread)
  if (tid < 2 * R) {
    const int which = tid >= R, r = which ? tid - R : tid;
    const int32_t s = ssrc[r];
    const uint16_t* src = s >= 0 ? (which ? vin : kin) + (int64_t(s) * g.h_kv + h) * D
                                 : (which ? d.vres : d.kres) + ((int64_t(seq) * g.h_kv + h) * R + (-1 - s)) * D;
    bulk_g2s(smem_addr((which ? vt : kt) + r * RS), src, uint32_t(D * 2), gbar);
  }
  if (!__syncthreads_and(mbar_wait_bounded(gbar, 0, kFlushWaitNs))) {
    if (tid == 0) atomicOr(d.err, KVQ_DEVERR_TIMEOUT);
    (void)mbar_wait_bounded(gbar, 0, kFlushWaitNs);   // keep the CTA until its copies land (bounded)
    return;
  }

  // 2. key channel statistics: thread (quarter, pair) scans channels 2 pair,
  //    2 pair + 1 (one 32-bit load per row) over a quarter of the rows; the
  //    first quarter's threads combine and make the pair's scales
  {
    static_assert(kFlushThreads == 2 * D, "64 channel pairs x 4 row quarters");
    const int cp = tid % (D / 2), qt = tid / (D / 2);
    const int r0 = qt * (R / 4), r1 = r0 + R / 4;
    float a[2] = {0.0f, 0.0f}, mn[2] = {INFINITY, INFINITY}, mx[2] = {-INFINITY, -INFINITY};
#pragma unroll 4
    for (int r = r0; r < r1; ++r) {
      const uint32_t pr = *reinterpret_cast<const uint32_t*>(kt + r * RS + 2 * cp);
      const float x[2] = {__uint_as_float(pr << 16), __uint_as_float(pr & 0xFFFF0000u)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (ASYM) {
          mn[e] = fminf(mn[e], x[e]);
          mx[e] = fmaxf(mx[e], x[e]);
        } else {
          a[e] = fmaxf(a[e], fabsf(x[e]));
        }
      }
    }
    if (qt > 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float* pq = part + (qt - 1) * 3 * D;
        pq[2 * cp + e] = a[e];
        pq[D + 2 * cp + e] = mn[e];
        pq[2 * D + 2 * cp + e] = mx[e];
      }
    }
    __syncthreads();
    if (qt == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = 2 * cp + e;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const float* pq = part + k * 3 * D;
          a[e] = fmaxf(a[e], pq[c]);
          mn[e] = fminf(mn[e], pq[D + c]);
          mx[e] = fmaxf(mx[e], pq[2 * D + c]);
        }
        if (ASYM) {
          kzp[c] = stored_value(mn[e], g.scale_fp32);
          ksc[c] = stored_value(__fdiv_rn(__fsub_rn(mx[e], mn[e]), float(Q)), g.scale_fp32);
        } else {
          ksc[c] = stored_value(__fdiv_rn(a[e], float(Q)), g.scale_fp32);
          kzp[c] = 0.0f;
        }
        kinv[c] = quant_inv(ksc[c]);
      }
    }
  }
  // value (token, group) extremes: warp w takes rows 2w, 2w + 1, 2w + 16, ...
  // (a half-warp per row); lane l holds channels 8 (l mod 16) .. + 7 (one
  // 16-byte load), reduced over the g_v / 8 lanes of its group; the scales
  // follow once every row is reduced
  {
    const int w = tid >> 5, lane = tid & 31, cl = lane & 15;
    const int lanes_per_group = g.g_v / 8;   // 4, 8 or 16: inside the half-warp
    for (int r0 = 2 * w; r0 < R; r0 += 2 * (T / 32)) {   // R is even: warp-uniform
      const int r = r0 + (lane >> 4);
      const uint4 raw = *reinterpret_cast<const uint4*>(vt + r * RS + 8 * cl);
      const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
      float x[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(rw[i] << 16);
        x[2 * i + 1] = __uint_as_float(rw[i] & 0xFFFF0000u);
      }
      if (ASYM) {
        float mn = x[0], mx = x[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
          mn = fminf(mn, x[i]);
          mx = fmaxf(mx, x[i]);
        }
        for (int off = 1; off < lanes_per_group; off <<= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        if ((cl & (lanes_per_group - 1)) == 0) {
          vzp[r * g.nvg + cl / lanes_per_group] = mn;   // raw extremes for now
          vsc[r * g.nvg + cl / lanes_per_group] = mx;
        }
      } else {
        float a = fabsf(x[0]);
#pragma unroll
        for (int i = 1; i < 8; ++i) a = fmaxf(a, fabsf(x[i]));
        for (int off = 1; off < lanes_per_group; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        if ((cl & (lanes_per_group - 1)) == 0) vsc[r * g.nvg + cl / lanes_per_group] = a;
      }
    }
  }
  __syncthreads();
  for (int m = tid; m < R * g.nvg; m += T) {   // the value scales, one (row, group) per thread
    if (ASYM) {
      const float mn = vzp[m], mx = vsc[m];
      vzp[m] = stored_value(mn, g.scale_fp32);
      vsc[m] = stored_value(__fdiv_rn(__fsub_rn(mx, mn), float(Q)), g.scale_fp32);
    } else {
      vsc[m] = stored_value(__fdiv_rn(vsc[m], float(Q)), g.scale_fp32);
      vzp[m] = 0.0f;
    }
    vinv[m] = quant_inv(vsc[m]);
  }
  __syncthreads();

  auto chunk_of = [&](int page) -> uint8_t* {
    return d.pool + int64_t(ent[3 + page]) * g.block_bytes + int64_t(h) * g.chunk_bytes;
  };
  const int lg_spp = g.lg_P - 4, spp_mask = (1 << lg_spp) - 1;   // 16-token sub-tiles per page (a power of two)

  // 3. key words, straight from the bf16 rows: word kw of a row holds the
  //    codes of key-list positions kw N .. kw N + N - 1, i.e. N / 2 pairs of
  //    adjacent channels.  A thread keeps one word column (the block size is
  //    a multiple of the words per row), so its channels' reciprocal scales
  //    and zero-points stay in registers across its rows.
  {
    constexpr int RW = D * BITS / 32;                 // words per key row
    static_assert(kFlushThreads % RW == 0, "one word column per thread");
    const int kw = tid % RW;
    int cp[N / 2];
    float iv[N], zq[N];
#pragma unroll
    for (int l = 0; l < N; ++l) {
      const int c = key_channel(kw * N + l);
      if ((l & 1) == 0) cp[l >> 1] = c;
      iv[l] = kinv[c];
      zq[l] = ASYM ? kzp[c] : 0.0f;
    }
    for (int rowi = tid / RW; rowi < R; rowi += kFlushThreads / RW) {   // warp-uniform trip count
      float xs[N];
#pragma unroll
      for (int m = 0; m < N / 2; ++m) {
        const uint32_t pr = *reinterpret_cast<const uint32_t*>(kt + rowi * RS + cp[m]);
        xs[2 * m] = __uint_as_float(pr << 16);
        xs[2 * m + 1] = __uint_as_float(pr & 0xFFFF0000u);
      }
      uint32_t word = 0;
      bool any_tie = false;   // which elements tie is found again on the rare exact path
#pragma unroll
      for (int l = 0; l < N; ++l) {
        bool tie;
        const int q = ASYM ? quant_code_nb(__fsub_rn(xs[l], zq[l]) * iv[l], 0, Q, tie)
                           : quant_code_nb(xs[l] * iv[l], -Q, Q, tie);
        any_tie |= tie;
        word |= (uint32_t(q) & MASK) << (BITS * word_field(l, N));
      }
      if (__any_sync(0xffffffffu, any_tie)) {
        for (int l = 0; l < N; ++l) {
          bool tie;
          (void)(ASYM ? quant_code_nb(__fsub_rn(xs[l], zq[l]) * iv[l], 0, Q, tie)
                      : quant_code_nb(xs[l] * iv[l], -Q, Q, tie));
          if (tie) {
            const int c = key_channel(kw * N + l);
            const int q = ASYM ? quant_asym_exact(xs[l], ksc[c], kzp[c], Q) : quant_sym_exact(xs[l], ksc[c], Q);
            const int sh = BITS * word_field(l, N);
            word = (word & ~(MASK << sh)) | ((uint32_t(q) & MASK) << sh);
          }
        }
      }
      const int sub = rowi >> 4, rr = rowi & 15;
      *reinterpret_cast<uint32_t*>(chunk_of(sub >> lg_spp) + (sub & spp_mask) * g.sub_bytes +
                                   rr * g.row_bytes + 4 * kw) = word;
    }
  }

  // 4. value words, straight from the bf16 rows: word w of lane record lam
  //    (gq = lam / 4, tq = lam % 4) of a sub-tile holds operand register reg
  //    of channel tile i for tokens (2tq, 2tq + 1) + 8 (reg / 2) and channel
  //    16 i + gq + 8 (reg % 2), each code with its token's scale for the
  //    channel's value group
  {
    // Thread (sub, lam, half) makes the record's words half·WPT .. half·WPT +
    // WPT - 1 and stores them at once: a warp writes 16 records, 512
    // contiguous bytes.  Its reads of the bf16 rows (channels 16 i + gq, token
    // rows 2 tq apart) fall in distinct banks up to a factor 2 thanks to the
    // padded row stride.
    constexpr int RECW = 2 * BITS;                    // words per lane record
    constexpr int WPT = RECW / 2;                     // words per thread
    const int lg_gv = __ffs(g.g_v) - 1;
    for (int W = tid; W < (R / 16) * 64; W += kFlushThreads) {   // warp-uniform trip count
      const int sub = W >> 6, lam = (W >> 1) & 31, half = W & 1;
      const int gq = lam >> 2, tq = lam & 3;
      uint32_t wd[WPT];
#pragma unroll
      for (int j = 0; j < WPT; ++j) {
        const int w = half * WPT + j;
        // the word's channels lie in 16 (32 for 2-bit codes) aligned
        // channels, inside one value group (g_v is 32, 64 or 128)
        const int gi = ((BITS == 2 ? 32 : BITS == 4 ? 16 : 8) * w) >> lg_gv;
        float xs[N];
        int tk[N / 2];
        uint32_t word = 0;
        bool any_tie = false;   // which elements tie is found again on the rare exact path
#pragma unroll
        for (int x = 0; x < N / 2; ++x) {
          int i, reg;
          if (BITS == 8) { i = w >> 1; reg = 2 * (w & 1) + x; }
          else if (BITS == 4) { i = w; reg = x; }
          else { i = 2 * w + ((x >> 1) & 1); reg = 2 * (x >> 2) + (x & 1); }
          const int c = 16 * i + gq + 8 * (reg & 1);
          const int t0 = 16 * sub + 2 * tq + 8 * (reg >> 1);
          tk[x] = t0;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = t0 + u, l = x + u * (N / 2);
            xs[l] = bf16_bits_to_float(vt[t * RS + c]);
            const int m = t * g.nvg + gi;
            bool tie;
            const int q = ASYM ? quant_code_nb(__fsub_rn(xs[l], vzp[m]) * vinv[m], 0, Q, tie)
                               : quant_code_nb(xs[l] * vinv[m], -Q, Q, tie);
            any_tie |= tie;
            word |= (uint32_t(q) & MASK) << (BITS * l);
          }
        }
        if (__any_sync(0xffffffffu, any_tie)) {
          for (int l = 0; l < N; ++l) {
            const int t = tk[l % (N / 2)] + l / (N / 2);
            const int m = t * g.nvg + gi;
            bool tie;
            (void)(ASYM ? quant_code_nb(__fsub_rn(xs[l], vzp[m]) * vinv[m], 0, Q, tie)
                        : quant_code_nb(xs[l] * vinv[m], -Q, Q, tie));
            if (tie) {
              const int q = ASYM ? quant_asym_exact(xs[l], vsc[m], vzp[m], Q) : quant_sym_exact(xs[l], vsc[m], Q);
              word = (word & ~(MASK << (BITS * l))) | ((uint32_t(q) & MASK) << (BITS * l));
            }
          }
        }
        wd[j] = word;
      }
      uint8_t* dst = chunk_of(sub >> lg_spp) + g.off_V + (sub & spp_mask) * g.sub_bytes +
                     lam * (8 * BITS) + half * (4 * WPT);
      if constexpr (WPT >= 4) {
#pragma unroll
        for (int v = 0; v < WPT / 4; ++v)
          reinterpret_cast<uint4*>(dst)[v] = make_uint4(wd[4 * v], wd[4 * v + 1], wd[4 * v + 2], wd[4 * v + 3]);
      } else {
        *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1]);
      }
    }
  }

  // 6. metadata: each page's slice of the key scales (list order), value scales
  //    (page, kslice and nvg = D / g_v are powers of two)
  const int npg = R >> g.lg_P, lg_nvg = __ffs(g.nvg) - 1;
  for (int idx = tid; idx < npg * g.kslice; idx += T) {
    const int page = idx >> g.lg_kslice, off = idx & (g.kslice - 1);
    const int c = key_channel(page * g.kslice + off);
    uint8_t* km = chunk_of(page) + g.off_Km;
    store_meta(km + off * g.es, ksc[c], g.scale_fp32);
    if (ASYM) store_meta(km + (g.kslice + off) * g.es, kzp[c], g.scale_fp32);
  }
  for (int idx = tid; idx < R * g.nvg; idx += T) {
    const int r = idx >> lg_nvg, gi = idx & (g.nvg - 1);
    const int page = r >> g.lg_P, rp = r & (g.P - 1);
    uint8_t* vm = chunk_of(page) + g.off_Vm;
    store_meta(vm + (rp * g.nvg + gi) * g.es, vsc[idx], g.scale_fp32);
    if (ASYM) store_meta(vm + (g.P * g.nvg + rp * g.nvg + gi) * g.es, vzp[idx], g.scale_fp32);
  }
}

// ---------------------------------------------------------------------------
__global__ void residual_kernel(const Geo g, const DevState d, const __grid_constant__ PlanView p,
                                const uint16_t* kin, const uint16_t* vin) {
  launch_dependents();
  constexpr int D = kD;
  const int64_t total = int64_t(p.n_res) * g.h_kv * 2 * (D / 8);
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int c8 = int(idx % (D / 8));
    int64_t rest = idx / (D / 8);
    const int which = int(rest % 2);
    rest /= 2;
    const int h = int(rest % g.h_kv);
    const int e = int(rest / g.h_kv);
    const int32_t src = plan_of(p)[p.off_res + 3 * e];
    const int32_t seq = plan_of(p)[p.off_res + 3 * e + 1];
    const int32_t slot = plan_of(p)[p.off_res + 3 * e + 2];
    if (!dcheck(src >= 0 && seq >= 0 && seq < g.max_seqs && slot >= 0 && slot < g.R, d.err, KVQ_DEVERR_INDEX))
      continue;
    const uint16_t* s = (which ? vin : kin) + (int64_t(src) * g.h_kv + h) * D;
    uint16_t* dst = (which ? d.vres : d.kres) + ((int64_t(seq) * g.h_kv + h) * g.R + slot) * D;
    reinterpret_cast<uint4*>(dst)[c8] = reinterpret_cast<const uint4*>(s)[c8];
  }
}

// BF16 control: the token's key and value rows of each head go unchanged into
// their page as natural bf16 rows (row r of sub-tile r / 16).  One warp per
// (token, head); lane l copies channels 4l .. 4l+3.
__global__ void __launch_bounds__(256) copy_token_kernel(const Geo g, const DevState d,
                                                         const __grid_constant__ PlanView p,
                                                         const uint16_t* kin, const uint16_t* vin) {
  launch_dependents();
  constexpr int D = kD;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t item = int64_t(blockIdx.x) * 8 + wib;
  if (item >= int64_t(p.n_tok) * g.h_kv) return;
  const int e = int(item / g.h_kv), h = int(item % g.h_kv);
  const int32_t src = plan_of(p)[p.off_tok + 3 * e];
  const int32_t blk = plan_of(p)[p.off_tok + 3 * e + 1];
  const int32_t tok = plan_of(p)[p.off_tok + 3 * e + 2];
  if (!dcheck(src >= 0 && blk >= 0 && blk < g.num_blocks && tok >= 0 && tok < g.P, d.err, KVQ_DEVERR_INDEX))
    return;   // the warp's item, uniform over the warp
  uint8_t* chunk = d.pool + int64_t(blk) * g.block_bytes + int64_t(h) * g.chunk_bytes;
  const int64_t row = int64_t(tok >> 4) * g.sub_bytes + (tok & 15) * (D * 2);
  const int64_t in = (int64_t(src) * g.h_kv + h) * D + 4 * lane;
  *reinterpret_cast<uint2*>(chunk + row + 8 * lane) = *reinterpret_cast<const uint2*>(kin + in);
  *reinterpret_cast<uint2*>(chunk + g.off_V + row + 8 * lane) = *reinterpret_cast<const uint2*>(vin + in);
}

// FP8 format: every element becomes e4m3(x / s_head) (an IEEE division, then
// round to nearest even with saturation at +-448).  Keys keep the key-list
// order with one byte per element in natural order; values go to lane records
// where operand register x of tile i holds its two tokens in bytes 2x, 2x + 1
// of word 2i + x / 2.  One warp per (token, head); each lane writes one key
// word and four value bytes.
__global__ void __launch_bounds__(256) fp8_token_kernel(const Geo g, const DevState d,
                                                        const __grid_constant__ PlanView p,
                                                        const uint16_t* kin, const uint16_t* vin) {
  launch_dependents();
  constexpr int D = kD;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t item = int64_t(blockIdx.x) * 8 + wib;
  if (item >= int64_t(p.n_tok) * g.h_kv) return;
  const int e = int(item / g.h_kv), h = int(item % g.h_kv);
  const int32_t src = plan_of(p)[p.off_tok + 3 * e];
  const int32_t blk = plan_of(p)[p.off_tok + 3 * e + 1];
  const int32_t tok = plan_of(p)[p.off_tok + 3 * e + 2];
  if (!dcheck(src >= 0 && blk >= 0 && blk < g.num_blocks && tok >= 0 && tok < g.P, d.err, KVQ_DEVERR_INDEX))
    return;   // the warp's item, uniform over the warp
  uint8_t* chunk = d.pool + int64_t(blk) * g.block_bytes + int64_t(h) * g.chunk_bytes;
  const int sub = tok >> 4, r = tok & 15;
  const float sk = d.fp8[h], sv = d.fp8[g.h_kv + h];
  const uint16_t* krow = kin + (int64_t(src) * g.h_kv + h) * D;
  const uint16_t* vrow = vin + (int64_t(src) * g.h_kv + h) * D;
  uint32_t word = 0;
  for (int b = 0; b < 4; ++b) {
    const float x = bf16_bits_to_float(krow[key_channel(4 * lane + b)]);
    word |= uint32_t(__nv_cvt_float_to_fp8(__fdiv_rn(x, sk), __NV_SATFINITE, __NV_E4M3)) << (8 * b);
  }
  *reinterpret_cast<uint32_t*>(chunk + sub * g.sub_bytes + r * g.row_bytes + 4 * lane) = word;
  const int tq = (r & 7) >> 1, hi = r & 1, second = r >> 3;
  uint8_t* vsub = chunk + g.off_V + sub * g.sub_bytes;
  for (int b = 0; b < 4; ++b) {
    const int c = 4 * lane + b, i = c >> 4, rr = c & 15, gq = rr & 7, upper = rr >> 3;
    const int reg = 2 * second + upper;
    const float x = bf16_bits_to_float(vrow[c]);
    vsub[(4 * gq + tq) * 64 + 4 * (2 * i + (reg >> 1)) + 2 * (reg & 1) + hi] =
        uint8_t(__nv_cvt_float_to_fp8(__fdiv_rn(x, sv), __NV_SATFINITE, __NV_E4M3));
  }
}

template <typename F>
cudaError_t by_format(const Geo& g, F&& f) {
  if (g.bits == 8) return g.asym ? f(std::integral_constant<int, 8>(), std::integral_constant<int, 1>())
                                 : f(std::integral_constant<int, 8>(), std::integral_constant<int, 0>());
  if (g.bits == 4) return g.asym ? f(std::integral_constant<int, 4>(), std::integral_constant<int, 1>())
                                 : f(std::integral_constant<int, 4>(), std::integral_constant<int, 0>());
  return g.asym ? f(std::integral_constant<int, 2>(), std::integral_constant<int, 1>())
                : f(std::integral_constant<int, 2>(), std::integral_constant<int, 0>());
}

size_t flush_smem_bytes(const Geo& g) {
  return size_t(2) * g.R * kD * 2 + size_t(3) * kD * 4 + size_t(3) * g.R * g.nvg * 4;
}

size_t flush_group_smem_bytes(const Geo& g) {
  return size_t(2) * g.R * kFlushRowStride * 2 + size_t(3) * kD * 4 +
         size_t(3) * g.R * g.nvg * 4 + size_t(9) * kD * 4 + size_t((g.R + 1) & ~1) * 4 + 8;
}

// Calls that flush at least this many groups use one CTA per (group, head);
// fewer (a decode step) keep one CTA per (group, head, sub-tile).
constexpr int kBulkFlushGroups = 16;

}  // namespace

cudaError_t launch_apply(const Geo& g, const DevState& d, const PlanView& p, const uint16_t* k,
                         const uint16_t* v, cudaStream_t s, int* launches) {
  const int64_t work = apply_work(g, p, k != nullptr);
  if (work == 0) return cudaSuccess;
  const int blocks = int(std::min<int64_t>((work + 255) / 256, 4096));
  apply_kernel<<<blocks, 256, 0, s>>>(g, d, p, k, v);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_quant_token(const Geo& g, const DevState& d, const PlanView& p,
                               const uint16_t* k, const uint16_t* v, cudaStream_t s, int* launches) {
  if (p.n_tok == 0) return cudaSuccess;
  const int64_t items = int64_t(p.n_tok) * g.h_kv;
  const int blocks = int((items + 7) / 8);
  if (g.bits == 16) {
    copy_token_kernel<<<blocks, 256, 0, s>>>(g, d, p, k, v);
    ++*launches;
    return cudaGetLastError();
  }
  if (g.fp8) {
    fp8_token_kernel<<<blocks, 256, 0, s>>>(g, d, p, k, v);
    ++*launches;
    return cudaGetLastError();
  }
  return by_format(g, [&](auto B, auto A) {
    quant_token_kernel<decltype(B)::value, decltype(A)::value><<<blocks, 256, 0, s>>>(g, d, p, k, v);
    ++*launches;
    return cudaGetLastError();
  });
}

cudaError_t launch_flush(const Geo& g, const DevState& d, const PlanView& p, const uint16_t* k,
                         const uint16_t* v, bool with_apply, bool fuse_rows, cudaStream_t s, int* launches) {
  if (p.n_flush == 0) return cudaSuccess;
  if (p.n_flush >= kBulkFlushGroups) {
    const size_t smem = flush_group_smem_bytes(g);
    const int64_t per_col = int64_t(g.h_kv) * kFlushThreads;
    const int64_t work = with_apply ? apply_work(g, p, fuse_rows) : 0;
    const int extra = int(std::min<int64_t>((work + per_col - 1) / per_col, 256));
    return by_format(g, [&](auto B, auto A) {
      auto kern = flush_group_kernel<decltype(B)::value, decltype(A)::value>;
      int dev = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e != cudaSuccess) return e;
      e = raise_smem_limit(dev, reinterpret_cast<const void*>(kern), smem);
      if (e != cudaSuccess) return e;
      kern<<<dim3(p.n_flush + extra, g.h_kv), kFlushThreads, smem, s>>>(g, d, p, k, v, fuse_rows ? 1 : 0);
      ++*launches;
      return cudaGetLastError();
    });
  }
  const size_t smem = flush_smem_bytes(g);
  // extra columns of (h_kv x R/16) CTAs for the apply body
  const int64_t per_col = int64_t(g.h_kv) * (g.R / 16) * kFlushThreads;
  const int64_t work = with_apply ? apply_work(g, p, fuse_rows) : 0;
  const int extra = int(std::min<int64_t>((work + per_col - 1) / per_col, 64));
  return by_format(g, [&](auto B, auto A) {
    auto kern = flush_kernel<decltype(B)::value, decltype(A)::value>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = raise_smem_limit(dev, reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(p.n_flush + extra, g.h_kv, g.R / 16), kFlushThreads, smem, s>>>(g, d, p, k, v,
                                                                              fuse_rows ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
  });
}

cudaError_t launch_residual(const Geo& g, const DevState& d, const PlanView& p, const uint16_t* k,
                            const uint16_t* v, cudaStream_t s, int* launches) {
  if (p.n_res == 0) return cudaSuccess;
  const int64_t total = int64_t(p.n_res) * g.h_kv * 2 * (kD / 8);
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 8192));
  residual_kernel<<<blocks, 256, 0, s>>>(g, d, p, k, v);
  ++*launches;
  return cudaGetLastError();
}

// A step's inputs from page-locked host memory the device maps: every thread
// loads 16-byte pieces over the bus, all in flight at once, and stores them
// into the library's device staging (a copy engine pays its per-copy latency
// instead).  Up to three segments per launch; sizes are multiples of 16 bytes.
namespace {
__global__ void __launch_bounds__(256) pull_kernel(const __grid_constant__ PullArgs a) {
  for (int sgi = 0; sgi < a.n; ++sgi) {
    const uint4* __restrict__ src = static_cast<const uint4*>(a.src[sgi]);
    uint4* __restrict__ dst = static_cast<uint4*>(a.dst[sgi]);
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.n16[sgi];
         i += int64_t(gridDim.x) * blockDim.x)
      dst[i] = src[i];
  }
}
}  // namespace

cudaError_t launch_pull(const PullArgs& a, cudaStream_t s, int* launches) {
  int64_t most = 0;
  for (int i = 0; i < a.n; ++i) most = std::max(most, a.n16[i]);
  if (most == 0) return cudaSuccess;
  pull_kernel<<<unsigned(std::min<int64_t>((most + 255) / 256, 1184)), 256, 0, s>>>(a);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace kvq
