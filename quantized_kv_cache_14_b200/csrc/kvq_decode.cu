// kvq_decode.cu -- decode attention directly over the packed low-bit paged
// cache, dequantizing inside the kernel.
//
// Computes out = softmax(q K^T / sqrt(d_h)) V for one query token per
// sequence (llmdaily.org day-65, "Why the KV cache grows so quickly"), where K
// and V are the dequantized cache x_hat = s q (+ z) ("From BF16 to INT8, INT4,
// or even fewer bits") plus the BF16 residual window ("Why some systems keep a
// full-precision window"), read through the block table ("How this connects
// to paging and prefix caching").  The pages' trade-off -- memory traffic
// saved versus dequantization work ("Why compression may also improve speed";
// oh-bug.com, misconception 1) -- decides the design:
//
//  * Work is a list of tiles: per (row, kv head), one tile per key group
//    (channel-axis keys) or per 16 tokens (token-axis keys), then the residual
//    window in 16-token tiles.  Every warp of a persistent grid takes a
//    contiguous, equal share of that list (split-K without a fixed split
//    size), so all SMs stay busy for any length mix.  A pair that spans
//    several warps leaves one (m, l, o) partial per warp; the reduce kernel
//    merges them by log-sum-exp.
//  * Each warp streams its tiles through its own ring of shared-memory stages
//    filled by bulk asynchronous copies (TMA, cp.async.bulk) completing on
//    mbarriers, so many KB per SM are in flight while it computes.
//  * The g = h_q / h_kv query heads sharing a kv head are processed together:
//    every cached byte is read once.  Scores S = K_hat q'^T and the product
//    P' V_hat run on mma.sync m16n8k16 with bf16 operands and fp32
//    accumulation: the integer codes are exact in bf16, the scale is folded
//    into the other operand (q' = q * s_channel for per-channel keys,
//    p' = p * s_token for per-token values) and that operand is split into
//    bf16 hi + lo columns (2 x 4 heads = the 8 columns of the mma), keeping 16
//    significant bits.  Zero-points enter as a per-group bias (keys) and a
//    p-weighted sum (values).  Codes are unpacked with one LOP3 + one bf16x2
//    FMA per pair of elements.
//  * Online softmax in the log2 domain with warp-shuffle reductions; the
//    running max is only moved when it grows by more than 8 (p <= 256).
#include <cstdint>

#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr uint32_t kWaitPolls = 1u << 20;

struct RowInfo {
  int seq;
  int qa;   // quantized positions attended
  int ra;   // residual positions attended
  int nq;   // quantized tiles
  int nr;   // residual tiles
  const int32_t* trow;
};

__device__ __forceinline__ RowInfo row_info(const DecodeArgs& a, int i, bool flag) {
  const Geo& g = a.g;
  RowInfo r;
  r.qa = r.ra = r.nq = r.nr = 0;
  r.trow = nullptr;
  const int seq = a.seqmap ? a.seqmap[i] : i;
  r.seq = seq;
  if (seq < 0 || seq >= g.max_seqs) {
    if (flag) atomicOr(a.err, KVQ_DEVERR_SEQ_ID);
    return r;
  }
  const int stored = a.stored_len[seq];
  int len = a.seq_lens[i];
  if (len < 0 || len > stored) {
    if (flag) atomicOr(a.err, KVQ_DEVERR_SEQ_LEN);
    len = min(max(len, 0), stored);
  }
  const int Lq = g.R ? (stored / g.R) * g.R : stored;
  r.qa = min(len, Lq);
  r.ra = max(0, len - Lq);
  r.nq = (r.qa + g.tileT - 1) / g.tileT;
  r.nr = (r.ra + 15) / 16;
  r.trow = a.table + int64_t(a.table_by_seq ? seq : i) * a.table_stride;
  return r;
}

// Exclusive prefix over s[1..n] (counts) -> s[0..n]; all threads participate.
__device__ void block_scan(int32_t* s, int n, int32_t* scratch) {
  const int T = blockDim.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int chunk = (n + T - 1) / T;
  const int lo = min(n, tid * chunk), hi = min(n, lo + chunk);
  int sum = 0;
  for (int j = lo; j < hi; ++j) sum += s[j + 1];
  int incl = sum;
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) scratch[w] = incl;
  __syncthreads();
  int base = 0;
  for (int k = 0; k < w; ++k) base += scratch[k];
  int run = base + incl - sum;
  for (int j = lo; j < hi; ++j) {
    run += s[j + 1];
    s[j + 1] = run;
  }
  if (tid == 0) s[0] = 0;
  __syncthreads();
}

struct It {
  int i, h, k, n;
};

__device__ __forceinline__ void it_seek(It& it, const int32_t* pre, int B, int hkv, int64_t u) {
  int lo = 0, hi = B;   // first j in [0, B] with pre[j] * hkv > u, minus one
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (int64_t(pre[mid + 1]) * hkv > u) hi = mid;
    else lo = mid + 1;
  }
  it.i = lo;
  it.n = pre[lo + 1] - pre[lo];
  const int64_t r = u - int64_t(pre[lo]) * hkv;
  it.h = int(r / it.n);
  it.k = int(r % it.n);
}

__device__ __forceinline__ bool it_next(It& it, const int32_t* pre, int B, int hkv) {
  if (++it.k < it.n) return false;
  it.k = 0;
  if (++it.h < hkv) return false;
  it.h = 0;
  do { ++it.i; } while (it.i < B && pre[it.i + 1] == pre[it.i]);
  if (it.i < B) it.n = pre[it.i + 1] - pre[it.i];
  return true;   // row changed
}

// Issue the bulk copies of one tile into a stage (lane 0 only).
template <int ASYM, int KAXIS>
__device__ void issue_tile(const DecodeArgs& a, const It& it, const RowInfo& ri, uint32_t dst,
                           uint32_t bar) {
  const Geo& g = a.g;
  if (it.k < ri.nq) {
    if (KAXIS) {
      const int npg = g.g_k / g.P;
      const int lb0 = it.k * npg;
      bool ok = lb0 + npg <= a.table_stride;
      for (int j = 0; ok && j < npg; ++j) {
        const int32_t b = ri.trow[lb0 + j];
        ok = b >= 0 && b < g.num_blocks;
      }
      if (!ok) {
        atomicOr(a.err, KVQ_DEVERR_BLOCK_ID);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      mbar_arrive_expect_tx(bar, uint32_t(npg * g.chunk_used));
      for (int j = 0; j < npg; ++j) {
        const uint8_t* src = a.pool + int64_t(ri.trow[lb0 + j]) * g.block_bytes +
                             int64_t(it.h) * g.chunk_bytes;
        bulk_g2s(dst + j * g.chunk_used, src, uint32_t(g.chunk_used), bar);
      }
    } else {
      const int T0 = 16 * it.k;
      const int lb = T0 / g.P, u = (T0 % g.P) / 16;
      const int32_t b = lb < a.table_stride ? ri.trow[lb] : -1;
      if (b < 0 || b >= g.num_blocks) {
        atomicOr(a.err, KVQ_DEVERR_BLOCK_ID);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint8_t* chunk = a.pool + int64_t(b) * g.block_bytes + int64_t(it.h) * g.chunk_bytes;
      if (g.P == 16) {
        mbar_arrive_expect_tx(bar, uint32_t(g.chunk_used));
        bulk_g2s(dst, chunk, uint32_t(g.chunk_used), bar);
      } else {
        const int vrow = 16 * g.nvg * g.es, krow = 16 * g.nkg * g.es;
        const uint32_t total = 2 * g.sub_bytes + (vrow + krow) * (1 + ASYM);
        mbar_arrive_expect_tx(bar, total);
        bulk_g2s(dst, chunk + u * g.sub_bytes, g.sub_bytes, bar);
        bulk_g2s(dst + g.sub_bytes, chunk + g.off_V + u * g.sub_bytes, g.sub_bytes, bar);
        const uint32_t vm = dst + 2 * g.sub_bytes, km = vm + g.vm16;
        bulk_g2s(vm, chunk + g.off_Vm + int64_t(16 * u) * g.nvg * g.es, vrow, bar);
        bulk_g2s(km, chunk + g.off_Km + int64_t(16 * u) * g.nkg * g.es, krow, bar);
        if (ASYM) {
          bulk_g2s(vm + vrow, chunk + g.off_Vm + int64_t(g.P + 16 * u) * g.nvg * g.es, vrow, bar);
          bulk_g2s(km + krow, chunk + g.off_Km + int64_t(g.P + 16 * u) * g.nkg * g.es, krow, bar);
        }
      }
    }
  } else {
    const int kr = it.k - ri.nq;
    const int64_t base = ((int64_t(ri.seq) * g.h_kv + it.h) * g.R + 16 * kr) * kD;
    mbar_arrive_expect_tx(bar, 2 * 16 * kD * 2);
    bulk_g2s(dst, a.kres + base, 16 * kD * 2, bar);
    bulk_g2s(dst + 16 * kD * 2, a.vres + base, 16 * kD * 2, bar);
  }
}

// Per-thread accumulation state of one (row, kv head) pair.
struct State {
  float o[8][4];     // channel tile i: (ch 16i+gq | +8) x (head tq hi | lo)
  float zacc[8];     // asymmetric values: p-weighted zero-point sums per tile
  float m, l;        // running max (log2 domain) and partial sum, head tq
};

__device__ __forceinline__ void state_reset(State& st) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int c = 0; c < 4; ++c) st.o[i][c] = 0.0f;
    st.zacc[i] = 0.0f;
  }
  st.m = -INFINITY;
  st.l = 0.0f;
}

// Online softmax over the two scores (tokens gq, gq+8; head tq) of a 16-token
// sub-tile; returns their weights p relative to the running max.
__device__ __forceinline__ void softmax_step(State& st, float s0, float s1, float& p0, float& p1) {
  float mx = fmaxf(s0, s1);
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
  if (mx > st.m + 8.0f) {   // also taken from -inf
    const float alpha = fast_exp2(st.m - mx);
    st.l *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
      for (int c = 0; c < 4; ++c) st.o[i][c] *= alpha;
      st.zacc[i] *= alpha;
    }
    st.m = mx;
  }
  const bool live = st.m != -INFINITY;
  p0 = live ? fast_exp2(s0 - st.m) : 0.0f;
  p1 = live ? fast_exp2(s1 - st.m) : 0.0f;
  st.l += p0 + p1;
}

// Scores of a 16-token sub-tile of packed keys: acc[] += K_hat q'^T for the
// k-steps of one key group; the caller folds groups.
template <int BITS, bool SGN>
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

// A operand (rows gq / gq+8, k-step j) of the score product from key words.
template <int BITS, bool SGN>
__device__ __forceinline__ void key_frag(const uint32_t (&wa)[BITS], const uint32_t (&wb)[BITS], int j,
                                         uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  if (BITS == 4) {
    const int jj = j >> 1, x = 2 * (j & 1);
    a0 = nib_pair<SGN>(wa[jj], x);
    a1 = nib_pair<SGN>(wb[jj], x);
    a2 = nib_pair<SGN>(wa[jj], x + 1);
    a3 = nib_pair<SGN>(wb[jj], x + 1);
  } else if (BITS == 2) {
    const int jj = j >> 2, x = 2 * (j & 3);
    a0 = crumb_pair<SGN>(wa[jj], x);
    a1 = crumb_pair<SGN>(wb[jj], x);
    a2 = crumb_pair<SGN>(wa[jj], x + 1);
    a3 = crumb_pair<SGN>(wb[jj], x + 1);
  } else {
    a0 = byte_pair<SGN>(wa[j], 0);
    a1 = byte_pair<SGN>(wb[j], 0);
    a2 = byte_pair<SGN>(wa[j], 1);
    a3 = byte_pair<SGN>(wb[j], 1);
  }
}

// A operand of the value product for channel tile i from a lane record.
template <int BITS, bool SGN>
__device__ __forceinline__ void value_frag(const uint32_t (&w)[2 * BITS], int i, uint32_t& a0,
                                           uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  if (BITS == 4) {
    a0 = nib_pair<SGN>(w[i], 0);
    a1 = nib_pair<SGN>(w[i], 1);
    a2 = nib_pair<SGN>(w[i], 2);
    a3 = nib_pair<SGN>(w[i], 3);
  } else if (BITS == 2) {
    const int b = 2 * (i & 1);
    a0 = crumb_pair<SGN>(w[i >> 1], b);
    a1 = crumb_pair<SGN>(w[i >> 1], b + 1);
    a2 = crumb_pair<SGN>(w[i >> 1], b + 4);
    a3 = crumb_pair<SGN>(w[i >> 1], b + 5);
  } else {
    a0 = byte_pair<SGN>(w[2 * i], 0);
    a1 = byte_pair<SGN>(w[2 * i], 1);
    a2 = byte_pair<SGN>(w[2 * i + 1], 0);
    a3 = byte_pair<SGN>(w[2 * i + 1], 1);
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

__device__ __forceinline__ float vmeta(const uint8_t* base, int idx, int es) {
  return es == 4 ? reinterpret_cast<const float*>(base)[idx]
                 : __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(base)[idx]));
}

// B operand (token rows 2tq, 2tq+1, 2tq+8, 2tq+9; column gq = head gq/2,
// hi|lo) of the value product, from the softmax weights pa0 (2tq), pb0
// (2tq+1), pa1 (2tq+8), pb1 (2tq+9) times each token's value scale.
__device__ __forceinline__ void pv_bfrag(float pa0, float pb0, float pa1, float pb1, float s0, float s1,
                                         float s2, float s3, bool lo, bool dead, uint32_t& b0,
                                         uint32_t& b1) {
  b0 = split_pack(pa0 * s0, pb0 * s1, lo);
  b1 = split_pack(pa1 * s2, pb1 * s3, lo);
  if (dead) b0 = b1 = 0u;
}

template <int BITS, int ASYM, int KAXIS>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int D = kD;
  constexpr bool SGN = !ASYM;
  extern __shared__ __align__(128) uint8_t smem[];
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int hh = gq >> 1;               // head of this lane's B column
  const bool is_lo = gq & 1;            // column carries the lo part
  const bool dead_col = hh >= g.G;      // padding column (fewer than 4 heads)

  int32_t* s_pre = reinterpret_cast<int32_t*>(smem);
  int32_t* s_scr = s_pre + (a.B + 1);
  uint8_t* my_stages = smem + a.pre_bytes + size_t(warp) * a.nstages * a.stage_bytes;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem + a.pre_bytes +
                                                  size_t(kDecodeWarps) * a.nstages * a.stage_bytes) +
                      warp * a.nstages;

  // ---- work list: tiles per row, prefix over rows -------------------------
  for (int i = tid; i < a.B; i += blockDim.x) {
    const RowInfo ri = row_info(a, i, blockIdx.x == 0);
    s_pre[i + 1] = ri.nq + ri.nr;
  }
  __syncthreads();
  block_scan(s_pre, a.B, s_scr);
  if (blockIdx.x == 0)
    for (int i = tid; i <= a.B; i += blockDim.x) a.prefix[i] = s_pre[i];

  const int64_t U = int64_t(s_pre[a.B]) * g.h_kv;
  const int gw = blockIdx.x * kDecodeWarps + warp;
  const int64_t u0 = int64_t(gw) * U / a.nw, u1 = int64_t(gw + 1) * U / a.nw;
  if (u0 >= u1) return;

  const uint32_t stage0 = smem_addr(my_stages);
  const uint32_t bar0 = smem_addr(my_bars);
  if (lane == 0) {
    for (int s = 0; s < a.nstages; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  __syncwarp();

  // ---- producer (lane 0): run ahead by nstages tiles ----------------------
  It pit;
  it_seek(pit, s_pre, a.B, g.h_kv, u0);
  RowInfo pri = row_info(a, pit.i, false);
  int64_t issued = u0;
  if (lane == 0) {
    for (int s = 0; s < a.nstages && issued < u1; ++s, ++issued) {
      issue_tile<ASYM, KAXIS>(a, pit, pri, stage0 + s * a.stage_bytes, bar0 + 8 * s);
      if (it_next(pit, s_pre, a.B, g.h_kv) && issued + 1 < u1) pri = row_info(a, pit.i, false);
    }
  }

  // ---- consumer (all lanes) -----------------------------------------------
  It cit;
  it_seek(cit, s_pre, a.B, g.h_kv, u0);
  RowInfo cri = row_info(a, cit.i, false);
  State st;
  state_reset(st);
  int cur_pair = -1;
  uint32_t bq[8][2];          // score B operand (q' hi|lo columns)
  float qf[KAXIS ? 32 : 1];   // channel axis: q of head hh at this lane's 32 channels
  float bias_t = 0.0f;        // channel-axis zero-point term of head tq (log2 units)
  const float C = a.qk_scale;

  auto load_q = [&](int row, int h, float* dst32) {
    const uint16_t* qrow = a.q + (int64_t(row) * g.h_q + h * g.G + min(hh, g.G - 1)) * D;
#pragma unroll
    for (int m = 0; m < 32; m += 2) {
      const uint32_t two = *reinterpret_cast<const uint32_t*>(qrow + key_channel(32 * tq + m));
      dst32[m] = __uint_as_float(two << 16);
      dst32[m + 1] = __uint_as_float(two & 0xFFFF0000u);
    }
  };
  // B operand from 32 fp32 values x[] in list order (4 per k-step)
  auto make_bq = [&](const float* x) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      bq[j][0] = dead_col ? 0u : split_pack(x[4 * j], x[4 * j + 1], is_lo);
      bq[j][1] = dead_col ? 0u : split_pack(x[4 * j + 2], x[4 * j + 3], is_lo);
    }
  };
  // token-axis asymmetric keys: sum of q over each key group, head tq
  float qsum[4] = {0.0f, 0.0f, 0.0f, 0.0f};

  auto emit = [&](int row, int h) {
    float l = st.l;
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    float zt[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float z = ASYM ? st.zacc[i] : 0.0f;
      if (ASYM) {
        z += __shfl_xor_sync(0xffffffffu, z, 4);
        z += __shfl_xor_sync(0xffffffffu, z, 8);
        z += __shfl_xor_sync(0xffffffffu, z, 16);
      }
      zt[i] = z;
    }
    if (tq < g.G) {
      const int64_t pair = int64_t(row) * g.h_kv + h;
      float* rec = a.partials + ((pair + gw) * g.G + tq) * (D + 2);
      if (gq == 0) {
        rec[0] = st.m;
        rec[1] = l;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        rec[2 + 16 * i + gq] = st.o[i][0] + st.o[i][1] + zt[i];
        rec[2 + 16 * i + gq + 8] = st.o[i][2] + st.o[i][3] + zt[i];
      }
    }
  };

  bool bq_holds_q = false;    // bq currently carries q itself (token axis, BF16 window)
  auto setup_pair = [&](int row, int h) {
    state_reset(st);
    bq_holds_q = !KAXIS;
    float qv[32];
    load_q(row, h, qv);
    if (KAXIS) {
#pragma unroll
      for (int m = 0; m < 32; ++m) qf[m] = qv[m];
    } else {
      make_bq(qv);
      if (ASYM) {
        // sum of q over each key group for head tq (token-axis zero-points)
        const uint16_t* qrow = a.q + (int64_t(row) * g.h_q + h * g.G + min(tq, g.G - 1)) * D;
        for (int gi = 0; gi < g.nkg; ++gi) {
          float s = 0.0f;
          for (int c = gi * g.g_k; c < (gi + 1) * g.g_k; ++c) s += bf16_bits_to_float(qrow[c]);
          qsum[gi] = s;
        }
      }
    }
  };

  const int mt_per_vg = g.g_v / 16;      // channel tiles per value group
  bool timed_out = false;

  for (int64_t u = u0; u < u1; ++u) {
    const int slot = int((u - u0) % a.nstages);
    const uint32_t parity = uint32_t(((u - u0) / a.nstages) & 1);
    const int pair_id = cit.i * g.h_kv + cit.h;
    if (pair_id != cur_pair) {
      if (cur_pair >= 0) emit(cur_pair / g.h_kv, cur_pair % g.h_kv);
      setup_pair(cit.i, cit.h);
      cur_pair = pair_id;
    }
    // every lane polls; the warp leaves together if any lane gave up
    const bool arrived = mbar_wait_bounded(bar0 + 8 * slot, parity, kWaitPolls);
    if (!__all_sync(0xffffffffu, arrived)) {
      timed_out = true;
      break;
    }
    const uint8_t* stg = my_stages + size_t(slot) * a.stage_bytes;

    if (cit.k < cri.nq) {
      // ------------------------- quantized tile -----------------------------
      const int nsub = KAXIS ? g.g_k / 16 : 1;
      const int tile_start = cit.k * g.tileT;
      if (KAXIS) {
        // q' = q * s_channel for this key group (scales striped over its pages)
        float xq[32];
        float zdot = 0.0f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int f0 = 32 * tq + 8 * c4;
          const uint8_t* km = stg + (f0 / g.kslice) * g.chunk_used + g.off_Km;
          const int off = f0 % g.kslice;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float s = vmeta(km, off + m, g.es);
            xq[8 * c4 + m] = qf[8 * c4 + m] * s;
            if (ASYM) zdot = fmaf(qf[8 * c4 + m], vmeta(km, g.kslice + off + m, g.es), zdot);
          }
        }
        make_bq(xq);
        bq_holds_q = false;
        if (ASYM) {
          zdot += __shfl_xor_sync(0xffffffffu, zdot, 1);
          zdot += __shfl_xor_sync(0xffffffffu, zdot, 2);
          bias_t = C * __shfl_sync(0xffffffffu, zdot, 8 * tq);   // lane (gq=2tq, 0): head tq
        }
      }
#pragma unroll 1
      for (int sb = 0; sb < nsub; ++sb) {
        const int pg = KAXIS ? sb / (g.P / 16) : 0;
        const int us = KAXIS ? sb % (g.P / 16) : 0;
        const uint8_t* cb = stg + pg * g.chunk_used;
        const uint8_t* ksub = cb + us * g.sub_bytes;
        const uint8_t* vsub = KAXIS ? cb + g.off_V + us * g.sub_bytes : stg + g.sub_bytes;
        const uint8_t* vms = KAXIS ? cb + g.off_Vm + 16 * us * g.nvg * g.es : stg + 2 * g.sub_bytes;
        const uint8_t* vmz = KAXIS ? cb + g.off_Vm + (g.P + 16 * us) * g.nvg * g.es
                                   : stg + 2 * g.sub_bytes + 16 * g.nvg * g.es;
        const uint8_t* kms = stg + 2 * g.sub_bytes + g.vm16;     // token axis only
        const uint8_t* kmz = kms + 16 * g.nkg * g.es;

        // scores
        uint32_t wa[BITS], wb[BITS];
        load_key_words<BITS, SGN>(ksub, gq, tq, wa, wb);
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float s0 = 0.0f, s1 = 0.0f;
        const int ks_per_group = KAXIS ? 8 : g.g_k / 16;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t a0, a1, a2, a3;
          key_frag<BITS, SGN>(wa, wb, j, a0, a1, a2, a3);
          mma_bf16(acc, a0, a1, a2, a3, bq[j][0], bq[j][1]);
          if ((j + 1) % ks_per_group == 0) {
            if (KAXIS) {
              s0 = acc[0] + acc[1];
              s1 = acc[2] + acc[3];
            } else {
              const int gi = j / ks_per_group;
              const float k0 = vmeta(kms, gq * g.nkg + gi, g.es);
              const float k1 = vmeta(kms, (gq + 8) * g.nkg + gi, g.es);
              s0 = fmaf(k0, acc[0] + acc[1], s0);
              s1 = fmaf(k1, acc[2] + acc[3], s1);
              if (ASYM) {
                s0 = fmaf(vmeta(kmz, gq * g.nkg + gi, g.es), qsum[gi & 3], s0);
                s1 = fmaf(vmeta(kmz, (gq + 8) * g.nkg + gi, g.es), qsum[gi & 3], s1);
              }
              acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
            }
          }
        }
        s0 = fmaf(s0, C, bias_t);
        s1 = fmaf(s1, C, bias_t);
        const int valid = cri.qa - (tile_start + 16 * sb);
        if (gq >= valid) s0 = -INFINITY;
        if (gq + 8 >= valid) s1 = -INFINITY;

        float p0, p1;
        softmax_step(st, s0, s1, p0, p1);

        // value product: P' V_hat, p' = p * s_value(token, group)
        const int sa = 8 * tq + hh, sbl = sa + 4;
        const float pa0 = __shfl_sync(0xffffffffu, p0, sa);
        const float pa1 = __shfl_sync(0xffffffffu, p1, sa);
        const float pb0 = __shfl_sync(0xffffffffu, p0, sbl);
        const float pb1 = __shfl_sync(0xffffffffu, p1, sbl);
        uint32_t vw[2 * BITS];
        load_value_words<BITS>(vsub, lane, vw);
        uint32_t b0 = 0, b1 = 0;
        float zs = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i % mt_per_vg == 0) {
            const int gi = i / mt_per_vg;
            const int n = g.nvg;
            pv_bfrag(pa0, pb0, pa1, pb1, vmeta(vms, (2 * tq) * n + gi, g.es),
                     vmeta(vms, (2 * tq + 1) * n + gi, g.es), vmeta(vms, (2 * tq + 8) * n + gi, g.es),
                     vmeta(vms, (2 * tq + 9) * n + gi, g.es), is_lo, dead_col, b0, b1);
            if (ASYM) zs = p0 * vmeta(vmz, gq * n + gi, g.es) + p1 * vmeta(vmz, (gq + 8) * n + gi, g.es);
          }
          uint32_t a0, a1, a2, a3;
          value_frag<BITS, SGN>(vw, i, a0, a1, a2, a3);
          mma_bf16(st.o[i], a0, a1, a2, a3, b0, b1);
          if (ASYM) st.zacc[i] += zs;
        }
      }
    } else {
      // ------------------------- BF16 residual tile -------------------------
      if (!bq_holds_q) {
        // B operand of q itself (exact in bf16: lo columns are zero)
        float qv[32];
        load_q(cit.i, cit.h, qv);
        make_bq(qv);
        bq_holds_q = true;
      }
      const uint32_t kaddr = smem_addr(stg), vaddr = kaddr + 16 * D * 2;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int mi = lane >> 3;   // matrix 0..3: (rows 0-7 | 8-15) x (cols 0-7 | 8-15)
        const int r = (lane & 7) + 8 * (mi & 1), c = 16 * j + 8 * (mi >> 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kaddr + (r * D + c) * 2, a0, a1, a2, a3);
        mma_bf16(acc, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      }
      float s0 = (acc[0] + acc[1]) * C, s1 = (acc[2] + acc[3]) * C;
      const int valid = cri.ra - 16 * (cit.k - cri.nq);
      if (gq >= valid) s0 = -INFINITY;
      if (gq + 8 >= valid) s1 = -INFINITY;
      float p0, p1;
      softmax_step(st, s0, s1, p0, p1);
      const int sa = 8 * tq + hh, sbl = sa + 4;
      const float pa0 = __shfl_sync(0xffffffffu, p0, sa);
      const float pa1 = __shfl_sync(0xffffffffu, p1, sa);
      const float pb0 = __shfl_sync(0xffffffffu, p0, sbl);
      const float pb1 = __shfl_sync(0xffffffffu, p1, sbl);
      uint32_t b0, b1;
      pv_bfrag(pa0, pb0, pa1, pb1, 1.0f, 1.0f, 1.0f, 1.0f, is_lo, dead_col, b0, b1);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int mi = lane >> 3;   // (tok 0-7 | 8-15) x (ch +0 | +8) -> a0..a3
        const int r = (lane & 7) + 8 * (mi >> 1), c = 16 * i + 8 * (mi & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vaddr + (r * D + c) * 2, a0, a1, a2, a3);
        mma_bf16(st.o[i], a0, a1, a2, a3, b0, b1);
      }
    }

    // release the stage and refill it with the tile nstages ahead
    fence_proxy_async();
    __syncwarp();
    if (lane == 0 && issued < u1) {
      issue_tile<ASYM, KAXIS>(a, pit, pri, stage0 + slot * a.stage_bytes, bar0 + 8 * slot);
      if (it_next(pit, s_pre, a.B, g.h_kv) && issued + 1 < u1) pri = row_info(a, pit.i, false);
      ++issued;
    }
    if (it_next(cit, s_pre, a.B, g.h_kv) && u + 1 < u1) cri = row_info(a, cit.i, false);
  }

  if (timed_out) {
    if (lane == 0) atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
    // drain this warp's copies still in flight (bounded), then leave
    for (int s = 0; s < a.nstages; ++s) {
      // parity of the most recent phase issued on stage s is unknown here;
      // poll both and stop at the limit
      (void)mbar_wait_bounded(bar0 + 8 * s, 0, kWaitPolls >> 4);
      (void)mbar_wait_bounded(bar0 + 8 * s, 1, kWaitPolls >> 4);
    }
    return;
  }
  if (cur_pair >= 0) emit(cur_pair / g.h_kv, cur_pair % g.h_kv);
}

// Merge the per-warp partials of each (row, kv head) by log-sum-exp.
__global__ void __launch_bounds__(128) reduce_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int D = kD;
  const Geo& g = a.g;
  const int p = blockIdx.x;
  const int i = p / g.h_kv, h = p % g.h_kv;
  const int32_t* pre = a.prefix;
  const int n = pre[i + 1] - pre[i];
  const int64_t U = int64_t(pre[a.B]) * g.h_kv;
  for (int idx = threadIdx.x; idx < g.G * D; idx += blockDim.x) {
    const int hd = idx / D, c = idx % D;
    float* out = a.out + (int64_t(i) * g.h_q + h * g.G + hd) * D + c;
    if (n == 0) {
      *out = 0.0f;
      continue;
    }
    // warps whose ranges hold this pair's tiles: start at the owner of its
    // first tile and jump from range end to range end (warps with empty
    // ranges in between own nothing and wrote nothing)
    const int64_t ua = int64_t(pre[i]) * g.h_kv + int64_t(h) * n, ub = ua + n - 1;
    const int64_t w0 = ((ua + 1) * a.nw - 1) / U, w1 = ((ub + 1) * a.nw - 1) / U;
    auto next_warp = [&](int64_t w) {
      const int64_t end = ((w + 1) * U) / a.nw;     // first tile after warp w's range
      return ((end + 1) * a.nw - 1) / U;
    };
    float M = -INFINITY;
    for (int64_t w = w0;; w = next_warp(w)) {
      M = fmaxf(M, a.partials[((p + w) * g.G + hd) * (D + 2)]);
      if (w >= w1) break;
    }
    float num = 0.0f, den = 0.0f;
    for (int64_t w = w0;; w = next_warp(w)) {
      const float* rec = a.partials + ((p + w) * g.G + hd) * (D + 2);
      const float sc = fast_exp2(rec[0] - M);
      den = fmaf(sc, rec[1], den);
      num = fmaf(sc, rec[2 + c], num);
      if (w >= w1) break;
    }
    *out = num / den;
  }
}

template <int BITS, int ASYM, int KAXIS>
const void* kernel_of() {
  return reinterpret_cast<const void*>(&decode_kernel<BITS, ASYM, KAXIS>);
}

}  // namespace

int decode_prefix_bytes(int B) { return ((B + 1 + 32) * 4 + 127) / 128 * 128; }

size_t decode_smem_bytes(int B, int nstages, int stage_bytes) {
  return size_t(decode_prefix_bytes(B)) + size_t(kDecodeWarps) * nstages * stage_bytes +
         size_t(kDecodeWarps) * nstages * 8;
}

const void* decode_kernel_ptr(const Geo& g) {
  const int key = (g.bits == 8 ? 0 : g.bits == 4 ? 1 : 2) * 4 + g.asym * 2 + g.k_axis;
  switch (key) {
    case 0: return kernel_of<8, 0, 0>();
    case 1: return kernel_of<8, 0, 1>();
    case 2: return kernel_of<8, 1, 0>();
    case 3: return kernel_of<8, 1, 1>();
    case 4: return kernel_of<4, 0, 0>();
    case 5: return kernel_of<4, 0, 1>();
    case 6: return kernel_of<4, 1, 0>();
    case 7: return kernel_of<4, 1, 1>();
    case 8: return kernel_of<2, 0, 0>();
    case 9: return kernel_of<2, 0, 1>();
    case 10: return kernel_of<2, 1, 0>();
    default: return kernel_of<2, 1, 1>();
  }
}

cudaError_t launch_decode(const DecodeArgs& a, int grid, size_t smem, cudaStream_t s,
                          cudaEvent_t between, int* launches) {
  const void* k = decode_kernel_ptr(a.g);
  void* args[] = {const_cast<DecodeArgs*>(&a)};
  cudaError_t e = cudaLaunchKernel(k, dim3(grid), dim3(kDecodeWarps * 32), args, smem, s);
  if (e != cudaSuccess) return e;
  ++*launches;
  if (between) {
    e = cudaEventRecord(between, s);
    if (e != cudaSuccess) return e;
  }
  const int pairs = a.B * a.g.h_kv;
  if (pairs == 0) return cudaSuccess;
  e = cudaLaunchKernel(reinterpret_cast<const void*>(&reduce_kernel), dim3(pairs), dim3(128), args, 0, s);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace kvq
