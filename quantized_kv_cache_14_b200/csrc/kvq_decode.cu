// kvq_decode.cu -- decode attention directly over the packed low-bit paged
// cache, dequantizing inside the kernel.
//
// Computes out = softmax(q K^T / sqrt(d_h)) V for one query token per
// sequence (llmdaily.org day-65, "Why the KV cache grows so quickly"), where K
// and V are the dequantized cache x_hat = s q (+ z) ("From BF16 to INT8, INT4,
// or even fewer bits") plus the BF16 window ("Why some systems keep a
// full-precision window"), read through the block table ("How this connects
// to paging and prefix caching").  The pages' trade-off -- memory traffic
// saved versus dequantization work ("Why compression may also improve speed";
// oh-bug.com, misconception 1) -- shapes the design:
//
//  * Work is a list of units per (row, kv head): quantized units of 64 tokens
//    (one key group when groups are longer), then the BF16 window in 16-token
//    tiles.  A persistent grid gives every CTA a contiguous, equal share of
//    the whole list (split-K whose split points come from balance), so all SMs
//    stay busy for any length mix.
//  * A CTA is four warps.  Warp w computes every fourth unit of the CTA's
//    share and stages its own units: two shared-memory stages per warp, each
//    filled by bulk asynchronous copies (TMA, cp.async.bulk) of whole page
//    chunks completing on the stage's mbarrier, issued two units ahead with
//    the block ids loaded one unit earlier still.
//  * The g = h_q / h_kv query heads sharing a kv head are processed together:
//    every cached byte is read once.  Scores K_hat q'^T and P' V_hat run on
//    mma.sync m16n8k16 with fp32 accumulation.  Codes are exact small integers
//    in fp16; the scale goes into the other operand (q' = q * s_channel per key
//    group, p' = p * s_token per value group), split into hi + lo parts that
//    take two of the 8 mma columns per head (4 heads x {hi, lo}).  Zero-points
//    enter as a per-group key bias and a p-weighted value sum.
//  * Online softmax in the log2 domain with warp-shuffle reductions, one step
//    per 64 tokens.  Each warp leaves one (m, l, o) record per pair its CTA
//    touched; the merge kernel combines them by log-sum-exp in a fixed order.
#include <cstdint>
#include <mutex>
#include <vector>

#include "kvq_device.cuh"
#include "kvq_tiles.cuh"

namespace kvq {
namespace {

constexpr uint64_t kWaitNs = 2000000000ull;   // give up on a copy after 2 s
// One warp's scratch: half of its q' operand in flight (32 lanes x 8 words), or
// the scores / weights of a 64-token chunk (8 x 32 floats); the two uses never
// overlap in time.
constexpr int kScratchBytes = 32 * 8 * 4;

struct SmemLayout {
  int stages, qbuf, bars, flag, total;
};

__host__ __device__ inline SmemLayout smem_layout(int B, const DecodePipe& p) {
  SmemLayout L;
  L.stages = ((B + 1 + 32 + 3 * B) * 4 + 127) / 128 * 128;   // prefix, scan scratch, per-row info
  L.qbuf = L.stages + p.nstages * p.stage_bytes;
  L.bars = L.qbuf + kDecodeWarps * kScratchBytes;
  L.flag = L.bars + p.nstages * 8;
  L.total = L.flag + 16;
  return L;
}

struct RowInfo {
  int seq;
  int qa;   // quantized positions attended
  int ra;   // window positions attended
  int nq;   // quantized units
  int nr;   // window tiles
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
  const int Lq = g.R ? (stored >> g.lg_gk) << g.lg_gk : stored;   // R == g_k
  r.qa = min(len, Lq);
  r.ra = max(0, len - Lq);
  r.nq = (r.qa + a.pipe.sup - 1) >> a.pipe.lg_sup;
  r.nr = (r.ra + 15) / 16;
  r.trow = a.table + int64_t(a.table_by_seq ? seq : i) * a.table_stride;
  return r;
}

// Exclusive prefix over s[1..n] (counts) -> s[0..n]; every thread of the CTA
// takes part.
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
  int lo = 0, hi = B;   // the row whose units hold u
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

// Bounded wait that also gives up as soon as another warp has aborted.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag) {
  return mbar_wait_bounded(bar, parity, kWaitNs, abort_flag);
}

// Per-thread accumulation state of one (row, kv head) pair.
struct State {
  float o[8][4];     // channel tile i: (ch 16i+gq | +8) x (head tq hi | lo)
  float zacc[8];     // asymmetric values: p-weighted zero-point sums per tile
  float zc[2][4];    // INT4 KIVI subnormal path: value offset terms per value group
  float m, l;        // running max (log2 domain) and partial sum, head tq
  bool raw;          // o holds subnormal-path sums not yet normalised
};

__device__ __forceinline__ void state_reset(State& st) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int c = 0; c < 4; ++c) st.o[i][c] = 0.0f;
    st.zacc[i] = 0.0f;
  }
#pragma unroll
  for (int gi = 0; gi < 2; ++gi)
#pragma unroll
    for (int c = 0; c < 4; ++c) st.zc[gi][c] = 0.0f;
  st.m = -INFINITY;
  st.l = 0.0f;
  st.raw = false;
}

// Where one 16-token sub-tile sits in a stage.
struct Sub {
  const uint8_t* k;     // key codes
  const uint8_t* v;     // value codes
  const uint8_t* vms;   // value scales, row 0 of the sub-tile; index r * nvg + group
  const uint8_t* vmz;   // value zero-points
  const uint8_t* kms;   // token-axis key scales, row 0; index r * nkg + group
  const uint8_t* kmz;
};

// The KIVI-style INT4 format (symmetric, keys per channel in groups of 64,
// values per token in groups of 64, fp16 scales, 16-token pages, a 64-token
// BF16 window, 4 query heads per kv head) gets its own kernel instance with
// every geometry field below a compile-time constant, so the per-sub-tile
// address arithmetic folds into immediates.  The host dispatches to it only
// when the runtime geometry equals these values field by field.
struct SpecInt4Kivi {
  static constexpr int bits = 4, asym = 0, k_axis = 1, g_k = 64, g_v = 64, scale_fp32 = 0, R = 64, P = 16, G = 4;
  static constexpr int n = 8, row_bytes = 64, sub_bytes = 1024, es = 2, nvg = 2, kslice = 32;
  static constexpr int off_V = 1024, off_Vm = 2048, off_Km = 2112, chunk_used = 2176;
  static constexpr int lg_P = 4, lg_gk = 6, lg_kslice = 5;
  static constexpr int ws_stages = 3;     // warp-specialised kernel: stages per warp pair
  static constexpr int unit_tokens = 64;  // its unit: one key group
};

// The INT2 asymmetric KIVI format (keys per channel G = 32, values per token
// G = 32, fp16 scale and zero-point, BF16 window 32, page 16, 4 query heads per
// kv head): only the warp-specialised kernel has a path of its own for it.
struct SpecInt2Kivi {
  static constexpr int bits = 2, asym = 1, k_axis = 1, g_k = 32, g_v = 32, scale_fp32 = 0, R = 32, P = 16, G = 4;
  static constexpr int n = 16, row_bytes = 32, sub_bytes = 512, es = 2, nvg = 4, kslice = 64;
  static constexpr int off_V = 512, off_Vm = 1024, off_Km = 1280, chunk_used = 1536;
  static constexpr int lg_P = 4, lg_gk = 5, lg_kslice = 6;
  static constexpr int ws_stages = 3;
  static constexpr int unit_tokens = 64;  // two key groups
};

// The INT8 format with keys and values per token (G = 128 = d_h: one fp16
// scale per token and head for each), no window, page 16, 4 query heads per
// kv head: the warp-specialised kernel takes units of 32 tokens (two pages of
// 4160 bytes) so that three stages per warp pair still fit two CTAs per SM.
struct SpecInt8Tok {
  static constexpr int bits = 8, asym = 0, k_axis = 0, g_k = 128, g_v = 128, scale_fp32 = 0, R = 0, P = 16, G = 4;
  static constexpr int n = 4, row_bytes = 128, sub_bytes = 2048, es = 2, nvg = 1, kslice = 0;
  static constexpr int off_V = 2048, off_Vm = 4096, off_Km = 4128, chunk_used = 4160;
  static constexpr int lg_P = 4, lg_gk = 7, lg_kslice = 0;
  static constexpr int ws_stages = 3;
  static constexpr int unit_tokens = 32;
};

template <int SPEC>
__device__ __forceinline__ Geo geo_of(const Geo& rt) {
  Geo g = rt;
  if constexpr (SPEC == 1) {
    using S = SpecInt4Kivi;
    g.bits = S::bits; g.asym = S::asym; g.k_axis = S::k_axis; g.g_k = S::g_k; g.g_v = S::g_v;
    g.scale_fp32 = S::scale_fp32; g.R = S::R; g.P = S::P; g.G = S::G; g.n = S::n;
    g.row_bytes = S::row_bytes; g.sub_bytes = S::sub_bytes; g.es = S::es; g.nvg = S::nvg;
    g.kslice = S::kslice; g.off_V = S::off_V; g.off_Vm = S::off_Vm; g.off_Km = S::off_Km;
    g.chunk_used = S::chunk_used; g.lg_P = S::lg_P; g.lg_gk = S::lg_gk; g.lg_kslice = S::lg_kslice;
  }
  return g;
}

template <class S>
bool spec_matches(const Geo& g) {
  return g.bits == S::bits && g.asym == S::asym && g.k_axis == S::k_axis && g.g_k == S::g_k &&
         g.g_v == S::g_v && g.scale_fp32 == S::scale_fp32 && g.R == S::R && g.P == S::P && g.G == S::G &&
         g.n == S::n && g.row_bytes == S::row_bytes && g.sub_bytes == S::sub_bytes && g.es == S::es &&
         g.nvg == S::nvg && g.kslice == S::kslice && g.off_V == S::off_V && g.off_Vm == S::off_Vm &&
         g.off_Km == S::off_Km && g.chunk_used == S::chunk_used && g.lg_P == S::lg_P && g.lg_gk == S::lg_gk &&
         g.lg_kslice == S::lg_kslice;
}

bool spec_int4_kivi(const Geo& g) { return spec_matches<SpecInt4Kivi>(g); }
bool spec_int2_kivi(const Geo& g) { return spec_matches<SpecInt2Kivi>(g); }
bool spec_int8_tok(const Geo& g) { return spec_matches<SpecInt8Tok>(g); }

template <int BITS, int ASYM, int KAXIS, int ES, int SPEC>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int D = kD;
  constexpr bool SGN = !ASYM;
  // The value product runs on fp16 operands when the stored scales are fp16:
  // with the running max exact (p <= 1), p' = p * s fits fp16's range.  Fp32
  // scales keep bf16 operands (fp32 range).
  // The FP8 format (ES == 1): e4m3 elements with one scale per kv head,
  // converted to fp16 operands; the scales are applied once per pair.
  constexpr bool F8 = ES == 1;
  constexpr bool PVH = ES == 2 || F8;
  // The BF16 control (16-bit "codes"): 16-token tiles of natural bf16 rows,
  // computed like the BF16 window.
  constexpr bool BF = BITS == 16;
  extern __shared__ __align__(128) uint8_t smem[];
  const Geo gs = geo_of<SPEC>(a.g);
  const Geo& g = SPEC ? gs : a.g;   // the generic instances read the geometry from the parameters
  const DecodePipe& pp = a.pipe;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SmemLayout L = smem_layout(a.B, pp);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem);
  int32_t* s_scr = s_pre + (a.B + 1);
  int32_t* s_row = s_scr + 32;   // per row: sequence, quantized and window positions attended
  uint8_t* stages = smem + L.stages;
  const uint32_t stage0 = smem_addr(stages);
  const uint32_t full0 = smem_addr(smem + L.bars);
  volatile int32_t* abort_flag = reinterpret_cast<int32_t*>(smem + L.flag);

  // Launched as a programmatic dependent of the previous kernel on the stream
  // (the append of a decode step): wait until that grid has completed and its
  // writes are visible before reading anything (returns at once when launched
  // plainly).  Then the merge grid may be scheduled; it waits for this one.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // ---- the work list: units per row, prefix over rows ---------------------
  for (int i = tid; i < a.B; i += blockDim.x) {
    const RowInfo ri = row_info(a, i, blockIdx.x == 0);
    s_pre[i + 1] = ri.nq + ri.nr;
    s_row[3 * i] = ri.seq;
    s_row[3 * i + 1] = ri.qa;
    s_row[3 * i + 2] = ri.ra;
  }
  if (tid == 0) {
    for (int s = 0; s < pp.nstages; ++s) mbar_init(full0 + 8 * s, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  block_scan(s_pre, a.B, s_scr);
  if (blockIdx.x == 0)
    for (int i = tid; i <= a.B; i += blockDim.x) a.prefix[i] = s_pre[i];

  const int64_t U = int64_t(s_pre[a.B]) * g.h_kv;
  const int64_t c0 = int64_t(blockIdx.x) * U / a.grid, c1 = int64_t(blockIdx.x + 1) * U / a.grid;
  if (c0 >= c1) return;
  const int N = int(c1 - c0);
  if (pp.nstages != kDecodeWarps && pp.nstages != 2 * kDecodeWarps) {   // stage indexing needs 4 or 8
    if (tid == 0) atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
    return;
  }

  // row info from the shared cache (no global reads after the prologue)
  auto rinfo = [&](int i) {
    RowInfo r;
    r.seq = s_row[3 * i];
    r.qa = s_row[3 * i + 1];
    r.ra = s_row[3 * i + 2];
    r.nq = (r.qa + pp.sup - 1) >> pp.lg_sup;
    r.nr = (r.ra + 15) >> 4;
    r.trow = a.table + int64_t(a.table_by_seq ? r.seq : i) * a.table_stride;
    return r;
  };
  // one unit forward; `n` counts units of the range, row info is refreshed
  // only while inside it
  auto step = [&](It& it, RowInfo& ri, int& n) {
    const bool row_changed = it_next(it, s_pre, a.B, g.h_kv);
    ++n;
    if (row_changed && n < N) ri = rinfo(it.i);
  };

  // four units forward at once when that stays inside one (row, head)
  auto advance4 = [&](It& it, RowInfo& ri, int& n) {
    if (it.k + kDecodeWarps < it.n) {
      it.k += kDecodeWarps;
      n += kDecodeWarps;
      return;
    }
    for (int t = 0; t < kDecodeWarps; ++t) step(it, ri, n);
  };

  // ---- staging: each warp fills its own two stages, two units ahead ---------
  // metadata rows of a 16-token sub-tile (none for FP8)
  const int vrow = F8 ? 0 : 16 * g.nvg * ES, krow = F8 ? 0 : 16 * g.nkg * ES;
  // this lane's block for the unit's copies (loaded early so the latency hides
  // under a unit of compute); -1 when out of the table
  auto load_blk = [&](const It& it, const RowInfo& ri) -> int32_t {
    if (it.k >= ri.nq) return 0;   // a BF16 window tile
    const int T0 = it.k * pp.sup;
    const int valid = min(pp.sup, ri.qa - T0);
    int pg, ncopy;
    if (BF) {
      ncopy = 2;                     // key tile and value tile of one page
      pg = T0 >> g.lg_P;
    } else if (KAXIS) {
      ncopy = ((valid + g.g_k - 1) >> g.lg_gk) << (g.lg_gk - g.lg_P);   // whole key groups
      pg = (T0 >> g.lg_P) + lane;
    } else {
      ncopy = (valid + 15) >> 4;
      pg = (T0 + 16 * min(lane, ncopy - 1)) >> g.lg_P;
    }
    if (lane >= ncopy) return 0;
    return pg < a.table_stride ? ri.trow[pg] : -1;
  };
  auto issue = [&](const It& it, const RowInfo& ri, int32_t blk, int sidx) {
    constexpr uint32_t FULL = 0xffffffffu;
    const uint32_t dst = stage0 + sidx * pp.stage_bytes;
    const uint32_t bar = full0 + 8 * sidx;
    uint32_t total;
    int ncopy, tok = 0;
    const bool window = it.k >= ri.nq;
    if (!window) {
      const int T0 = it.k * pp.sup;
      const int valid = min(pp.sup, ri.qa - T0);
      if (BF) {
        ncopy = 2;
        total = 2 * 16 * kD * 2;
        tok = T0;
      } else if (KAXIS) {
        ncopy = ((valid + g.g_k - 1) >> g.lg_gk) << (g.lg_gk - g.lg_P);
        total = uint32_t(ncopy * g.chunk_used);
      } else {
        ncopy = (valid + 15) >> 4;
        total = uint32_t(ncopy) * (g.P == 16 ? uint32_t(g.chunk_used)
                                             : uint32_t(2 * g.sub_bytes + (vrow + krow) * (1 + ASYM)));
        tok = T0 + 16 * min(lane, ncopy - 1);
      }
    } else {
      ncopy = 2;
      total = 2 * 16 * kD * 2;
    }
    bool bad = !window && __any_sync(FULL, lane < ncopy && (blk < 0 || blk >= g.num_blocks));
    bool dbad = false;
    if (KVQ_DEBUG && !bad) {
      // the copies fit the stage, and a window tile's rows lie in the window
      dbad = !dcheck(total <= uint32_t(pp.stage_bytes), a.err, KVQ_DEVERR_SMEM) ||
             !dcheck(!window || (ri.seq >= 0 && ri.seq < g.max_seqs && 16 * (it.k - ri.nq) + 16 <= g.R), a.err,
                     KVQ_DEVERR_INDEX);
      dbad = __any_sync(FULL, dbad);
    }
    // this warp's generic-proxy reads of the stage come before the copies' writes
    fence_proxy_async();
    if (bad || dbad) {
      if (lane == 0) {
        if (bad) atomicOr(a.err, KVQ_DEVERR_BLOCK_ID);
        mbar_arrive_expect_tx(bar, 0);
      }
      return;
    }
    if (lane == 0) mbar_arrive_expect_tx(bar, total);
    __syncwarp();
    if (lane >= ncopy) return;
    if (window) {
      const int kr = it.k - ri.nq;
      const int64_t base = ((int64_t(ri.seq) * g.h_kv + it.h) * g.R + 16 * kr) * kD;
      bulk_g2s(dst + lane * (16 * kD * 2), (lane ? a.vres : a.kres) + base, 16 * kD * 2, bar);
      return;
    }
    const uint8_t* chunk = a.pool + int64_t(blk) * g.block_bytes + int64_t(it.h) * g.chunk_bytes;
    if (BF) {
      const int u = (tok & (g.P - 1)) >> 4;
      bulk_g2s(dst + lane * (16 * kD * 2), chunk + (lane ? g.off_V : 0) + int64_t(u) * g.sub_bytes, 16 * kD * 2, bar);
    } else if (KAXIS) {
      bulk_g2s(dst + lane * g.chunk_used, chunk, uint32_t(g.chunk_used), bar);
    } else if (g.P == 16) {
      bulk_g2s(dst + lane * pp.qsub, chunk, uint32_t(g.chunk_used), bar);
    } else {
      const int u = (tok & (g.P - 1)) >> 4;
      const uint32_t d = dst + lane * pp.qsub;
      bulk_g2s(d, chunk + u * g.sub_bytes, g.sub_bytes, bar);
      bulk_g2s(d + g.sub_bytes, chunk + g.off_V + u * g.sub_bytes, g.sub_bytes, bar);
      const uint32_t vm = d + 2 * g.sub_bytes, km = vm + g.vm16;
      if (!F8) {
        bulk_g2s(vm, chunk + g.off_Vm + int64_t(16 * u) * g.nvg * ES, vrow, bar);
        bulk_g2s(km, chunk + g.off_Km + int64_t(16 * u) * g.nkg * ES, krow, bar);
      }
      if (ASYM) {
        bulk_g2s(vm + vrow, chunk + g.off_Vm + int64_t(g.P + 16 * u) * g.nvg * ES, vrow, bar);
        bulk_g2s(km + krow, chunk + g.off_Km + int64_t(g.P + 16 * u) * g.nkg * ES, krow, bar);
      }
    }
  };

  // ------------------------------ consumers -----------------------------------
  // Consumer warp w owns the units n of the range with n % 4 == w: it waits for
  // the unit's stage, computes all of it alone and releases the stage.  It
  // walks every unit of the range to see the pair boundaries, so it leaves one
  // (m, l, o) record for every pair the CTA touches (empty where it owned no
  // unit of the pair), which is what the merge reads.
  const int gq = lane >> 2, tq = lane & 3;
  const int hh = gq >> 1;               // head of this lane's B column
  const bool is_lo = gq & 1;            // the column carries the lo part
  const bool dead_col = hh >= g.G;      // padding column (fewer than 4 heads)
  const float C = a.qk_scale;
  const int vg_shift = __ffs(g.g_v >> 4) - 1;               // channel tiles per value group, log2
  const int kg_shift = KAXIS ? 3 : __ffs(g.g_k >> 4) - 1;   // k-steps per key group, log2
  uint32_t* qbw = reinterpret_cast<uint32_t*>(smem + L.qbuf + warp * kScratchBytes);   // this warp's scratch
  float* spw = reinterpret_cast<float*>(qbw);

  State st;
  state_reset(st);
  uint32_t bq[8][2];          // score B operand: fp16 q' hi|lo columns, fp16 q, or bf16 q (window)
  bool bq_bf16 = false;       // bq carries bf16 q for the BF16 window
  float cs = C;               // score scale: C times the power of two taken out of the fp16 operand
  float vscale = 1.0f;        // FP8: the pair's value scale, applied to its record
  float bias_t = 0.0f;        // channel-axis zero-points: key bias of head tq for the loaded group
  uint32_t qw[4][2];          // channel axis: q of head h at key-list channels 4*lane .. 4*lane+3
  uint32_t qh[4][2];          // the same as fp16, scaled by a power of two per pair (fp16 scales)
  float qsum[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // token-axis zero-points: sum of q per key group

  auto qrow = [&](int row, int h, int head) {
    return a.q + (int64_t(row) * g.h_q + h * g.G + min(head, g.G - 1)) * D;
  };
  auto load_bq_from_q = [&](int row, int h) {
    const uint16_t* qr = qrow(row, h, hh);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t t0 = *reinterpret_cast<const uint32_t*>(qr + key_channel(32 * tq + 4 * j));
      const uint32_t t1 = *reinterpret_cast<const uint32_t*>(qr + key_channel(32 * tq + 4 * j + 2));
      // q is exact in bf16: its hi part is q itself and its lo part is zero
      bq[j][0] = (dead_col || is_lo) ? 0u : t0;
      bq[j][1] = (dead_col || is_lo) ? 0u : t1;
    }
  };

  // Token axis: q itself as the fp16 operand, scaled by a power of two per pair
  // so the largest |q| of the kv head's query heads lies in [2^14, 2^15).
  auto load_bq_f16 = [&](int row, int h) {
    load_bq_from_q(row, h);
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(bq[j][e] << 16)), fabsf(__uint_as_float(bq[j][e] & 0xFFFF0000u))));
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int ex = amax > 0.0f ? min(max(int((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 14, -100), 100) : 0;
    const float down = pow2f(-ex);
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const __half2 hq = __floats2half2_rn(__uint_as_float(bq[j][e] << 16) * down,
                                             __uint_as_float(bq[j][e] & 0xFFFF0000u) * down);
        bq[j][e] = *reinterpret_cast<const uint32_t*>(&hq);
      }
    cs = C * pow2f(ex);
    return down;
  };

  // subnormal-path sums -> ordinary sums: drop the offset terms, undo the
  // 2^-24 (rows gq) and 2^-20 (rows gq + 8) scales
  auto normalize = [&]() {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int gi = i >> 2;
      st.o[i][0] = (st.o[i][0] - st.zc[gi][0]) * 16777216.0f;
      st.o[i][1] = (st.o[i][1] - st.zc[gi][1]) * 16777216.0f;
      st.o[i][2] = (st.o[i][2] - st.zc[gi][2]) * 1048576.0f;
      st.o[i][3] = (st.o[i][3] - st.zc[gi][3]) * 1048576.0f;
    }
#pragma unroll
    for (int gi = 0; gi < 2; ++gi)
#pragma unroll
      for (int c = 0; c < 4; ++c) st.zc[gi][c] = 0.0f;
    st.raw = false;
  };

  auto emit = [&](int row, int h) {
    if (SPEC && st.raw) normalize();
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
    if (tq < g.G && dcheck(int64_t(row) * g.h_kv + h + blockIdx.x < int64_t(a.B) * g.h_kv + a.grid, a.err,
                           KVQ_DEVERR_INDEX)) {
      const int64_t pair = int64_t(row) * g.h_kv + h;
      float* rec = a.partials + (((pair + blockIdx.x) * kDecodeWarps + warp) * g.G + tq) * (D + 2);
      if (gq == 0) {
        rec[0] = st.m;
        rec[1] = l;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        rec[2 + 16 * i + gq] = (st.o[i][0] + st.o[i][1] + zt[i]) * vscale;
        rec[2 + 16 * i + gq + 8] = (st.o[i][2] + st.o[i][3] + zt[i]) * vscale;
      }
    }
  };

  auto setup_pair = [&](int row, int h) {
    state_reset(st);
    bq_bf16 = false;
    bias_t = 0.0f;
    if (KAXIS) {
      // this lane's share of the q' job: key-list channels 4*lane .. 4*lane+3 of every head
      const int f = 4 * lane;
#pragma unroll
      for (int h2 = 0; h2 < 4; ++h2) {
        const uint16_t* qr = qrow(row, h, h2);
        const bool live = h2 < g.G;
        qw[h2][0] = live ? *reinterpret_cast<const uint32_t*>(qr + key_channel(f)) : 0u;
        qw[h2][1] = live ? *reinterpret_cast<const uint32_t*>(qr + key_channel(f + 2)) : 0u;
      }
      if (ES == 2) {
        // q as fp16 with the largest |q| of the pair in [1/2, 1): then
        // q * s stays below 65504 for every fp16 scale s.  The subnormal-code
        // path multiplies half of q by 16, so it takes [2^-5, 2^-4) instead.
        float amax = 0.0f;
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(qw[h2][e] << 16)),
                                     fabsf(__uint_as_float(qw[h2][e] & 0xFFFF0000u))));
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int ex = amax > 0.0f ? min(max(int((__float_as_uint(amax) >> 23) & 0xFF) - 127 + (SPEC ? 5 : 1), -100), 100)
                                   : 0;
        const float down = pow2f(-ex);
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const __half2 v = __floats2half2_rn(__uint_as_float(qw[h2][e] << 16) * down,
                                                __uint_as_float(qw[h2][e] & 0xFFFF0000u) * down);
            qh[h2][e] = *reinterpret_cast<const uint32_t*>(&v);
          }
        cs = C * pow2f(ex);
      }
    } else if (BF) {
      load_bq_from_q(row, h);
      bq_bf16 = true;
    } else {
      const float down = load_bq_f16(row, h);
      if (F8) {
        cs *= a.fp8[h];             // keys: s_k[h] times the scores
        vscale = a.fp8[g.h_kv + h]; // values: s_v[h] times the weighted sum
      }
      if (ASYM) {
        // in the operand's scaled domain, like the products it is added to
        const uint16_t* qr = qrow(row, h, tq);
        for (int gi = 0; gi < g.nkg; ++gi) {
          float s = 0.0f;
          for (int c = gi * g.g_k; c < (gi + 1) * g.g_k; ++c) s += bf16_bits_to_float(qr[c]);
          qsum[gi & 3] = s * down;
        }
      }
    }
  };

  // Channel axis: q' = q * s_channel of key group gi of the unit in `stg`, as
  // this lane's score B operand.  Each lane scales 4 channels of every head and
  // writes both bf16 parts into the warp's buffer in operand order (16-byte
  // slots XOR-swizzled so the four 16-byte reads per lane are conflict-free).
  auto qprime_job = [&](const uint8_t* stg, int gi, bool b0x16 = false) {
    const int f = 4 * lane;
    const int lg_ppg = g.lg_gk - g.lg_P;   // pages per key group, log2
    const uint8_t* km = stg + ((gi << lg_ppg) + (f >> g.lg_kslice)) * g.chunk_used + g.off_Km;
    const int off = f & (g.kslice - 1);
    const int t0 = lane >> 3, j = lane & 7;
    uint32_t qv[4][4];   // per head: hi pair, hi pair, lo pair, lo pair of this lane's 4 channels
    auto put = [&](int h2, uint32_t h0, uint32_t h1, uint32_t l0, uint32_t l1) {
      qv[h2][0] = h0; qv[h2][1] = h1; qv[h2][2] = l0; qv[h2][3] = l1;
    };
    // Lane L's values of head h belong to lanes (gq = 2h | 2h + 1, tq = L / 8),
    // k-step L % 8.  Two passes over the 1 KB scratch move k-steps 0-3, then
    // 4-7; each reader's 8 words are two 16-byte slots, XOR-swizzled so the
    // reads are conflict-free.
    auto transpose = [&]() {
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        __syncwarp();   // the scratch is free
        if ((j >> 2) == pass) {
          const int j4 = j & 3;
#pragma unroll
          for (int h2 = 0; h2 < 4; ++h2) {
            const int thi = 8 * h2 + t0, tlo = thi + 4;
            *reinterpret_cast<uint2*>(qbw + thi * 8 + 4 * ((j4 >> 1) ^ ((thi >> 2) & 1)) + 2 * (j4 & 1)) =
                make_uint2(qv[h2][0], qv[h2][1]);
            *reinterpret_cast<uint2*>(qbw + tlo * 8 + 4 * ((j4 >> 1) ^ ((tlo >> 2) & 1)) + 2 * (j4 & 1)) =
                make_uint2(qv[h2][2], qv[h2][3]);
          }
        }
        __syncwarp();
        const uint4* qb = reinterpret_cast<const uint4*>(qbw + lane * 8);
        const int sw = (lane >> 2) & 1;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const uint4 x = qb[v ^ sw];
          bq[4 * pass + 2 * v][0] = x.x; bq[4 * pass + 2 * v][1] = x.y;
          bq[4 * pass + 2 * v + 1][0] = x.z; bq[4 * pass + 2 * v + 1][1] = x.w;
        }
      }
      __syncwarp();   // all reads done before the scratch holds scores
      bq_bf16 = false;
    };
    if constexpr (ES == 2) {
      // fp16 scales: q'_hi = f16(q s) and q'_lo = f16(q s - q'_hi) by one fp16
      // multiply and one fp16 FMA per pair (the FMA's residual is exact, so
      // q'_hi + q'_lo = q s exactly unless a part underflows)
      const uint2 sr = *reinterpret_cast<const uint2*>(km + off * 2);
      const __half2 s01 = *reinterpret_cast<const __half2*>(&sr.x), s23 = *reinterpret_cast<const __half2*>(&sr.y);
#pragma unroll
      for (int h2 = 0; h2 < 4; ++h2) {
        // key-list positions 4L, 4L + 1 feed the b0 register of the score
        // product; the subnormal path wants them 16 times larger (exact)
        const __half2 qa = b0x16 ? __hmul2(*reinterpret_cast<const __half2*>(&qh[h2][0]), __float2half2_rn(16.0f))
                                 : *reinterpret_cast<const __half2*>(&qh[h2][0]);
        const __half2 qb = *reinterpret_cast<const __half2*>(&qh[h2][1]);
        const __half2 ha = __hmul2(qa, s01), hb = __hmul2(qb, s23);
        const __half2 la = __hfma2(qa, s01, __hneg2(ha)), lb = __hfma2(qb, s23, __hneg2(hb));
        put(h2, *reinterpret_cast<const uint32_t*>(&ha), *reinterpret_cast<const uint32_t*>(&hb),
            *reinterpret_cast<const uint32_t*>(&la), *reinterpret_cast<const uint32_t*>(&lb));
      }
      if (ASYM) {
        const uint2 zr = *reinterpret_cast<const uint2*>(km + (g.kslice + off) * 2);
        const float2 z01 = __half22float2(*reinterpret_cast<const __half2*>(&zr.x));
        const float2 z23 = __half22float2(*reinterpret_cast<const __half2*>(&zr.y));
        float dz[4];
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {
          dz[h2] = __uint_as_float(qw[h2][0] << 16) * z01.x + __uint_as_float(qw[h2][0] & 0xFFFF0000u) * z01.y +
                   __uint_as_float(qw[h2][1] << 16) * z23.x + __uint_as_float(qw[h2][1] & 0xFFFF0000u) * z23.y;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) dz[h2] += __shfl_xor_sync(0xffffffffu, dz[h2], o);
        }
        const int ht = min(tq, g.G - 1);
        bias_t = C * (ht == 0 ? dz[0] : ht == 1 ? dz[1] : ht == 2 ? dz[2] : dz[3]);
      }
      transpose();
      return;
    }
    float sc[4];
    meta4(km, off, ES, sc);
    float zc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (ASYM) meta4(km, g.kslice + off, ES, zc);
    float dz[4];
    float x[4][4];
    float amax = 0.0f;
#pragma unroll
    for (int h2 = 0; h2 < 4; ++h2) {
      const float q0 = __uint_as_float(qw[h2][0] << 16), q1 = __uint_as_float(qw[h2][0] & 0xFFFF0000u);
      const float q2 = __uint_as_float(qw[h2][1] << 16), q3 = __uint_as_float(qw[h2][1] & 0xFFFF0000u);
      x[h2][0] = q0 * sc[0]; x[h2][1] = q1 * sc[1]; x[h2][2] = q2 * sc[2]; x[h2][3] = q3 * sc[3];
#pragma unroll
      for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(x[h2][e]));
      if (ASYM) dz[h2] = q0 * zc[0] + q1 * zc[1] + q2 * zc[2] + q3 * zc[3];
    }
    // one power of two per group puts the largest |q'| in [2^14, 2^15)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int ex = amax > 0.0f ? min(max(int((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 14, -100), 100) : 0;
    const float down = pow2f(-ex);
    cs = C * pow2f(ex);
#pragma unroll
    for (int h2 = 0; h2 < 4; ++h2) {
      uint32_t h0, l0, h1, l1;
      split2h(x[h2][0] * down, x[h2][1] * down, h0, l0);
      split2h(x[h2][2] * down, x[h2][3] * down, h1, l1);
      put(h2, h0, h1, l0, l1);
    }
    if (ASYM) {
#pragma unroll
      for (int h2 = 0; h2 < 4; ++h2)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) dz[h2] += __shfl_xor_sync(0xffffffffu, dz[h2], o);
      const int ht = min(tq, g.G - 1);
      bias_t = C * (ht == 0 ? dz[0] : ht == 1 ? dz[1] : ht == 2 ? dz[2] : dz[3]);
    }
    transpose();
  };

  // Scores of one 16-token quantized sub-tile: tokens gq, gq + 8 for head tq,
  // scaled into the log2 domain; positions at or past `valid` are -inf.
  auto score_sub = [&](const Sub& sb, int valid, float& s0, float& s1, bool one_chain = false) {
    uint32_t wa[BITS], wb[BITS];
    load_key_words<BITS>(sb.k, gq, tq, wa, wb);
    float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float r0 = 0.0f, r1 = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t a0, a1, a2, a3;
      if (F8) {
        a0 = fp8x2_to_h2(wa[j]);
        a1 = fp8x2_to_h2(wb[j]);
        a2 = fp8x2_to_h2(wa[j] >> 16);
        a3 = fp8x2_to_h2(wb[j] >> 16);
      } else {
        key_frag<BITS, SGN, true>(wa, wb, j, a0, a1, a2, a3);
      }
      if ((j & 1) && !one_chain) mma_f16(acc1, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      else mma_f16(acc0, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      if (!KAXIS && !F8 && ((j + 1) & ((1 << kg_shift) - 1)) == 0) {
        const int gi = j >> kg_shift;
        const float t0 = acc0[0] + acc0[1] + acc1[0] + acc1[1];
        const float t1 = acc0[2] + acc0[3] + acc1[2] + acc1[3];
        r0 = fmaf(meta_at(sb.kms, gq * g.nkg + gi, ES), t0, r0);
        r1 = fmaf(meta_at(sb.kms, (gq + 8) * g.nkg + gi, ES), t1, r1);
        if (ASYM) {
          r0 = fmaf(meta_at(sb.kmz, gq * g.nkg + gi, ES), qsum[gi & 3], r0);
          r1 = fmaf(meta_at(sb.kmz, (gq + 8) * g.nkg + gi, ES), qsum[gi & 3], r1);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) acc0[c] = acc1[c] = 0.0f;
      }
    }
    if (one_chain) {
      r0 = acc0[0] + acc0[1];
      r1 = acc0[2] + acc0[3];
    } else if (KAXIS || F8) {
      r0 = acc0[0] + acc0[1] + acc1[0] + acc1[1];
      r1 = acc0[2] + acc0[3] + acc1[2] + acc1[3];
    }
    s0 = gq < valid ? fmaf(r0, cs, bias_t) : -INFINITY;
    s1 = gq + 8 < valid ? fmaf(r1, cs, bias_t) : -INFINITY;
  };

  // Value product of one sub-tile: P' V_hat with p' = p * s_value(token, group).
  auto pv_sub = [&](const Sub& sb, float p0, float p1, bool live) {
    const int sa = 8 * tq + hh, sbl = sa + 4;
    const float pa0 = __shfl_sync(0xffffffffu, p0, sa);
    const float pa1 = __shfl_sync(0xffffffffu, p1, sa);
    const float pb0 = __shfl_sync(0xffffffffu, p0, sbl);
    const float pb1 = __shfl_sync(0xffffffffu, p1, sbl);
    uint32_t vw[2 * BITS];
    load_value_words<BITS>(sb.v, lane, vw);
    const int n = g.nvg;
    uint32_t b0 = 0, b1 = 0;
    float zs = 0.0f;
    // fp16 value product: p = p_hi + p_lo in fp16 once per sub-tile; per value
    // group p' = p s is then f16(p_hi s) plus f16(p_lo s + the exact residual
    // of p_hi s), one multiply and two FMAs per pair (relative error 2^-21)
    uint32_t pha = 0, pla = 0, phb = 0, plb = 0;
    if (PVH) {
      split2h(pa0, pb0, pha, pla);
      split2h(pa1, pb1, phb, plb);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & ((1 << vg_shift) - 1)) == 0) {
        const int gi = i >> vg_shift;
        uint32_t h0, l0, h1, l1;
        if (F8) {   // one value scale per head, applied to the record: p' = p
          h0 = pha; l0 = pla; h1 = phb; l1 = plb;
        } else if (PVH) {
          const uint16_t* vs = reinterpret_cast<const uint16_t*>(sb.vms);
          __half2 sa2, sb2;
          if (n == 2) {
            // rows 2tq, 2tq + 1 (and + 8) hold both groups' scales in 8 bytes
            const uint2 ra = *reinterpret_cast<const uint2*>(vs + 4 * tq);
            const uint2 rb = *reinterpret_cast<const uint2*>(vs + 4 * tq + 16);
            const uint32_t sel = gi ? 0x7632u : 0x5410u;
            const uint32_t xa = __byte_perm(ra.x, ra.y, sel), xb = __byte_perm(rb.x, rb.y, sel);
            sa2 = *reinterpret_cast<const __half2*>(&xa);
            sb2 = *reinterpret_cast<const __half2*>(&xb);
          } else {
            sa2 = __halves2half2(__ushort_as_half(vs[(2 * tq) * n + gi]), __ushort_as_half(vs[(2 * tq + 1) * n + gi]));
            sb2 = __halves2half2(__ushort_as_half(vs[(2 * tq + 8) * n + gi]),
                                 __ushort_as_half(vs[(2 * tq + 9) * n + gi]));
          }
          auto two = [](uint32_t ph, uint32_t pl, __half2 sv, uint32_t& hi, uint32_t& lo) {
            const __half2 a = *reinterpret_cast<const __half2*>(&ph), b = *reinterpret_cast<const __half2*>(&pl);
            const __half2 h = __hmul2(a, sv);
            const __half2 l = __hfma2(b, sv, __hfma2(a, sv, __hneg2(h)));
            hi = *reinterpret_cast<const uint32_t*>(&h);
            lo = *reinterpret_cast<const uint32_t*>(&l);
          };
          two(pha, pla, sa2, h0, l0);
          two(phb, plb, sb2, h1, l1);
        } else {
          const float x0 = pa0 * meta_at(sb.vms, (2 * tq) * n + gi, ES);
          const float x1 = pb0 * meta_at(sb.vms, (2 * tq + 1) * n + gi, ES);
          const float x2 = pa1 * meta_at(sb.vms, (2 * tq + 8) * n + gi, ES);
          const float x3 = pb1 * meta_at(sb.vms, (2 * tq + 9) * n + gi, ES);
          split2(x0, x1, h0, l0);
          split2(x2, x3, h1, l1);
        }
        b0 = (dead_col || !live) ? 0u : (is_lo ? l0 : h0);
        b1 = (dead_col || !live) ? 0u : (is_lo ? l1 : h1);
        if (ASYM)
          zs = live ? p0 * meta_at(sb.vmz, gq * n + gi, ES) + p1 * meta_at(sb.vmz, (gq + 8) * n + gi, ES)
                    : 0.0f;
      }
      uint32_t a0, a1, a2, a3;
      if (F8) {
        a0 = fp8x2_to_h2(vw[2 * i]);
        a1 = fp8x2_to_h2(vw[2 * i] >> 16);
        a2 = fp8x2_to_h2(vw[2 * i + 1]);
        a3 = fp8x2_to_h2(vw[2 * i + 1] >> 16);
      } else {
        value_frag<BITS, SGN, PVH>(vw, i, a0, a1, a2, a3);
      }
      if (PVH) mma_f16(st.o[i], a0, a1, a2, a3, b0, b1);
      else mma_bf16(st.o[i], a0, a1, a2, a3, b0, b1);
      if (ASYM) st.zacc[i] += zs;
    }
  };

  // Online softmax over up to 64 tokens (4 sub-tiles x 2 scores per lane).
  auto softmax_chunk = [&](const float (&s)[8], float (&p)[8]) {
    float mx = fmaxf(fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3])), fmaxf(fmaxf(s[4], s[5]), fmaxf(s[6], s[7])));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (mx > st.m) {   // also taken from -inf; keeps p <= 1
      const float alpha = fast_exp2(st.m - mx);
      st.l *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int c = 0; c < 4; ++c) st.o[i][c] *= alpha;
        st.zacc[i] *= alpha;
      }
      if (SPEC) {
#pragma unroll
        for (int gi = 0; gi < 2; ++gi)
#pragma unroll
          for (int c = 0; c < 4; ++c) st.zc[gi][c] *= alpha;
      }
      st.m = mx;
    }
    const bool live = st.m != -INFINITY;
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      p[k] = live ? fast_exp2(s[k] - st.m) : 0.0f;
      sum += p[k];
    }
    st.l += sum;
  };

  // ---- INT4 KIVI, whole 64-token units: codes as fp16 subnormals ----------
  // A nibble masked into the low mantissa bits of an fp16 half, exponent field
  // zero, is the subnormal u * 2^-24 (bits 0-3) or u * 2^-20 (bits 4-7), u the
  // field read as unsigned: one LOP3 per operand register, no FMA.  Flipping
  // the field's top bit makes u = code + 8.  The constant 8 is removed exactly
  // by the same products over all-zero codes (u = 8): per unit for the keys,
  // per sub-tile and value group for the values.  Operand registers at bits
  // 4-7 carry the extra 16: on the key side they are the k-half fed by the b1
  // register, so q' of the b0 half is 16 times larger; on the value side they
  // are channel rows gq + 8, rescaled when the sums are normalised.
  constexpr uint32_t ZA0 = 0x00080008u, ZA1 = 0x00800080u;   // all-zero codes, bits 0-3 / 4-7
  auto score_sub_sn = [&](const Sub& sb, float cs20, float bias, float& s0, float& s1) {
    uint32_t wa[4], wb[4];
    load_key_words<4>(sb.k, gq, tq, wa, wb);
    float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int jj = j >> 1;
      const uint32_t va = (j & 1) ? (wa[jj] >> 8) : wa[jj], vb = (j & 1) ? (wb[jj] >> 8) : wb[jj];
      const uint32_t a0 = and_xor(va, 0x000F000Fu, ZA0), a1 = and_xor(vb, 0x000F000Fu, ZA0);
      const uint32_t a2 = and_xor(va, 0x00F000F0u, ZA1), a3 = and_xor(vb, 0x00F000F0u, ZA1);
      if (j & 1) mma_f16(acc1, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      else mma_f16(acc0, a0, a1, a2, a3, bq[j][0], bq[j][1]);
    }
    s0 = fmaf(acc0[0] + acc0[1] + acc1[0] + acc1[1], cs20, bias);
    s1 = fmaf(acc0[2] + acc0[3] + acc1[2] + acc1[3], cs20, bias);
  };
  auto pv_sub_sn = [&](const Sub& sb, float p0, float p1) {
    const int sa = 8 * tq + hh, sbl = sa + 4;
    const float pa0 = __shfl_sync(0xffffffffu, p0, sa);
    const float pa1 = __shfl_sync(0xffffffffu, p1, sa);
    const float pb0 = __shfl_sync(0xffffffffu, p0, sbl);
    const float pb1 = __shfl_sync(0xffffffffu, p1, sbl);
    uint32_t vw[8];
    load_value_words<4>(sb.v, lane, vw);
    uint32_t pha, pla, phb, plb;
    split2h(pa0, pb0, pha, pla);
    split2h(pa1, pb1, phb, plb);
    const uint16_t* vs = reinterpret_cast<const uint16_t*>(sb.vms);
    // rows 2tq, 2tq + 1 (and + 8) hold both groups' scales in 8 bytes
    const uint2 ra = *reinterpret_cast<const uint2*>(vs + 4 * tq);
    const uint2 rb = *reinterpret_cast<const uint2*>(vs + 4 * tq + 16);
    uint32_t b0 = 0, b1 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & 3) == 0) {
        const int gi = i >> 2;
        const uint32_t sel = gi ? 0x7632u : 0x5410u;
        const uint32_t xa = __byte_perm(ra.x, ra.y, sel), xb = __byte_perm(rb.x, rb.y, sel);
        const __half2 sa2 = *reinterpret_cast<const __half2*>(&xa), sb2 = *reinterpret_cast<const __half2*>(&xb);
        auto two = [](uint32_t ph, uint32_t pl, __half2 sv, uint32_t& hi, uint32_t& lo) {
          const __half2 a = *reinterpret_cast<const __half2*>(&ph), b = *reinterpret_cast<const __half2*>(&pl);
          const __half2 h = __hmul2(a, sv);
          const __half2 l = __hfma2(b, sv, __hfma2(a, sv, __hneg2(h)));
          hi = *reinterpret_cast<const uint32_t*>(&h);
          lo = *reinterpret_cast<const uint32_t*>(&l);
        };
        uint32_t h0, l0, h1, l1;
        two(pha, pla, sa2, h0, l0);
        two(phb, plb, sb2, h1, l1);
        b0 = is_lo ? l0 : h0;
        b1 = is_lo ? l1 : h1;
        mma_f16(st.zc[gi], ZA0, ZA1, ZA0, ZA1, b0, b1);   // the offset 8 of every code
      }
      const uint32_t w = vw[i], w8 = w >> 8;
      mma_f16(st.o[i], and_xor(w, 0x000F000Fu, ZA0), and_xor(w, 0x00F000F0u, ZA1), and_xor(w8, 0x000F000Fu, ZA0),
              and_xor(w8, 0x00F000F0u, ZA1), b0, b1);
    }
  };
  // A 16-token tile of the BF16 window (natural row-major layout).
  auto process_window = [&](const uint8_t* stg, int valid) {
    const uint32_t kaddr = smem_addr(stg), vaddr = kaddr + 16 * D * 2;
    float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int mi = lane >> 3;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = (lane & 7) + 8 * (mi & 1), c = 16 * j + 8 * (mi >> 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(kaddr + (r * D + c) * 2, a0, a1, a2, a3);
      if (j & 1) mma_bf16(acc1, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      else mma_bf16(acc0, a0, a1, a2, a3, bq[j][0], bq[j][1]);
    }
    float s[8], p[8];
    s[0] = gq < valid ? (acc0[0] + acc0[1] + acc1[0] + acc1[1]) * C : -INFINITY;
    s[1] = gq + 8 < valid ? (acc0[2] + acc0[3] + acc1[2] + acc1[3]) * C : -INFINITY;
#pragma unroll
    for (int k = 2; k < 8; ++k) s[k] = -INFINITY;
    softmax_chunk(s, p);
    const int sa = 8 * tq + hh, sbl = sa + 4;
    const float pa0 = __shfl_sync(0xffffffffu, p[0], sa);
    const float pa1 = __shfl_sync(0xffffffffu, p[1], sa);
    const float pb0 = __shfl_sync(0xffffffffu, p[0], sbl);
    const float pb1 = __shfl_sync(0xffffffffu, p[1], sbl);
    uint32_t h0, l0, h1, l1;
    split2(pa0, pb0, h0, l0);
    split2(pa1, pb1, h1, l1);
    const uint32_t b0 = dead_col ? 0u : (is_lo ? l0 : h0);
    const uint32_t b1 = dead_col ? 0u : (is_lo ? l1 : h1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane & 7) + 8 * (mi >> 1), c = 16 * i + 8 * (mi & 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(vaddr + (r * D + c) * 2, a0, a1, a2, a3);
      mma_bf16(st.o[i], a0, a1, a2, a3, b0, b1);
    }
  };

  // Where sub-tile `tok0 / 16` of a quantized unit sits in its stage.
  auto sub_at = [&](const uint8_t* stg, int tok0) {
    Sub sb;
    if (KAXIS) {
      const uint8_t* cb = stg + (tok0 >> g.lg_P) * g.chunk_used;
      const int us = (tok0 & (g.P - 1)) >> 4;
      sb.k = cb + us * g.sub_bytes;
      sb.v = cb + g.off_V + us * g.sub_bytes;
      sb.vms = cb + g.off_Vm + 16 * us * g.nvg * ES;
      sb.vmz = cb + g.off_Vm + (g.P + 16 * us) * g.nvg * ES;
      sb.kms = sb.kmz = nullptr;
    } else {
      const uint8_t* sbase = stg + (tok0 >> 4) * pp.qsub;
      sb.k = sbase;
      sb.v = sbase + g.sub_bytes;
      sb.vms = sbase + 2 * g.sub_bytes;
      sb.vmz = sb.vms + 16 * g.nvg * ES;
      sb.kms = sbase + 2 * g.sub_bytes + g.vm16;
      sb.kmz = sb.kms + 16 * g.nkg * ES;
    }
    return sb;
  };

  // sub-tiles per softmax chunk: 4, or one key group when groups are shorter
  const int ch = KAXIS ? min(4, g.g_k >> 4) : 4;

  // This warp computes units n = warp, warp + 4, ... of the range (K of them);
  // it owns SPW = nstages / 4 stages (2, or 1 when shared memory is short) and
  // its k-th unit lives in stage SPW * warp + k % SPW.  The walk iterator
  // `itc` visits every unit so that a record is left for every pair the CTA
  // touches; `iti` runs SPW of this warp's units ahead for the copies.
  const int SPW = pp.nstages / kDecodeWarps;   // 1 or 2 (the host guarantees it)
  const int K = N > warp ? (N - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
  It itc;
  it_seek(itc, s_pre, a.B, g.h_kv, c0);
  RowInfo ric = rinfo(itc.i);
  int nc = 0;
  It iti = itc;
  RowInfo rii = ric;
  int ni = 0;
  for (int t = 0; t < warp && t < N; ++t) step(iti, rii, ni);
  int issued = 0;
  if (K > 0) {
    const int32_t b0 = load_blk(iti, rii);
    issue(iti, rii, b0, SPW * warp);
    ++issued;
  }
  if (SPW == 2 && K > 1) {
    advance4(iti, rii, ni);
    const int32_t b1 = load_blk(iti, rii);
    issue(iti, rii, b1, SPW * warp + 1);
    ++issued;
  }
  int32_t blk_next = 0;
  if (K > SPW) {
    advance4(iti, rii, ni);
    blk_next = load_blk(iti, rii);
  }

  int cur_pair = itc.i * g.h_kv + itc.h;
  bool needs_setup = true;
  bool aborted = false;
  // leaves the walk iterator on unit `target`, recording every pair it passes
  auto walk_to = [&](int target) {
    if (itc.k + (target - nc) < itc.n) {   // still inside the same (row, head): no boundary
      itc.k += target - nc;
      nc = target;
      return;
    }
    while (nc < target) {
      step(itc, ric, nc);
      const int pid = itc.i * g.h_kv + itc.h;
      if (pid != cur_pair) {
        emit(cur_pair / g.h_kv, cur_pair % g.h_kv);
        state_reset(st);
        cur_pair = pid;
        needs_setup = true;
      }
    }
  };
  int consumed = 0;
  for (int k = 0; k < K; ++k) {
    walk_to(warp + kDecodeWarps * k);
    if (needs_setup) {
      setup_pair(itc.i, itc.h);
      needs_setup = false;
    }
    const int use = SPW == 2 ? (k >> 1) : k;   // earlier uses of this unit's stage
    const int sidx = SPW * warp + (SPW == 2 ? (k & 1) : 0);
    // every lane polls; the warp gives up together
    const bool arrived = wait_or_abort(full0 + 8 * sidx, uint32_t(use & 1), abort_flag);
    if (!__all_sync(0xffffffffu, arrived)) {
      if (lane == 0) {
        atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      aborted = true;
      break;
    }
    ++consumed;
    const uint8_t* stg = stages + size_t(sidx) * pp.stage_bytes;
    if (BF && itc.k < ric.nq) {
      process_window(stg, min(16, ric.qa - itc.k * 16));
    } else if (itc.k < ric.nq) {
      const int T0 = itc.k * pp.sup;
      const int valid_unit = min(pp.sup, ric.qa - T0);
      const int nsub = (valid_unit + 15) >> 4;
      int loaded = -1;
      if (SPEC && valid_unit == 64) {
        // A whole 64-token unit of the INT4 KIVI format: one key group, four
        // 16-token pages in the stage at fixed offsets; straight-line code
        // with scores and weights in registers, codes as fp16 subnormals.
        qprime_job(stg, 0, true);
        float accb[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // the key offset: q' against all-zero codes
#pragma unroll
        for (int j = 0; j < 8; ++j) mma_f16(accb, ZA0, ZA0, ZA1, ZA1, bq[j][0], bq[j][1]);
        const float cs20 = cs * 1048576.0f, bias = -(accb[0] + accb[1]) * cs20;
        float sc[8], pc[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) score_sub_sn(sub_at(stg, 16 * t), cs20, bias, sc[2 * t], sc[2 * t + 1]);
        softmax_chunk(sc, pc);
#pragma unroll
        for (int t = 0; t < 4; ++t) pv_sub_sn(sub_at(stg, 16 * t), pc[2 * t], pc[2 * t + 1]);
        st.raw = true;
      } else if (SPEC && st.raw) {
        normalize();
      }
      for (int c = 0; c < nsub && !(SPEC && valid_unit == 64); c += ch) {
        if (KAXIS && ((16 * c) >> g.lg_gk) != loaded) {
          loaded = (16 * c) >> g.lg_gk;
          qprime_job(stg, loaded);
        }
        // scores of the chunk's sub-tiles go through this lane's own slots of
        // the warp scratch, which keeps the loops rolled (small code, no spills)
        const int nt = min(ch, nsub - c);
#pragma unroll 1
        for (int t = 0; t < nt; ++t) {
          const int tok0 = 16 * (c + t);
          float s0, s1;
          score_sub(sub_at(stg, tok0), valid_unit - tok0, s0, s1);
          spw[(2 * t) * 32 + lane] = s0;
          spw[(2 * t + 1) * 32 + lane] = s1;
        }
        float sc[8], pc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) sc[q] = q < 2 * nt ? spw[q * 32 + lane] : -INFINITY;
        softmax_chunk(sc, pc);
#pragma unroll
        for (int q = 0; q < 8; ++q) spw[q * 32 + lane] = pc[q];
#pragma unroll 1
        for (int t = 0; t < nt; ++t)
          pv_sub(sub_at(stg, 16 * (c + t)), spw[(2 * t) * 32 + lane], spw[(2 * t + 1) * 32 + lane], true);
      }
    } else {
      if (SPEC && st.raw) normalize();
      if (!bq_bf16) {
        load_bq_from_q(itc.i, itc.h);
        bq_bf16 = true;
        bias_t = 0.0f;
      }
      process_window(stg, ric.ra - 16 * (itc.k - ric.nq));
    }
    __syncwarp();
    if (k + SPW < K) {
      issue(iti, rii, blk_next, sidx);   // the stage just read takes unit k + SPW
      ++issued;
      if (k + SPW + 1 < K) {
        advance4(iti, rii, ni);
        blk_next = load_blk(iti, rii);
      }
    }
  }
  if (aborted) {
    // keep the CTA until its copies in flight have landed (bounded)
    for (int j = consumed; j < issued; ++j) {
      const int sj = SPW * warp + (SPW == 2 ? (j & 1) : 0);
      (void)mbar_wait_bounded(full0 + 8 * sj, uint32_t((SPW == 2 ? (j >> 1) : j) & 1), kWaitNs);
    }
    return;
  }
  walk_to(N - 1);
  emit(cur_pair / g.h_kv, cur_pair % g.h_kv);
}

// Merge: one CTA per (row, kv head, query head).  The records of a pair are
// the consumer warps of every CTA whose range holds its units.  The CTA's
// warps (4, 8 or 16: more when few pairs share the grid, so a long sequence's
// pair, held by dozens of CTAs, is merged in few rounds) split those CTAs
// into contiguous runs; each lane keeps a running log-sum-exp over four
// channels, and the runs are then combined in warp order -- a fixed summation
// order for a given grid and batch.
constexpr int kMergeWarps = 16;
constexpr int kMergeThreads = kMergeWarps * 32;

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int D = kD;
  // launched as a programmatic dependent of the decode grid: wait until that
  // grid has completed and its writes are visible (returns at once otherwise)
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  __shared__ float s_m[kMergeWarps], s_den[kMergeWarps];
  __shared__ float s_num[kMergeWarps][D];
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int G = g.G;
  const int p = blockIdx.x / G, hd = blockIdx.x % G;
  const int i = p / g.h_kv, h = p % g.h_kv;
  const int32_t* pre = a.prefix;
  const int n = pre[i + 1] - pre[i];
  float* out = a.out + (int64_t(i) * g.h_q + h * G + hd) * D;
  if (n == 0) {
    if (tid < D) out[tid] = 0.0f;
    return;
  }
  const int64_t U = int64_t(pre[a.B]) * g.h_kv;
  const int64_t GR = a.grid;
  const int64_t ua = int64_t(pre[i]) * g.h_kv + int64_t(h) * n, ub = ua + n - 1;
  const int64_t k0 = ((ua + 1) * GR - 1) / U, k1 = ((ub + 1) * GR - 1) / U;
  // With at least as many units as CTAs every CTA from k0 to k1 holds units of
  // the pair.  With fewer, each unit has a CTA of its own and the others wrote
  // nothing: walk the pair's units instead (then all values are below 2^20).
  const bool by_unit = U < GR;
  const int64_t nk = by_unit ? ub - ua + 1 : k1 - k0 + 1;
  const int nw = blockDim.x >> 5;
  const int64_t kb = (int64_t(w) * nk) / nw, ke = (int64_t(w + 1) * nk) / nw;
  const int64_t rec_stride = int64_t(G) * (D + 2);
  float M = -INFINITY, den = 0.0f;
  float num[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t t = kb; t < ke; ++t) {
    const int64_t k = by_unit ? int64_t((int(ua + t + 1) * int(GR) - 1) / int(U)) : k0 + t;
    if (!dcheck(k >= 0 && k < GR && int64_t(p) + k < int64_t(a.B) * g.h_kv + GR, a.err, KVQ_DEVERR_INDEX)) continue;
    const float* rec = a.partials + ((int64_t(p) + k) * kDecodeWarps * G + hd) * (D + 2);
    float m[kDecodeWarps], l[kDecodeWarps];
    float2 o[kDecodeWarps][2];
#pragma unroll
    for (int r = 0; r < kDecodeWarps; ++r) {
      const float* rr = rec + r * rec_stride;
      m[r] = rr[0];
      l[r] = rr[1];
      o[r][0] = *reinterpret_cast<const float2*>(rr + 2 + 4 * lane);
      o[r][1] = *reinterpret_cast<const float2*>(rr + 4 + 4 * lane);
    }
    float mx = M;
#pragma unroll
    for (int r = 0; r < kDecodeWarps; ++r) mx = fmaxf(mx, m[r]);
    if (mx == -INFINITY) continue;
    const float sc = fast_exp2(M - mx);   // 0 while M is -inf
    den *= sc;
#pragma unroll
    for (int c = 0; c < 4; ++c) num[c] *= sc;
#pragma unroll
    for (int r = 0; r < kDecodeWarps; ++r) {
      const float wt = fast_exp2(m[r] - mx);
      den = fmaf(wt, l[r], den);
      num[0] = fmaf(wt, o[r][0].x, num[0]);
      num[1] = fmaf(wt, o[r][0].y, num[1]);
      num[2] = fmaf(wt, o[r][1].x, num[2]);
      num[3] = fmaf(wt, o[r][1].y, num[3]);
    }
    M = mx;
  }
  if (lane == 0) {
    s_m[w] = M;
    s_den[w] = den;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) s_num[w][4 * lane + c] = num[c];
  __syncthreads();
  if (tid >= D) return;
  float Mt = -INFINITY;
#pragma unroll
  for (int r = 0; r < kMergeWarps; ++r)
    if (r < nw) Mt = fmaxf(Mt, s_m[r]);
  float dt = 0.0f, nt = 0.0f;
  if (Mt != -INFINITY) {
#pragma unroll
    for (int r = 0; r < kMergeWarps; ++r) {
      if (r >= nw) break;
      const float wt = fast_exp2(s_m[r] - Mt);   // 0 for a run with nothing
      dt = fmaf(wt, s_den[r], dt);
      nt = fmaf(wt, s_num[r][tid], nt);
    }
  }
  out[tid] = dt > 0.0f ? nt / dt : 0.0f;
}

// ---------------------------------------------------------------------------
// Warp-specialised decode of the two KIVI-style formats that have whole-unit
// straight-line paths: INT4 symmetric (keys per channel G = 64, values per
// token G = 64, BF16 window 64) and INT2 asymmetric (G = 32 for both, fp16
// scale and zero-point, BF16 window 32), 4 query heads per kv head, page 16.
// A unit is 64 tokens (one INT4 key group, two INT2 key groups).  A CTA holds
// four pairs of warps; pair p takes the units n = p, p + 4, ... of the CTA's
// share (as warp p of decode_kernel does) through three shared-memory stages
// of its own.
//  * The score warp waits for a unit's stage, forms q' (and the key offset)
//    for its key group, computes the 64 scores with the subnormal-code path,
//    takes the online-softmax step, and hands the unit's weights p and the
//    rescale factor alpha of its running max to the value warp through a
//    slot in shared memory (its next unit's scores are computed while the
//    value warp still reads the slot; only the write waits).
//  * The value warp takes the weights, rescales its accumulators by alpha,
//    runs the value products, frees the slot and the stage, and issues the
//    bulk copies of the pair's unit three ahead into that stage.
// Each warp keeps half the state of a decode_kernel warp (the score warp q'
// and q, the value warp the accumulators), so two CTAs of eight warps fit per
// SM: four warps per scheduler, each running a shorter dependency chain.
// Every wait is bounded; the pair leaves the same (m, l, o) records as
// decode_kernel (m, l from the score warp, o from the value warp).
constexpr int kWsPairs = kDecodeWarps;
constexpr int kWsThreads = 2 * kWsPairs * 32;
constexpr int kWsPbufFloats = 4 * 4 * 16;   // weights of a unit: [sub-tile][head][token]

struct WsLayout {
  int stages, qbuf, pbuf, alpha, bars, flag, fill, total;
};

// A stage holds a unit's 4 pages or a 16-token window tile (K and V rows).
template <class S>
__host__ __device__ constexpr int ws_stage_bytes() {
  return (S::unit_tokens / 16) * S::chunk_used > 2 * 16 * kD * 2 ? (S::unit_tokens / 16) * S::chunk_used
                                                                  : 2 * 16 * kD * 2;
}

// S::ws_stages stages per pair, the weight slots, the barriers.
template <class S>
__host__ __device__ inline WsLayout ws_layout(int B) {
  WsLayout L;
  L.stages = ((B + 1 + 32 + 3 * B) * 4 + 127) / 128 * 128;   // prefix, scan scratch, per-row info
  L.qbuf = L.stages + kWsPairs * S::ws_stages * ws_stage_bytes<S>();
  L.pbuf = L.qbuf;
  L.alpha = L.pbuf + kWsPairs * kWsPbufFloats * 4;
  L.bars = L.alpha + kWsPairs * 4 * 4;
  L.flag = L.bars + kWsPairs * (S::ws_stages + 2) * 8;
  L.fill = L.flag + 16;   // debug build: pages each stage's copies filled (-1: a window tile)
  L.total = L.fill + (KVQ_DEBUG ? (kWsPairs * S::ws_stages * 4 + 15) / 16 * 16 : 0);
  return L;
}

template <class S>
__global__ void __launch_bounds__(kWsThreads, 2) decode_ws_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int D = kD;
  constexpr bool I2 = S::bits == 2;
  constexpr bool I8 = S::bits == 8;
  constexpr int UT = S::unit_tokens;                      // tokens per quantized unit
  constexpr int kWsStages = S::ws_stages;                 // stages per pair
  constexpr int kWsStageBytes = ws_stage_bytes<S>();      // one 64-token unit or window tile
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ __align__(128) uint8_t smem[];
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool vwarp = warp >= kWsPairs;
  const int pr = warp & (kWsPairs - 1);
  const WsLayout L = ws_layout<S>(a.B);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem);
  int32_t* s_scr = s_pre + (a.B + 1);
  int32_t* s_row = s_scr + 32;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bars = sbase + L.bars + 8u * uint32_t(pr * (kWsStages + 2));
  auto full_bar = [&](int s) { return bars + 8u * s; };
  const uint32_t pfull_bar = bars + 8u * kWsStages, pempty_bar = pfull_bar + 8u;
  auto stage_of = [&](int s) { return smem + L.stages + (pr * kWsStages + s) * kWsStageBytes; };
  float* pbuf = reinterpret_cast<float*>(smem + L.pbuf) + pr * kWsPbufFloats;
  float* alphas = reinterpret_cast<float*>(smem + L.alpha) + pr * 4;
  volatile int32_t* abort_flag = reinterpret_cast<int32_t*>(smem + L.flag);
  int32_t* fill = reinterpret_cast<int32_t*>(smem + L.fill) + pr * kWsStages;   // debug build only
  // debug build: a read of page t of stage s (t = -1: a window tile) must find
  // it filled by the copies of the unit being read
  auto page_filled = [&](int s, int t) {
    return dcheck(t < 0 ? fill[s] == -1 : fill[s] > t, a.err, KVQ_DEVERR_SMEM);
  };

  // Launched as a programmatic dependent of the previous kernel on the stream
  // (the append of a decode step): wait until that grid has completed and its
  // writes are visible before reading anything (returns at once when launched
  // plainly).  Then the merge grid may be scheduled; it waits for this one.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // ---- the work list: units per row, prefix over rows ---------------------
  for (int i = tid; i < a.B; i += blockDim.x) {
    const RowInfo ri = row_info(a, i, blockIdx.x == 0);
    s_pre[i + 1] = ri.nq + ri.nr;
    s_row[3 * i] = ri.seq;
    s_row[3 * i + 1] = ri.qa;
    s_row[3 * i + 2] = ri.ra;
  }
  if (tid == 0) {
    for (int b = 0; b < kWsPairs * (kWsStages + 2); ++b) mbar_init(sbase + L.bars + 8u * b, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  block_scan(s_pre, a.B, s_scr);
  if (blockIdx.x == 0)
    for (int i = tid; i <= a.B; i += blockDim.x) a.prefix[i] = s_pre[i];

  const int64_t U = int64_t(s_pre[a.B]) * g.h_kv;
  const int64_t c0 = int64_t(blockIdx.x) * U / a.grid, c1 = int64_t(blockIdx.x + 1) * U / a.grid;
  if (c0 >= c1) return;
  const int N = int(c1 - c0);
  const int K = N > pr ? (N - pr + kWsPairs - 1) / kWsPairs : 0;   // units of this pair

  auto rinfo = [&](int i) {
    RowInfo r;
    r.seq = s_row[3 * i];
    r.qa = s_row[3 * i + 1];
    r.ra = s_row[3 * i + 2];
    r.nq = (r.qa + UT - 1) / UT;
    r.nr = (r.ra + 15) >> 4;
    r.trow = a.table + int64_t(a.table_by_seq ? r.seq : i) * a.table_stride;
    return r;
  };
  auto step = [&](It& it, RowInfo& ri, int& n) {
    const bool row_changed = it_next(it, s_pre, a.B, g.h_kv);
    ++n;
    if (row_changed && n < N) ri = rinfo(it.i);
  };
  auto advance4 = [&](It& it, RowInfo& ri, int& n) {
    if (it.k + kWsPairs < it.n) {
      it.k += kWsPairs;
      n += kWsPairs;
      return;
    }
    for (int t = 0; t < kWsPairs; ++t) step(it, ri, n);
  };

  const int gq = lane >> 2, tq = lane & 3;
  const int hh = gq >> 1;               // head of this lane's B column
  const bool is_lo = gq & 1;            // the column carries the lo part
  const float C = a.qk_scale;
  constexpr uint32_t ZA0 = 0x00080008u, ZA1 = 0x00800080u;   // all-zero codes, bits 0-3 / 4-7
  constexpr uint32_t ZB8 = 0x00800080u;                       // INT8: the zero code, sign bit flipped

  It itc;
  it_seek(itc, s_pre, a.B, g.h_kv, c0);
  RowInfo ric = rinfo(itc.i);
  int nc = 0;
  int cur_pair = itc.i * g.h_kv + itc.h;
  bool needs_setup = true;
  auto rec_of = [&](int pair, int head) {
    return a.partials + (((int64_t(pair) + blockIdx.x) * kWsPairs + pr) * S::G + head) * (D + 2);
  };
  // Sub-tile t of a quantized unit's stage: page t of the unit.
  auto page_of = [&](const uint8_t* stg, int t) { return stg + t * S::chunk_used; };

  if (!vwarp) {
    // ============================ score warp ================================
    float m = -INFINITY, l = 0.0f;
    uint32_t bq[8][2];
    uint32_t qF[8][2];   // q in score-operand order, fp16, times the code weights
    float bias8 = 0.0f;  // INT8: q against all-128 codes, head tq
    float cs = C;
    bool bq_bf16 = false;
    auto qrow = [&](int row, int h, int head) { return a.q + (int64_t(row) * g.h_q + h * S::G + head) * D; };
    auto emit_k = [&](int pair) {
      float lt = l;
      lt += __shfl_xor_sync(FULL, lt, 4);
      lt += __shfl_xor_sync(FULL, lt, 8);
      lt += __shfl_xor_sync(FULL, lt, 16);
      if (gq == 0 && dcheck(int64_t(pair) + blockIdx.x < int64_t(a.B) * g.h_kv + a.grid, a.err, KVQ_DEVERR_INDEX)) {
        float* rec = rec_of(pair, tq);
        rec[0] = m;
        rec[1] = lt;
      }
    };
    auto walk_to = [&](int target) {
      if (itc.k + (target - nc) < itc.n) {
        itc.k += target - nc;
        nc = target;
        return;
      }
      while (nc < target) {
        step(itc, ric, nc);
        const int pid = itc.i * g.h_kv + itc.h;
        if (pid != cur_pair) {
          emit_k(cur_pair);
          m = -INFINITY;
          l = 0.0f;
          cur_pair = pid;
          needs_setup = true;
        }
      }
    };
    // q of the pair's heads in score-operand order (lane (gq, tq) holds, for
    // product j, channels 16 j + 2 tq + {0, 1} and + {8, 9} of head gq / 2),
    // fp16, times the code weights of its fields.
    //  * INT4: a nibble at bits 0-3 is worth c 2^-24, at bits 4-7 c 2^-20, so
    //    the b0 half carries the factor 16 and the products come out in units
    //    of 2^-20; the largest |q| lies in [2^-5, 2^-4), so 16 q s < 65504.
    //  * INT2: the code at bits 2y..2y+1 of a half-word is worth c 4^y 2^-24
    //    (y = 0..3, one shift by 8 bringing the upper byte down).  Product j
    //    takes its b0 half from y = 0 (j even) or 2 (j odd) and its b1 half
    //    from y + 1, so q carries the factors 2^-18 / weight: 64 and 16 (j
    //    even), 4 and 1 (j odd), and the products come out in units of 2^-18.
    //    The largest |q| lies in [2^-7, 2^-6): then 64 q s stays below 65504.
    //  * INT8 (keys per token): a byte at bits 0-7 of a half-word is worth
    //    c 2^-24 in either byte of the word (one shift by 8), so no factor;
    //    the key scale multiplies the score per token, so q itself is the
    //    operand for every unit of the pair (lo columns zero: q is exact in
    //    fp16 once scaled so that its largest |q| lies in [1/2, 1)).
    // An element pushed into the fp16 subnormal range is off by at most 2^-25.
    auto setup_op = [&](int row, int h) {
      const uint16_t* qr = qrow(row, h, hh);
      uint32_t t[8][2];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        t[j][0] = *reinterpret_cast<const uint32_t*>(qr + key_channel(32 * tq + 4 * j));
        t[j][1] = *reinterpret_cast<const uint32_t*>(qr + key_channel(32 * tq + 4 * j + 2));
      }
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(t[j][e] << 16)), fabsf(__uint_as_float(t[j][e] & 0xFFFF0000u))));
      amax = __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(amax)));
      constexpr int kExUp = I2 ? 7 : I8 ? 1 : 5;
      const int ex = amax > 0.0f ? min(max(int((__float_as_uint(amax) >> 23) & 0xFF) - 127 + kExUp, -100), 100) : 0;
      const float down = pow2f(-ex);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float f = down * (I2 ? ((j & 1) ? (e ? 1.0f : 4.0f) : (e ? 16.0f : 64.0f)) : I8 ? 1.0f : (e ? 1.0f : 16.0f));
          const __half2 v = __floats2half2_rn(__uint_as_float(t[j][e] << 16) * f, __uint_as_float(t[j][e] & 0xFFFF0000u) * f);
          qF[j][e] = *reinterpret_cast<const uint32_t*>(&v);
        }
      cs = C * pow2f(ex);
      bq_bf16 = false;
      if constexpr (I8) {
        // the operand of every unit of the pair, and the offset term: the
        // codes carry 128 (sign bit flipped), q against all-128 codes
        float accb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          bq[j][0] = is_lo ? 0u : qF[j][0];
          bq[j][1] = is_lo ? 0u : qF[j][1];
          mma_f16(accb, ZB8, ZB8, ZB8, ZB8, bq[j][0], bq[j][1]);
        }
        bias8 = accb[0];
      }
    };
    // INT4: q' = q s of the unit's key group as the score operand (hi in the
    // even columns, lo in the odd ones); this lane's 32 key-list positions
    // 32 tq .. 32 tq + 31 have their scales on page tq (32 per page)
    auto group_q4 = [&](const uint8_t* stg) {
      const uint4* ks = reinterpret_cast<const uint4*>(stg + tq * S::chunk_used + S::off_Km);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 sv = ks[v];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * v + jj;
          const uint32_t sw[2] = {jj ? sv.z : sv.x, jj ? sv.w : sv.y};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const __half2 x = *reinterpret_cast<const __half2*>(&qF[j][e]), sc2 = *reinterpret_cast<const __half2*>(&sw[e]);
            const __half2 hi = __hmul2(x, sc2);
            const __half2 lo = __hfma2(x, sc2, __hneg2(hi));
            bq[j][e] = is_lo ? *reinterpret_cast<const uint32_t*>(&lo) : *reinterpret_cast<const uint32_t*>(&hi);
          }
        }
      }
      bq_bf16 = false;
    };
    // INT2, key group gk of a unit (pages 2 gk, 2 gk + 1): q' = q s as the score
    // operand (hi in the even columns, lo in the odd ones) and the zero-point
    // term sum_c q_c z_c of head tq, from this lane's 32 key-list positions
    // 32 tq .. 32 tq + 31 (scales, then zero-points, in operand order).  The
    // zero-point product runs on the tensor cores: z over the factors against
    // the operand-order q.
    auto group_q2 = [&](const uint8_t* stg, int gk) -> float {
      const uint8_t* km = stg + (2 * gk + (tq >> 1)) * S::chunk_used + S::off_Km + 64 * (tq & 1);
      const uint4* ks = reinterpret_cast<const uint4*>(km);
      const uint4* kz = reinterpret_cast<const uint4*>(km + 2 * S::kslice);
      float za0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, za1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 sv = ks[v], zv = kz[v];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * v + jj;
          const uint32_t sw[2] = {jj ? sv.z : sv.x, jj ? sv.w : sv.y};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const __half2 x = *reinterpret_cast<const __half2*>(&qF[j][e]), sc2 = *reinterpret_cast<const __half2*>(&sw[e]);
            const __half2 hi = __hmul2(x, sc2);
            const __half2 lo = __hfma2(x, sc2, __hneg2(hi));
            bq[j][e] = is_lo ? *reinterpret_cast<const uint32_t*>(&lo) : *reinterpret_cast<const uint32_t*>(&hi);
          }
          const uint32_t z0 = jj ? zv.z : zv.x, z1 = jj ? zv.w : zv.y;
          uint32_t zs0, zs1;
          if (jj) {   // factors 4 and 1
            const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&z0), __float2half2_rn(0.25f));
            zs0 = *reinterpret_cast<const uint32_t*>(&r);
            zs1 = z1;
          } else {    // factors 64 and 16
            const __half2 r0 = __hmul2(*reinterpret_cast<const __half2*>(&z0), __float2half2_rn(0.015625f));
            const __half2 r1 = __hmul2(*reinterpret_cast<const __half2*>(&z1), __float2half2_rn(0.0625f));
            zs0 = *reinterpret_cast<const uint32_t*>(&r0);
            zs1 = *reinterpret_cast<const uint32_t*>(&r1);
          }
          mma_f16(jj ? za1 : za0, zs0, zs0, zs1, zs1, qF[j][0], qF[j][1]);
        }
      }
      bq_bf16 = false;
      return za0[0] + za1[0];
    };
    // INT2 scores of one 16-token page: rows gq, gq + 8 hold 32 bytes of codes
    // each, this lane's 8 at byte 8 tq
    auto score_sub2 = [&](const uint8_t* ksub, float cs18, float csb, int valid, float& s0, float& s1) {
      const uint2 x = *reinterpret_cast<const uint2*>(ksub + gq * S::row_bytes + 8 * tq);
      const uint2 y = *reinterpret_cast<const uint2*>(ksub + (gq + 8) * S::row_bytes + 8 * tq);
      const uint32_t wa[2] = {x.x, x.y}, wb[2] = {y.x, y.y};
      const uint32_t ua[2] = {x.x >> 8, x.y >> 8}, ub[2] = {y.x >> 8, y.y >> 8};
      float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int jj = j >> 2;
        const uint32_t va = (j & 2) ? ua[jj] : wa[jj], vb = (j & 2) ? ub[jj] : wb[jj];
        const uint32_t m0 = (j & 1) ? 0x00300030u : 0x00030003u, m1 = (j & 1) ? 0x00C000C0u : 0x000C000Cu;
        if (j & 1) mma_f16(acc1, va & m0, vb & m0, va & m1, vb & m1, bq[j][0], bq[j][1]);
        else mma_f16(acc0, va & m0, vb & m0, va & m1, vb & m1, bq[j][0], bq[j][1]);
      }
      s0 = gq < valid ? fmaf(acc0[0] + acc0[1] + acc1[0] + acc1[1], cs18, csb) : -INFINITY;
      s1 = gq + 8 < valid ? fmaf(acc0[2] + acc0[3] + acc1[2] + acc1[3], cs18, csb) : -INFINITY;
    };
    // INT8 scores of one 16-token page: rows gq, gq + 8 hold 128 bytes of
    // codes each, this lane's 32 at byte 32 tq; word j feeds product j (bytes
    // 0, 2 its b0 half, bytes 1, 3 its b1 half); then the token's key scale
    auto score_sub8 = [&](const uint8_t* page, float cs24, int valid, float& s0, float& s1) {
      const uint4* ra = reinterpret_cast<const uint4*>(page + gq * S::row_bytes + 32 * tq);
      const uint4* rb = reinterpret_cast<const uint4*>(page + (gq + 8) * S::row_bytes + 32 * tq);
      const uint4 x0 = ra[0], x1 = ra[1], y0 = rb[0], y1 = rb[1];
      const uint32_t wa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const uint32_t wb[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
      float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t a0 = and_xor(wa[j], 0x00FF00FFu, ZB8), a1 = and_xor(wb[j], 0x00FF00FFu, ZB8);
        const uint32_t a2 = and_xor(wa[j] >> 8, 0x00FF00FFu, ZB8), a3 = and_xor(wb[j] >> 8, 0x00FF00FFu, ZB8);
        if (j & 1) mma_f16(acc1, a0, a1, a2, a3, bq[j][0], bq[j][1]);
        else mma_f16(acc0, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      }
      const uint16_t* ks = reinterpret_cast<const uint16_t*>(page + S::off_Km);
      const float sa = __half2float(__ushort_as_half(ks[gq])), sb = __half2float(__ushort_as_half(ks[gq + 8]));
      s0 = gq < valid ? (acc0[0] + acc1[0] - bias8) * (cs24 * sa) : -INFINITY;
      s1 = gq + 8 < valid ? (acc0[2] + acc1[2] - bias8) * (cs24 * sb) : -INFINITY;
    };
    auto score_sub = [&](const uint8_t* ksub, float cs20, float bias, int valid, float& s0, float& s1) {
      uint32_t wa[4], wb[4];
      load_key_words<4>(ksub, gq, tq, wa, wb);
      float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int jj = j >> 1;
        const uint32_t va = (j & 1) ? (wa[jj] >> 8) : wa[jj], vb = (j & 1) ? (wb[jj] >> 8) : wb[jj];
        const uint32_t a0 = and_xor(va, 0x000F000Fu, ZA0), a1 = and_xor(vb, 0x000F000Fu, ZA0);
        const uint32_t a2 = and_xor(va, 0x00F000F0u, ZA1), a3 = and_xor(vb, 0x00F000F0u, ZA1);
        if (j & 1) mma_f16(acc1, a0, a1, a2, a3, bq[j][0], bq[j][1]);
        else mma_f16(acc0, a0, a1, a2, a3, bq[j][0], bq[j][1]);
      }
      s0 = gq < valid ? fmaf(acc0[0] + acc0[1] + acc1[0] + acc1[1], cs20, bias) : -INFINITY;
      s1 = gq + 8 < valid ? fmaf(acc0[2] + acc0[3] + acc1[2] + acc1[3], cs20, bias) : -INFINITY;
    };
    for (int k = 0; k < K; ++k) {
      walk_to(pr + kWsPairs * k);
      if (needs_setup) {
        setup_op(itc.i, itc.h);
        needs_setup = false;
      }
      const int s = k % kWsStages;
      if (!__all_sync(FULL, wait_or_abort(full_bar(s), uint32_t((k / kWsStages) & 1), abort_flag))) {
        if (lane == 0) {
          atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        return;
      }
      const uint8_t* stg = stage_of(s);
      float sc[8];
      if (itc.k < ric.nq) {
        const int valid = min(UT, ric.qa - itc.k * UT);
        (void)page_filled(s, I8 ? (valid <= 16 ? 0 : 1) : I2 && valid <= 32 ? 1 : 3);
        if constexpr (I8) {
          // one or two pages (keys per token: the last unit of a row may end
          // inside its first page); the unit's other scores are -inf
          const float cs24 = cs * 16777216.0f;
          score_sub8(page_of(stg, 0), cs24, valid, sc[0], sc[1]);
          if (valid > 16) score_sub8(page_of(stg, 1), cs24, valid - 16, sc[2], sc[3]);
          else sc[2] = sc[3] = -INFINITY;
#pragma unroll
          for (int t = 4; t < 8; ++t) sc[t] = -INFINITY;
        } else if constexpr (I2) {
          // one or two key groups of 32 tokens (the quantized length is a
          // multiple of 32); a missing second group scores -inf
          const float cs18 = cs * 262144.0f;
#pragma unroll
          for (int gk = 0; gk < 2; ++gk) {
            if (gk == 0 || valid > 32) {
              const float csb = cs * group_q2(stg, gk);
              score_sub2(page_of(stg, 2 * gk), cs18, csb, valid - 32 * gk, sc[4 * gk], sc[4 * gk + 1]);
              score_sub2(page_of(stg, 2 * gk + 1), cs18, csb, valid - 32 * gk - 16, sc[4 * gk + 2], sc[4 * gk + 3]);
            } else {
              sc[4] = sc[5] = sc[6] = sc[7] = -INFINITY;
            }
          }
        } else {
          group_q4(stg);
          float accb[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // the key offset: q' against all-zero codes
#pragma unroll
          for (int j = 0; j < 8; ++j) mma_f16(accb, ZA0, ZA0, ZA1, ZA1, bq[j][0], bq[j][1]);
          const float cs20 = cs * 1048576.0f, bias = -(accb[0] + accb[1]) * cs20;
#pragma unroll
          for (int t = 0; t < 4; ++t) score_sub(page_of(stg, t), cs20, bias, valid - 16 * t, sc[2 * t], sc[2 * t + 1]);
        }
      } else {
        // a 16-token tile of the BF16 window: q in bf16 against natural rows
        (void)page_filled(s, -1);
        if (!bq_bf16) {
          const uint16_t* qr = qrow(itc.i, itc.h, hh);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t t0 = *reinterpret_cast<const uint32_t*>(qr + key_channel(32 * tq + 4 * j));
            const uint32_t t1 = *reinterpret_cast<const uint32_t*>(qr + key_channel(32 * tq + 4 * j + 2));
            bq[j][0] = is_lo ? 0u : t0;   // q is exact in bf16: its lo part is zero
            bq[j][1] = is_lo ? 0u : t1;
          }
          bq_bf16 = true;
        }
        const int valid = ric.ra - 16 * (itc.k - ric.nq);
        const uint32_t kaddr = smem_addr(stg);
        float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const int mi = lane >> 3;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = (lane & 7) + 8 * (mi & 1), c = 16 * j + 8 * (mi >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kaddr + (r * D + c) * 2, a0, a1, a2, a3);
          if (j & 1) mma_bf16(acc1, a0, a1, a2, a3, bq[j][0], bq[j][1]);
          else mma_bf16(acc0, a0, a1, a2, a3, bq[j][0], bq[j][1]);
        }
        sc[0] = gq < valid ? (acc0[0] + acc0[1] + acc1[0] + acc1[1]) * C : -INFINITY;
        sc[1] = gq + 8 < valid ? (acc0[2] + acc0[3] + acc1[2] + acc1[3]) * C : -INFINITY;
#pragma unroll
        for (int t = 2; t < 8; ++t) sc[t] = -INFINITY;
      }
      // online softmax over the unit (log2 domain); alpha rescales what came before
      float mx = fmaxf(fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])), fmaxf(fmaxf(sc[4], sc[5]), fmaxf(sc[6], sc[7])));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
      float alpha = 1.0f;
      if (mx > m) {   // also taken from -inf; keeps p <= 1
        alpha = fast_exp2(m - mx);
        l *= alpha;
        m = mx;
      }
      const bool live = m != -INFINITY;
      float pc[8], sum = 0.0f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        pc[t] = live ? fast_exp2(sc[t] - m) : 0.0f;
        sum += pc[t];
      }
      l += sum;
      // hand the weights to the value warp (the slot is free once it took k - 1)
      if (k >= 1 && !__all_sync(FULL, wait_or_abort(pempty_bar, uint32_t((k - 1) & 1), abort_flag))) {
        if (lane == 0) {
          atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        return;
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        pbuf[t * 64 + tq * 16 + gq] = pc[2 * t];
        pbuf[t * 64 + tq * 16 + gq + 8] = pc[2 * t + 1];
      }
      if (gq == 0) alphas[tq] = alpha;
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull_bar);
    }
    walk_to(N - 1);
    emit_k(cur_pair);
  } else {
    // ============================ value warp ================================
    State st;
    state_reset(st);
    float zv[4][4];   // INT2: p-weighted value zero-point sums per value group
    auto zv_reset = [&]() {
#pragma unroll
      for (int gv = 0; gv < 4; ++gv)
#pragma unroll
        for (int c = 0; c < 4; ++c) zv[gv][c] = 0.0f;
    };
    zv_reset();
    auto normalize = [&]() {
      if constexpr (I2) {
        // row gq of channel tile i holds codes worth 2^-24 (i even) or 2^-20
        // (i odd), row gq + 8 four times that; then the zero-point terms
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float fa = (i & 1) ? 1048576.0f : 16777216.0f, fb = (i & 1) ? 262144.0f : 4194304.0f;
          st.o[i][0] = fmaf(st.o[i][0], fa, zv[i >> 1][0]);
          st.o[i][1] = fmaf(st.o[i][1], fa, zv[i >> 1][1]);
          st.o[i][2] = fmaf(st.o[i][2], fb, zv[i >> 1][2]);
          st.o[i][3] = fmaf(st.o[i][3], fb, zv[i >> 1][3]);
        }
        zv_reset();
      } else if constexpr (I8) {
        // every code at 2^-24, with the offset 128 of the flipped sign bit
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) st.o[i][c] = (st.o[i][c] - st.zc[0][c]) * 16777216.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) st.zc[0][c] = 0.0f;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int gi = i >> 2;
          st.o[i][0] = (st.o[i][0] - st.zc[gi][0]) * 16777216.0f;
          st.o[i][1] = (st.o[i][1] - st.zc[gi][1]) * 16777216.0f;
          st.o[i][2] = (st.o[i][2] - st.zc[gi][2]) * 1048576.0f;
          st.o[i][3] = (st.o[i][3] - st.zc[gi][3]) * 1048576.0f;
        }
#pragma unroll
        for (int gi = 0; gi < 2; ++gi)
#pragma unroll
          for (int c = 0; c < 4; ++c) st.zc[gi][c] = 0.0f;
      }
      st.raw = false;
    };
    auto emit_v = [&](int pair) {
      if (st.raw) normalize();
      if (!dcheck(int64_t(pair) + blockIdx.x < int64_t(a.B) * g.h_kv + a.grid, a.err, KVQ_DEVERR_INDEX)) return;
      float* rec = rec_of(pair, tq);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        rec[2 + 16 * i + gq] = st.o[i][0] + st.o[i][1];
        rec[2 + 16 * i + gq + 8] = st.o[i][2] + st.o[i][3];
      }
    };
    auto walk_to = [&](int target) {
      if (itc.k + (target - nc) < itc.n) {
        itc.k += target - nc;
        nc = target;
        return;
      }
      while (nc < target) {
        step(itc, ric, nc);
        const int pid = itc.i * g.h_kv + itc.h;
        if (pid != cur_pair) {
          emit_v(cur_pair);
          state_reset(st);
          if constexpr (I2) zv_reset();
          cur_pair = pid;
        }
      }
    };
    // this lane's block for a unit's copies (-1 when out of the table)
    // pages of a quantized unit: 4, or 2 for an INT2 unit whose attended
    // tokens all lie in its first key group (a key group's scales span both
    // of its pages, so pages follow whole groups)
    auto unit_pages = [&](const It& it, const RowInfo& ri) {
      if constexpr (I8) return ri.qa - UT * it.k <= 16 ? 1 : 2;   // token axis: pages as far as tokens go
      return I2 && ri.qa - 64 * it.k <= 32 ? 2 : 4;
    };
    auto load_blk = [&](const It& it, const RowInfo& ri) -> int32_t {
      if (it.k >= ri.nq || lane >= unit_pages(it, ri)) return 0;   // a window tile, or no page for this lane
      const int pg = ((it.k * UT) >> 4) + lane;
      return pg < a.table_stride ? ri.trow[pg] : -1;
    };
    auto issue = [&](const It& it, const RowInfo& ri, int32_t blk, int s) {
      const uint32_t dst = sbase + L.stages + uint32_t((pr * kWsStages + s) * kWsStageBytes);
      const uint32_t bar = full_bar(s);
      const bool window = it.k >= ri.nq;
      const int npg = window ? 0 : unit_pages(it, ri);
      const int ncopy = window ? 2 : npg;
      const uint32_t total = window ? 2 * 16 * D * 2 : npg * S::chunk_used;
      const bool bad = !window && __any_sync(FULL, lane < npg && (blk < 0 || blk >= g.num_blocks));
      bool dbad = false;
      if (KVQ_DEBUG) {
        // the copies fit the stage, a window tile's rows lie in the window;
        // record what the stage will hold for the readers' checks
        dbad = !dcheck(s >= 0 && s < kWsStages && total <= uint32_t(kWsStageBytes), a.err, KVQ_DEVERR_SMEM) ||
               !dcheck(!window || (ri.seq >= 0 && ri.seq < g.max_seqs && 16 * (it.k - ri.nq) + 16 <= S::R), a.err,
                       KVQ_DEVERR_INDEX);
        dbad = __any_sync(FULL, dbad);
        if (lane == 0 && s >= 0 && s < kWsStages) fill[s] = bad || dbad ? 0 : (window ? -1 : npg);
      }
      // the pair's generic-proxy reads of the stage come before the copies' writes
      fence_proxy_async();
      if (bad || dbad) {
        if (lane == 0) {
          if (bad) atomicOr(a.err, KVQ_DEVERR_BLOCK_ID);
          mbar_arrive_expect_tx(bar, 0);
        }
        return;
      }
      if (lane == 0) mbar_arrive_expect_tx(bar, total);
      __syncwarp();
      if (lane >= ncopy) return;
      if (window) {
        const int kr = it.k - ri.nq;
        const int64_t base = ((int64_t(ri.seq) * g.h_kv + it.h) * S::R + 16 * kr) * D;
        bulk_g2s(dst + lane * (16 * D * 2), (lane ? a.vres : a.kres) + base, 16 * D * 2, bar);
        return;
      }
      const uint8_t* chunk = a.pool + int64_t(blk) * g.block_bytes + int64_t(it.h) * g.chunk_bytes;
      bulk_g2s(dst + lane * S::chunk_used, chunk, uint32_t(S::chunk_used), bar);
    };
    // the value product of one 16-token page: weights p of tokens (2tq, 2tq + 1)
    // and (2tq + 8, 2tq + 9) of head hh as fp16 hi + lo, times each value group's
    // per-token scale; codes as fp16 subnormals (see score warp)
    auto pv_sub = [&](const uint8_t* page, float pa0, float pb0, float pa1, float pb1) {
      uint32_t vw[8];
      load_value_words<4>(page + S::off_V, lane, vw);
      uint32_t pha, pla, phb, plb;
      split2h(pa0, pb0, pha, pla);
      split2h(pa1, pb1, phb, plb);
      const uint16_t* vs = reinterpret_cast<const uint16_t*>(page + S::off_Vm);
      // rows 2tq, 2tq + 1 (and + 8) hold both groups' scales in 8 bytes
      const uint2 ra = *reinterpret_cast<const uint2*>(vs + 4 * tq);
      const uint2 rb = *reinterpret_cast<const uint2*>(vs + 4 * tq + 16);
      uint32_t b0 = 0, b1 = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((i & 3) == 0) {
          const int gi = i >> 2;
          const uint32_t sel = gi ? 0x7632u : 0x5410u;
          const uint32_t xa = __byte_perm(ra.x, ra.y, sel), xb = __byte_perm(rb.x, rb.y, sel);
          const __half2 sa2 = *reinterpret_cast<const __half2*>(&xa), sb2 = *reinterpret_cast<const __half2*>(&xb);
          auto two = [](uint32_t ph, uint32_t pl, __half2 sv, uint32_t& hi, uint32_t& lo) {
            const __half2 x = *reinterpret_cast<const __half2*>(&ph), y = *reinterpret_cast<const __half2*>(&pl);
            const __half2 h = __hmul2(x, sv);
            const __half2 lw = __hfma2(y, sv, __hfma2(x, sv, __hneg2(h)));
            hi = *reinterpret_cast<const uint32_t*>(&h);
            lo = *reinterpret_cast<const uint32_t*>(&lw);
          };
          uint32_t h0, l0, h1, l1;
          two(pha, pla, sa2, h0, l0);
          two(phb, plb, sb2, h1, l1);
          b0 = is_lo ? l0 : h0;
          b1 = is_lo ? l1 : h1;
          mma_f16(st.zc[gi], ZA0, ZA1, ZA0, ZA1, b0, b1);   // the offset 8 of every code
        }
        const uint32_t w = vw[i], w8 = w >> 8;
        mma_f16(st.o[i], and_xor(w, 0x000F000Fu, ZA0), and_xor(w, 0x00F000F0u, ZA1), and_xor(w8, 0x000F000Fu, ZA0),
                and_xor(w8, 0x00F000F0u, ZA1), b0, b1);
      }
    };

    // INT2 value product of one 16-token page: this lane's 16 bytes of codes
    // (one word per value group of 32 channels, two channel tiles each), the
    // weights p' = p s of each value group as fp16 hi + lo, and the zero-point
    // term: z of tokens (2tq, 2tq + 1) and (2tq + 8, 2tq + 9) against p hi + lo,
    // the same for every channel of the group.  Tile 2 gv takes the codes at
    // y = 0, 1 (rows gq, gq + 8), tile 2 gv + 1 those at y = 2, 3, each from the
    // word and from the word shifted down by 8 (the second half of the tokens).
    auto pv_sub2 = [&](const uint8_t* page, float pa0, float pb0, float pa1, float pb1) {
      const uint4 vq = *reinterpret_cast<const uint4*>(page + S::off_V + 16 * lane);
      const uint32_t vw[4] = {vq.x, vq.y, vq.z, vq.w};
      uint32_t pha, pla, phb, plb;
      split2h(pa0, pb0, pha, pla);
      split2h(pa1, pb1, phb, plb);
      // token rows of 4 scales: rows 2tq, 2tq + 1 in 16 bytes, rows 2tq + 8,
      // 2tq + 9 likewise; the zero-points follow the 16 rows of scales
      const uint16_t* vs = reinterpret_cast<const uint16_t*>(page + S::off_Vm);
      const uint4 ra = *reinterpret_cast<const uint4*>(vs + 8 * tq);
      const uint4 rb = *reinterpret_cast<const uint4*>(vs + 8 * tq + 32);
      const uint4 qa = *reinterpret_cast<const uint4*>(vs + 64 + 8 * tq);
      const uint4 qb = *reinterpret_cast<const uint4*>(vs + 64 + 8 * tq + 32);
      const uint32_t bza = is_lo ? pla : pha, bzb = is_lo ? plb : phb;
      auto two = [](uint32_t ph, uint32_t pl, uint32_t svb, uint32_t& hi, uint32_t& lo) {
        const __half2 x = *reinterpret_cast<const __half2*>(&ph), y = *reinterpret_cast<const __half2*>(&pl);
        const __half2 sv = *reinterpret_cast<const __half2*>(&svb);
        const __half2 h = __hmul2(x, sv);
        const __half2 lw = __hfma2(y, sv, __hfma2(x, sv, __hneg2(h)));
        hi = *reinterpret_cast<const uint32_t*>(&h);
        lo = *reinterpret_cast<const uint32_t*>(&lw);
      };
#pragma unroll
      for (int gv = 0; gv < 4; ++gv) {
        const uint32_t sel = (gv & 1) ? 0x7632u : 0x5410u;
        const uint32_t sa = __byte_perm(gv < 2 ? ra.x : ra.y, gv < 2 ? ra.z : ra.w, sel);
        const uint32_t sb = __byte_perm(gv < 2 ? rb.x : rb.y, gv < 2 ? rb.z : rb.w, sel);
        const uint32_t za = __byte_perm(gv < 2 ? qa.x : qa.y, gv < 2 ? qa.z : qa.w, sel);
        const uint32_t zb = __byte_perm(gv < 2 ? qb.x : qb.y, gv < 2 ? qb.z : qb.w, sel);
        uint32_t h0, l0, h1, l1;
        two(pha, pla, sa, h0, l0);
        two(phb, plb, sb, h1, l1);
        const uint32_t b0 = is_lo ? l0 : h0, b1 = is_lo ? l1 : h1;
        mma_f16(zv[gv], za, za, zb, zb, bza, bzb);
        const uint32_t w = vw[gv], w8 = w >> 8;
        mma_f16(st.o[2 * gv], w & 0x00030003u, w & 0x000C000Cu, w8 & 0x00030003u, w8 & 0x000C000Cu, b0, b1);
        mma_f16(st.o[2 * gv + 1], w & 0x00300030u, w & 0x00C000C0u, w8 & 0x00300030u, w8 & 0x00C000C0u, b0, b1);
      }
    };

    // INT8 value product of one 16-token page: this lane's 64-byte record
    // (words 2i, 2i + 1 the operand registers of channel tile i, bytes 0, 2
    // and 1, 3 of each), the weights p' = p s of the token's scale as fp16
    // hi + lo, and the offset 128 of every code against all-128 codes
    auto pv_sub8 = [&](const uint8_t* page, float pa0, float pb0, float pa1, float pb1) {
      const uint4* vr = reinterpret_cast<const uint4*>(page + S::off_V + 64 * lane);
      uint32_t w[16];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 x = vr[v];
        w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
      }
      uint32_t pha, pla, phb, plb;
      split2h(pa0, pb0, pha, pla);
      split2h(pa1, pb1, phb, plb);
      const uint16_t* vs = reinterpret_cast<const uint16_t*>(page + S::off_Vm);   // one scale per token
      const uint32_t sa = *reinterpret_cast<const uint32_t*>(vs + 2 * tq), sb = *reinterpret_cast<const uint32_t*>(vs + 2 * tq + 8);
      auto two = [](uint32_t ph, uint32_t pl, uint32_t svb, uint32_t& hi, uint32_t& lo) {
        const __half2 x = *reinterpret_cast<const __half2*>(&ph), y = *reinterpret_cast<const __half2*>(&pl);
        const __half2 sv = *reinterpret_cast<const __half2*>(&svb);
        const __half2 h = __hmul2(x, sv);
        const __half2 lw = __hfma2(y, sv, __hfma2(x, sv, __hneg2(h)));
        hi = *reinterpret_cast<const uint32_t*>(&h);
        lo = *reinterpret_cast<const uint32_t*>(&lw);
      };
      uint32_t h0, l0, h1, l1;
      two(pha, pla, sa, h0, l0);
      two(phb, plb, sb, h1, l1);
      const uint32_t b0 = is_lo ? l0 : h0, b1 = is_lo ? l1 : h1;
      mma_f16(st.zc[0], ZB8, ZB8, ZB8, ZB8, b0, b1);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t w0 = w[2 * i], w1 = w[2 * i + 1];
        mma_f16(st.o[i], and_xor(w0, 0x00FF00FFu, ZB8), and_xor(w0 >> 8, 0x00FF00FFu, ZB8),
                and_xor(w1, 0x00FF00FFu, ZB8), and_xor(w1 >> 8, 0x00FF00FFu, ZB8), b0, b1);
      }
    };

    // copies: the pair's first three units, then one unit three ahead per unit
    It iti = itc;
    RowInfo rii = ric;
    int ni = 0;
    for (int t = 0; t < pr && t < N; ++t) step(iti, rii, ni);
    int issued = 0, consumed = 0;
    for (; issued < K && issued < kWsStages; ++issued) {
      if (issued) advance4(iti, rii, ni);
      issue(iti, rii, load_blk(iti, rii), issued);
    }
    int32_t blk_next = 0;
    if (K > kWsStages) {
      advance4(iti, rii, ni);
      blk_next = load_blk(iti, rii);
    }
    bool aborted = false;
    for (int k = 0; k < K; ++k) {
      walk_to(pr + kWsPairs * k);
      const int s = k % kWsStages;
      const bool ok = wait_or_abort(pfull_bar, uint32_t(k & 1), abort_flag) &&
                      wait_or_abort(full_bar(s), uint32_t((k / kWsStages) & 1), abort_flag);
      if (!__all_sync(FULL, ok)) {
        if (lane == 0) {
          atomicOr(a.err, KVQ_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        aborted = true;
        break;
      }
      ++consumed;
      const float alpha = alphas[tq];
      if (__any_sync(FULL, alpha != 1.0f)) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) st.o[i][c] *= alpha;
        if constexpr (I2) {
#pragma unroll
          for (int gv = 0; gv < 4; ++gv)
#pragma unroll
            for (int c = 0; c < 4; ++c) zv[gv][c] *= alpha;
        } else {
#pragma unroll
          for (int gi = 0; gi < 2; ++gi)
#pragma unroll
            for (int c = 0; c < 4; ++c) st.zc[gi][c] *= alpha;
        }
      }
      const float* pb = pbuf;
      const uint8_t* stg = stage_of(s);
      if (itc.k < ric.nq) {
        (void)page_filled(s, unit_pages(itc, ric) - 1);
        if constexpr (I8) {
          const int nt = unit_pages(itc, ric);   // 1 or 2 pages
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (t < nt) {
              const float2 x = *reinterpret_cast<const float2*>(pb + t * 64 + hh * 16 + 2 * tq);
              const float2 y = *reinterpret_cast<const float2*>(pb + t * 64 + hh * 16 + 2 * tq + 8);
              pv_sub8(page_of(stg, t), x.x, x.y, y.x, y.y);
            }
          }
        } else if constexpr (I2) {
          const int nt = unit_pages(itc, ric);   // 2 or 4 pages
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (t < nt) {
              const float2 x = *reinterpret_cast<const float2*>(pb + t * 64 + hh * 16 + 2 * tq);
              const float2 y = *reinterpret_cast<const float2*>(pb + t * 64 + hh * 16 + 2 * tq + 8);
              pv_sub2(page_of(stg, t), x.x, x.y, y.x, y.y);
            }
          }
        } else {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 x = *reinterpret_cast<const float2*>(pb + t * 64 + hh * 16 + 2 * tq);
            const float2 y = *reinterpret_cast<const float2*>(pb + t * 64 + hh * 16 + 2 * tq + 8);
            pv_sub(page_of(stg, t), x.x, x.y, y.x, y.y);
          }
        }
        st.raw = true;
      } else {
        (void)page_filled(s, -1);
        if (st.raw) normalize();
        const float2 x = *reinterpret_cast<const float2*>(pb + hh * 16 + 2 * tq);
        const float2 y = *reinterpret_cast<const float2*>(pb + hh * 16 + 2 * tq + 8);
        uint32_t h0, l0, h1, l1;
        split2(x.x, x.y, h0, l0);
        split2(y.x, y.y, h1, l1);
        const uint32_t b0 = is_lo ? l0 : h0, b1 = is_lo ? l1 : h1;
        const uint32_t vaddr = smem_addr(stg) + 16 * D * 2;
        const int mi = lane >> 3;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = (lane & 7) + 8 * (mi >> 1), c = 16 * i + 8 * (mi & 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vaddr + (r * D + c) * 2, a0, a1, a2, a3);
          mma_bf16(st.o[i], a0, a1, a2, a3, b0, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(pempty_bar);
      if (k + kWsStages < K) {   // the stage just read takes unit k + 3
        issue(iti, rii, blk_next, s);
        ++issued;
        if (k + kWsStages + 1 < K) {
          advance4(iti, rii, ni);
          blk_next = load_blk(iti, rii);
        }
      }
    }
    if (aborted) {
      // keep the CTA until this pair's copies in flight have landed (bounded)
      for (int u = consumed; u < issued; ++u)
        (void)mbar_wait_bounded(full_bar(u % kWsStages), uint32_t((u / kWsStages) & 1), kWaitNs);
      return;
    }
    walk_to(N - 1);
    emit_v(cur_pair);
  }
}

template <int BITS, int ASYM, int KAXIS, int ES, int SPEC = 0>
const void* kernel_of() {
  return reinterpret_cast<const void*>(&decode_kernel<BITS, ASYM, KAXIS, ES, SPEC>);
}

}  // namespace

const void* decode_kernel_ptr(const Geo& g) {
  if (spec_int4_kivi(g)) return kernel_of<4, 0, 1, 2, 1>();
  if (g.bits == 16) return kernel_of<16, 0, 0, 2>();
  if (g.fp8) return kernel_of<8, 0, 0, 1>();
  const int key = ((g.bits == 8 ? 0 : g.bits == 4 ? 1 : 2) * 4 + g.asym * 2 + g.k_axis) * 2 + (g.es == 4);
  switch (key) {
#define KVQ_CASE(k, b, as, ax) \
    case 2 * (k): return kernel_of<b, as, ax, 2>(); \
    case 2 * (k) + 1: return kernel_of<b, as, ax, 4>();
    KVQ_CASE(0, 8, 0, 0) KVQ_CASE(1, 8, 0, 1) KVQ_CASE(2, 8, 1, 0) KVQ_CASE(3, 8, 1, 1)
    KVQ_CASE(4, 4, 0, 0) KVQ_CASE(5, 4, 0, 1) KVQ_CASE(6, 4, 1, 0) KVQ_CASE(7, 4, 1, 1)
    KVQ_CASE(8, 2, 0, 0) KVQ_CASE(9, 2, 0, 1) KVQ_CASE(10, 2, 1, 0) KVQ_CASE(11, 2, 1, 1)
#undef KVQ_CASE
    default: return nullptr;
  }
}

// The warp-specialised kernel of a plan (pipe.ws: 1 INT4 KIVI, 2 INT2 KIVI,
// 3 INT8 with keys per token).
static const void* ws_kernel_ptr(int ws) {
  return ws == 3   ? reinterpret_cast<const void*>(&decode_ws_kernel<SpecInt8Tok>)
         : ws == 2 ? reinterpret_cast<const void*>(&decode_ws_kernel<SpecInt2Kivi>)
                   : reinterpret_cast<const void*>(&decode_ws_kernel<SpecInt4Kivi>);
}

static size_t ws_smem_bytes(int ws, int B) {
  return size_t(ws == 3   ? ws_layout<SpecInt8Tok>(B).total
                : ws == 2 ? ws_layout<SpecInt2Kivi>(B).total
                          : ws_layout<SpecInt4Kivi>(B).total);
}

size_t decode_smem_bytes(const Geo& g, const DecodePipe& p, int B) {
  (void)g;
  return p.ws ? ws_smem_bytes(p.ws, B) : size_t(smem_layout(B, p).total);
}

size_t decode_partials_bytes(const Geo& g, int B, int grid) {
  return (size_t(B) * g.h_kv + size_t(grid)) * kDecodeWarps * g.G * (kD + 2) * sizeof(float);
}

// The dynamic shared-memory limit is an attribute of the kernel on a device,
// shared by every handle, thread and allocation-free call.  Plans for
// different batch sizes or formats need different amounts, so the limit only
// ever rises: lowering it for a small plan would make a live plan's larger
// launches fail.  One record for every kernel of the library, under a mutex.
cudaError_t raise_smem_limit(int dev, const void* kern, size_t smem) {
  struct Entry {
    int dev;
    const void* kern;
    size_t smem;
  };
  static std::mutex mu;
  static std::vector<Entry> set;
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& en : set)
    if (en.dev == dev && en.kern == kern) {
      if (smem <= en.smem) return cudaSuccess;
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (e == cudaSuccess) en.smem = smem;
      return e;
    }
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e == cudaSuccess) set.push_back({dev, kern, smem});
  return e;
}

cudaError_t plan_decode(const Geo& g, int max_B, DecodePipe* out) {
  DecodePipe p{};
  p.sup = g.bits == 16 ? 16 : g.k_axis ? (g.g_k > 64 ? g.g_k : 64) : 64;
  p.lg_sup = p.sup == 128 ? 7 : p.sup == 64 ? 6 : 4;
  p.qsub = g.k_axis ? 0 : 2 * g.sub_bytes + g.vm16 + g.km16;
  const int qunit = g.bits == 16 ? 2 * 16 * kD * 2
                    : g.k_axis   ? (p.sup / g.P) * g.chunk_used
                                 : kDecodeWarps * p.qsub;
  const int res = g.R ? 2 * 16 * kD * 2 : 0;
  p.stage_bytes = (((qunit > res ? qunit : res) + 127) / 128) * 128;
  int dev = 0, max_optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  // aim for three resident CTAs per SM (about 72 KB of shared memory each)
  // with two stages per consumer warp; the stage count stays a multiple of
  // the warp count so warp w always owns stages w, w + 4, ...
  int per_sm = 0;
  e = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e != cudaSuccess) return e;
  int reserved = 0;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  // two stages per warp when three CTAs still fit per SM, else one; the kernel
  // indexes stages as (nstages / 4) * warp + ..., so nstages must be 4 or 8
  p.nstages = 2 * kDecodeWarps;
  if (3 * (size_t(smem_layout(max_B, p).total) + size_t(reserved)) > size_t(per_sm)) p.nstages = kDecodeWarps;
  if (size_t(smem_layout(max_B, p).total) > size_t(max_optin)) return cudaErrorInvalidConfiguration;
  const size_t smem = size_t(smem_layout(max_B, p).total);
  if (smem > size_t(max_optin)) return cudaErrorInvalidConfiguration;
  const void* kern = decode_kernel_ptr(g);
  e = raise_smem_limit(dev, kern, smem);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p.ctas_per_sm, kern, kDecodeThreads, smem);
  if (e != cudaSuccess) return e;
  if (p.ctas_per_sm < 1) return cudaErrorInvalidConfiguration;
  p.ws = 0;
  const int ws = spec_int4_kivi(g) ? 1 : spec_int2_kivi(g) ? 2 : spec_int8_tok(g) ? 3 : 0;
  if (ws) {
    // the warp-specialised kernel when two of its CTAs fit per SM
    const size_t wsm = ws_smem_bytes(ws, max_B);
    if (2 * (wsm + size_t(reserved)) <= size_t(per_sm) && wsm <= size_t(max_optin)) {
      const void* wk = ws_kernel_ptr(ws);
      e = raise_smem_limit(dev, wk, wsm);
      if (e != cudaSuccess) return e;
      int occ = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, wk, kWsThreads, wsm);
      if (e != cudaSuccess) return e;
      if (occ >= 2) {
        p.ws = ws;
        p.ctas_per_sm = occ;
        if (ws == 3) {   // its units are 32 tokens: the per-row unit counts follow
          p.sup = 32;
          p.lg_sup = 5;
        }
      }
    }
  }
  *out = p;
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, cudaEvent_t between, int* launches) {
  const void* k = a.pipe.ws ? ws_kernel_ptr(a.pipe.ws) : decode_kernel_ptr(a.g);
  void* args[] = {const_cast<DecodeArgs*>(&a)};
  const size_t smem = decode_smem_bytes(a.g, a.pipe, a.B);
  // a programmatic dependent launch: the grid is scheduled while the previous
  // kernel on the stream (an append) runs, and waits for it on the device
  cudaLaunchConfig_t dcfg = {};
  dcfg.gridDim = dim3(a.grid);
  dcfg.blockDim = dim3(a.pipe.ws ? kWsThreads : kDecodeThreads);
  dcfg.dynamicSmemBytes = smem;
  dcfg.stream = s;
  cudaLaunchAttribute dattr[1];
  dattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  dattr[0].val.programmaticStreamSerializationAllowed = 1;
  dcfg.attrs = dattr;
  dcfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelExC(&dcfg, k, args);
  if (e != cudaSuccess) return e;
  ++*launches;
  if (between) {
    e = cudaEventRecord(between, s);
    if (e != cudaSuccess) return e;
  }
  const int items = a.B * a.g.h_kv * a.g.G;
  if (items == 0) return cudaSuccess;
  // The merge is a programmatic dependent launch, so its launch overlaps the
  // decode grid's tail; with an event between the two it is a plain launch.
  cudaLaunchConfig_t cfg = {};
  // about grid / (B h_kv) CTAs hold each pair: 4 warps up to 4 of them, 8 up
  // to 8, else 16
  const int per_pair = (a.grid + a.B * a.g.h_kv - 1) / (a.B * a.g.h_kv);
  const int merge_warps = per_pair <= 4 ? 4 : per_pair <= 8 ? 8 : kMergeWarps;
  cfg.gridDim = dim3(items);
  cfg.blockDim = dim3(32 * merge_warps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = between ? 0 : 1;
  e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(&merge_kernel), args);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace kvq
