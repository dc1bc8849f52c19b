// kvq_runtime.cpp -- host runtime of libkvq.so: the C ABI of include/kvq.h.
//
// Owns the device pool, the BF16 residual windows, the block table and the
// workspace; keeps the authoritative host bookkeeping (lengths, block tables,
// the free list) and turns each kvq_append into a compact plan that one H2D
// copy and a few kernels execute (llmdaily.org day-65, "How this connects to
// paging and prefix caching": blocks allocated on demand and addressed
// through a block table).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <deque>
#include <mutex>
#include <string>
#include <unordered_set>
#include <vector>

#include <cuda_runtime.h>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

#define KVQ_CUDA(call)                                                                     \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess)                                                                 \
      return fail(KVQ_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));       \
  } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// splitmix64 (Steele, Lea, Flood 2014).
uint64_t splitmix64(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

bool is_group_size(int g) { return g == 16 || g == 32 || g == 64 || g == 128; }

kvq_status validate(const kvq_config* c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "config is null");
  if (c->bits != 2 && c->bits != 4 && c->bits != 8 && c->bits != 16)
    return fail(KVQ_ERR_INVALID_ARG, "bits must be 2, 4, 8 or 16");
  if (c->fp8 != 0 && c->fp8 != 1) return fail(KVQ_ERR_INVALID_ARG, "fp8 must be 0 or 1");
  if (c->fp8 && (c->bits != 8 || c->k_axis != KVQ_AXIS_TOKEN || c->residual != 0 || c->asym != 0 ||
                 c->scale_fp32 != 0 || c->g_k != 128 || c->g_v != 128))
    return fail(KVQ_ERR_INVALID_ARG,
                "the FP8 format needs bits 8, k_axis 0, residual 0, asym 0, scale_fp32 0, g_k = g_v = 128");
  if (c->bits == 16 && (c->k_axis != KVQ_AXIS_TOKEN || c->residual != 0 || c->asym != 0 || c->scale_fp32 != 0 ||
                        c->g_k != 128 || c->g_v != 128))
    return fail(KVQ_ERR_INVALID_ARG,
                "the BF16 control (bits 16) needs k_axis 0, residual 0, asym 0, scale_fp32 0, g_k = g_v = 128");
  if (c->asym != 0 && c->asym != 1) return fail(KVQ_ERR_INVALID_ARG, "asym must be 0 or 1");
  if (c->scale_fp32 != 0 && c->scale_fp32 != 1) return fail(KVQ_ERR_INVALID_ARG, "scale_fp32 must be 0 or 1");
  if (c->d_h != kvq::kD) return fail(KVQ_ERR_UNSUPPORTED, "d_h must be 128");
  if (c->h_kv < 1 || c->h_q < 1 || c->h_q % c->h_kv != 0)
    return fail(KVQ_ERR_INVALID_ARG, "h_q must be a positive multiple of h_kv");
  const int G = c->h_q / c->h_kv;
  if (G != 1 && G != 2 && G != 4) return fail(KVQ_ERR_UNSUPPORTED, "h_q / h_kv must be 1, 2 or 4");
  if (c->g_v != 32 && c->g_v != 64 && c->g_v != 128) return fail(KVQ_ERR_UNSUPPORTED, "g_v must be 32, 64 or 128");
  if (c->page < 16 || (c->page & (c->page - 1)) != 0)
    return fail(KVQ_ERR_INVALID_ARG, "page must be a power of two >= 16");
  if (c->k_axis == KVQ_AXIS_TOKEN) {
    if (c->g_k != 32 && c->g_k != 64 && c->g_k != 128)
      return fail(KVQ_ERR_UNSUPPORTED, "token-axis g_k must be 32, 64 or 128");
    if (c->residual != 0) return fail(KVQ_ERR_INVALID_ARG, "token-axis keys take no residual window");
    if (c->page > 4096) return fail(KVQ_ERR_UNSUPPORTED, "page must be <= 4096");
  } else if (c->k_axis == KVQ_AXIS_CHANNEL) {
    if (!is_group_size(c->g_k)) return fail(KVQ_ERR_UNSUPPORTED, "channel-axis g_k must be 16, 32, 64 or 128");
    if (c->residual != c->g_k) return fail(KVQ_ERR_INVALID_ARG, "channel-axis keys need residual == g_k");
    if (c->page > c->g_k || c->g_k % c->page != 0)
      return fail(KVQ_ERR_UNSUPPORTED, "channel-axis keys need page to divide g_k");
  } else {
    return fail(KVQ_ERR_INVALID_ARG, "k_axis must be 0 (token) or 1 (channel)");
  }
  if (c->max_seqs < 1 || c->num_blocks < 1 || c->max_blocks_per_seq < 1)
    return fail(KVQ_ERR_INVALID_ARG, "capacity fields must be positive");
  if (c->fail_alloc_after < -1) return fail(KVQ_ERR_INVALID_ARG, "fail_alloc_after must be >= -1");
  return KVQ_OK;
}

kvq::Geo make_geo(const kvq_config& c) {
  kvq::Geo g{};
  const int D = kvq::kD, A = 1 + c.asym;
  g.bits = c.bits; g.asym = c.asym; g.k_axis = c.k_axis; g.g_k = c.g_k; g.g_v = c.g_v;
  g.scale_fp32 = c.scale_fp32; g.R = c.residual; g.P = c.page; g.h_q = c.h_q; g.h_kv = c.h_kv;
  g.G = c.h_q / c.h_kv;
  g.n = 32 / c.bits;
  g.row_bytes = D * c.bits / 8;
  g.sub_bytes = 16 * g.row_bytes;
  g.es = c.scale_fp32 ? 4 : 2;
  g.nvg = D / c.g_v;
  g.secK = (c.page / 16) * g.sub_bytes;
  g.secV = g.secK;
  g.secVm = int(align_up(size_t(c.page) * g.nvg * g.es * A, 16));
  g.fp8 = c.fp8;
  if (c.bits == 16 || c.fp8) {   // BF16 control and FP8: no per-group metadata
    g.nkg = 1;
    g.kslice = 0;
    g.secVm = 0;
    g.secKm = 0;
  } else if (c.k_axis == KVQ_AXIS_TOKEN) {
    g.nkg = D / c.g_k;
    g.kslice = 0;
    g.secKm = int(align_up(size_t(c.page) * g.nkg * g.es * A, 16));
  } else {
    g.nkg = 1;
    g.kslice = D / (c.g_k / c.page);
    g.secKm = int(align_up(size_t(g.kslice) * g.es * A, 16));
  }
  g.off_V = g.secK;
  g.off_Vm = g.off_V + g.secV;
  g.off_Km = g.off_Vm + g.secVm;
  g.chunk_used = g.off_Km + g.secKm;
  g.chunk_bytes = int64_t(align_up(size_t(g.chunk_used), 32));
  g.block_bytes = int64_t(c.h_kv) * g.chunk_bytes;
  g.num_blocks = c.num_blocks;
  g.max_seqs = c.max_seqs;
  g.mbps = c.max_blocks_per_seq;
  g.tileT = c.k_axis == KVQ_AXIS_CHANNEL ? c.g_k : 16;
  auto lg = [](int v) { int r = 0; while ((1 << r) < v) ++r; return r; };
  g.lg_P = lg(c.page);
  g.lg_gk = lg(c.g_k);
  g.lg_kslice = g.kslice ? lg(g.kslice) : 0;
  g.vm16 = g.secVm ? int(align_up(size_t(16) * g.nvg * g.es * A, 16)) : 0;
  g.km16 = g.secKm ? int(align_up(size_t(16) * g.nkg * g.es * A, 16)) : 0;
  g.qtile_bytes = c.k_axis == KVQ_AXIS_CHANNEL ? (c.g_k / c.page) * g.chunk_used
                                               : 2 * g.sub_bytes + g.vm16 + g.km16;
  return g;
}

int64_t blocks_for_len(const kvq_config& c, int64_t len) {
  if (c.residual == 0) return (len + c.page - 1) / c.page;
  return (len / c.residual) * (c.residual / c.page);
}

struct PinnedSlot {
  int32_t* host = nullptr;
  size_t cap = 0;   // int32 entries
  cudaEvent_t ev = nullptr;
  bool pending = false;
};

}  // namespace

struct kvq_handle_s {
  kvq_config cfg{};
  kvq::Geo geo{};
  std::vector<int32_t> len;     // stored length per sequence
  std::vector<int32_t> table;   // [max_seqs][mbps], -1 = none
  std::vector<int32_t> nblk;    // blocks per sequence
  std::vector<int32_t> refcnt;  // per block: block-table rows that hold it (0 = free)
  std::deque<int32_t> freelist;
  int64_t alloc_count = 0;
  // device
  int device = 0;
  uint8_t* d_pool = nullptr;
  uint16_t* d_kres = nullptr;
  uint16_t* d_vres = nullptr;
  int32_t* d_table = nullptr;
  int32_t* d_len = nullptr;
  uint32_t* d_err = nullptr;
  int32_t* d_plan = nullptr;
  size_t plan_cap = 0;          // int32 entries
  float* d_part = nullptr;
  size_t part_bytes = 0;
  int32_t* d_prefix = nullptr;
  int32_t* d_seqmap = nullptr;
  int32_t* d_rowlen = nullptr;  // per-row attended lengths of a prefill call
  float* d_fp8 = nullptr;       // FP8 format: [2][h_kv] scales
  std::vector<float> fp8;       // host copy
  PinnedSlot slots[4];
  int slot_next = 0;
  int sm_count = 0;
  int decode_ctas = 0;
  int decode_override = 0;
  kvq::DecodePipe pipe{};
  size_t bytes_workspace = 0;
  cudaEvent_t decode_event = nullptr;
  int launches = 0;
  // device staging of kvq_step_host: new K/V rows, q, output (grown on demand)
  uint8_t* d_in = nullptr;   // one buffer: a call's K rows, V rows and q, back to back
  float* d_out = nullptr;
  int32_t io_rows = 0;    // K/V rows the staging holds
  int32_t io_batch = 0;   // q / output rows the staging holds
  // chunked prefill: plan and split records (grown on demand)
  int32_t* d_pfplan = nullptr;
  size_t pfplan_cap = 0;  // int32 entries
  float* d_pfpart = nullptr;
  size_t pfpart_cap = 0;  // floats
  int pf_ctas_per_sm = 0; // resident prefill CTAs per SM (0: not queried yet)
};

namespace {

kvq_status device_guard(kvq_handle h) {
  if (h->cfg.host_only) return fail(KVQ_ERR_INVALID_ARG, "handle is host-only");
  KVQ_CUDA(cudaSetDevice(h->device));
  return KVQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Copies `ints` int32 values from `src` into a pinned slot and then to the
// device buffer `dst` on `stream`.
kvq_status stage_upload(kvq_handle h, const int32_t* src, size_t ints, int32_t* dst, cudaStream_t stream) {
  PinnedSlot& s = h->slots[h->slot_next];
  h->slot_next = (h->slot_next + 1) % 4;
  if (s.pending) {
    KVQ_CUDA(cudaEventSynchronize(s.ev));
    s.pending = false;
  }
  if (s.cap < ints) {
    if (s.host) KVQ_CUDA(cudaFreeHost(s.host));
    s.host = nullptr;
    s.cap = std::max(ints, size_t(1) << 16);
    KVQ_CUDA(cudaMallocHost(&s.host, s.cap * sizeof(int32_t)));
  }
  std::memcpy(s.host, src, ints * sizeof(int32_t));
  KVQ_CUDA(cudaMemcpyAsync(dst, s.host, ints * sizeof(int32_t), cudaMemcpyHostToDevice, stream));
  KVQ_CUDA(cudaEventRecord(s.ev, stream));
  s.pending = true;
  return KVQ_OK;
}

kvq_status ensure_plan_capacity(kvq_handle h, size_t ints) {
  if (ints <= h->plan_cap) return KVQ_OK;
  // earlier launches may still read the old plan: wait for the device
  KVQ_CUDA(cudaDeviceSynchronize());
  if (h->d_plan) KVQ_CUDA(cudaFree(h->d_plan));
  h->d_plan = nullptr;
  size_t cap = std::max(ints, h->plan_cap * 2);
  KVQ_CUDA(cudaMalloc(&h->d_plan, cap * sizeof(int32_t)));
  h->bytes_workspace += (cap - h->plan_cap) * sizeof(int32_t);
  h->plan_cap = cap;
  return KVQ_OK;
}

// A plan: sections of int32 entries, uploaded as one array.
struct Plan {
  std::vector<int32_t> tok, flush, src, res, tab, lens, zero;
};

kvq_status run_plan(kvq_handle h, const Plan& pl, const uint16_t* k, const uint16_t* v,
                    cudaStream_t stream) {
  constexpr int kHeader = 0;
  kvq::PlanView pv{};
  pv.n_tok = int(pl.tok.size() / 3);
  pv.n_flush = int(pl.flush.size() / kvq::kFlushEntryInts);
  pv.n_res = int(pl.res.size() / 3);
  pv.n_tab = int(pl.tab.size() / 2);
  pv.n_len = int(pl.lens.size() / 2);
  pv.n_zero = int(pl.zero.size());
  size_t off = kHeader;
  pv.off_tok = int(off); off += pl.tok.size();
  pv.off_flush = int(off); off += pl.flush.size();
  pv.off_src = int(off); off += pl.src.size();
  pv.off_res = int(off); off += pl.res.size();
  pv.off_tab = int(off); off += pl.tab.size();
  pv.off_len = int(off); off += pl.lens.size();
  pv.off_zero = int(off); off += pl.zero.size();
  if (off == 0) return KVQ_OK;
  if (off <= size_t(kvq::kPlanInline)) {
    // small plans ride in the launch parameters: no upload on the stream
    int32_t* o = pv.inl;
    for (const auto* sec : {&pl.tok, &pl.flush, &pl.src, &pl.res, &pl.tab, &pl.lens, &pl.zero})
      o = std::copy(sec->begin(), sec->end(), o);
    pv.plan = nullptr;
  } else {
    std::vector<int32_t> flat;
    flat.reserve(off);
    for (const auto* sec : {&pl.tok, &pl.flush, &pl.src, &pl.res, &pl.tab, &pl.lens, &pl.zero})
      flat.insert(flat.end(), sec->begin(), sec->end());
    kvq_status st = ensure_plan_capacity(h, off);
    if (st != KVQ_OK) return st;
    st = stage_upload(h, flat.data(), off, h->d_plan, stream);
    if (st != KVQ_OK) return st;
    pv.plan = h->d_plan;
  }
  kvq::DevState d{h->d_pool, h->d_kres, h->d_vres, h->d_table, h->d_len, h->d_err, h->d_fp8};
  // The window rows go into the first launch unless one of them would land in
  // a window slot that a flush of this call still reads (a multi-token append
  // that completes a group and leaves tokens behind); token rows keep their
  // own order (zeroing first).
  const bool tok = !pl.tok.empty(), flush = !pl.flush.empty();
  bool rows_in = k && !tok;
  if (rows_in && flush && !pl.res.empty()) {
    const int R = h->geo.R;
    std::unordered_set<int64_t> reads;
    for (int e = 0; e < pv.n_flush; ++e) {
      const int64_t seq = pl.flush[size_t(e) * kvq::kFlushEntryInts];
      for (int r = 0; r < R; ++r) {
        const int32_t src = pl.src[size_t(e) * R + r];
        if (src < 0) reads.insert(seq * R + (-1 - src));
      }
    }
    for (size_t i = 0; i + 2 < pl.res.size() && rows_in; i += 3)
      if (reads.count(int64_t(pl.res[i + 1]) * R + pl.res[i + 2])) rows_in = false;
  }
  if (flush && !tok) {
    // one launch: flush CTAs plus apply CTAs (tables, lengths, window rows)
    KVQ_CUDA(kvq::launch_flush(h->geo, d, pv, k, v, true, rows_in, stream, &h->launches));
  } else {
    KVQ_CUDA(kvq::launch_apply(h->geo, d, pv, rows_in ? k : nullptr, rows_in ? v : nullptr, stream,
                               &h->launches));
    KVQ_CUDA(kvq::launch_quant_token(h->geo, d, pv, k, v, stream, &h->launches));
    KVQ_CUDA(kvq::launch_flush(h->geo, d, pv, k, v, false, false, stream, &h->launches));
  }
  if (!rows_in) KVQ_CUDA(kvq::launch_residual(h->geo, d, pv, k, v, stream, &h->launches));
  return KVQ_OK;
}

void destroy_device(kvq_handle h) {
  if (h->cfg.host_only) return;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  cudaFree(h->d_pool);
  cudaFree(h->d_kres);
  cudaFree(h->d_vres);
  cudaFree(h->d_table);
  cudaFree(h->d_len);
  cudaFree(h->d_err);
  cudaFree(h->d_plan);
  cudaFree(h->d_part);
  cudaFree(h->d_prefix);
  cudaFree(h->d_seqmap);
  cudaFree(h->d_rowlen);
  cudaFree(h->d_fp8);
  cudaFree(h->d_in);
  cudaFree(h->d_out);
  cudaFree(h->d_pfplan);
  cudaFree(h->d_pfpart);
  for (auto& s : h->slots) {
    if (s.host) cudaFreeHost(s.host);
    if (s.ev) cudaEventDestroy(s.ev);
  }
}

kvq_status create_device(kvq_handle h) {
  const kvq_config& c = h->cfg;
  const kvq::Geo& g = h->geo;
  h->device = c.device;
  KVQ_CUDA(cudaSetDevice(h->device));
  KVQ_CUDA(cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, h->device));
  const size_t pool = size_t(c.num_blocks) * size_t(g.block_bytes);
  KVQ_CUDA(cudaMalloc(&h->d_pool, pool));
  KVQ_CUDA(cudaMemset(h->d_pool, 0, pool));
  const size_t res = std::max<size_t>(1, size_t(c.max_seqs) * c.h_kv * c.residual * c.d_h) * 2;
  KVQ_CUDA(cudaMalloc(&h->d_kres, res));
  KVQ_CUDA(cudaMalloc(&h->d_vres, res));
  KVQ_CUDA(cudaMemset(h->d_kres, 0, res));
  KVQ_CUDA(cudaMemset(h->d_vres, 0, res));
  const size_t tab = size_t(c.max_seqs) * c.max_blocks_per_seq * sizeof(int32_t);
  KVQ_CUDA(cudaMalloc(&h->d_table, tab));
  KVQ_CUDA(cudaMemset(h->d_table, 0xFF, tab));
  KVQ_CUDA(cudaMalloc(&h->d_len, size_t(c.max_seqs) * sizeof(int32_t)));
  KVQ_CUDA(cudaMemset(h->d_len, 0, size_t(c.max_seqs) * sizeof(int32_t)));
  KVQ_CUDA(cudaMalloc(&h->d_err, sizeof(uint32_t)));
  KVQ_CUDA(cudaMemset(h->d_err, 0, sizeof(uint32_t)));
  KVQ_CUDA(cudaMalloc(&h->d_fp8, size_t(2) * c.h_kv * sizeof(float)));
  KVQ_CUDA(cudaMemcpy(h->d_fp8, h->fp8.data(), size_t(2) * c.h_kv * sizeof(float), cudaMemcpyHostToDevice));
  for (auto& s : h->slots) KVQ_CUDA(cudaEventCreateWithFlags(&s.ev, cudaEventDisableTiming));

  // decode pipeline: stage ring of a producer warp and four consumer warps
  cudaError_t pe = kvq::plan_decode(g, c.max_seqs, &h->pipe);
  if (pe == cudaErrorInvalidConfiguration) return fail(KVQ_ERR_UNSUPPORTED, "decode tile does not fit on this device");
  KVQ_CUDA(pe);
  h->decode_ctas = std::min(h->sm_count * h->pipe.ctas_per_sm, kvq::kMaxDecodeGrid);

  // workspace: split partials for up to max_seqs rows and any grid we launch
  h->part_bytes = kvq::decode_partials_bytes(g, c.max_seqs, kvq::kMaxDecodeGrid);
  KVQ_CUDA(cudaMalloc(&h->d_part, h->part_bytes));
  // NaN-fill: a merge that ever read a slot no warp wrote shows up as NaN
  KVQ_CUDA(cudaMemset(h->d_part, 0xFF, h->part_bytes));
  KVQ_CUDA(cudaMalloc(&h->d_prefix, size_t(c.max_seqs + 1) * sizeof(int32_t)));
  KVQ_CUDA(cudaMalloc(&h->d_seqmap, size_t(c.max_seqs) * sizeof(int32_t)));
  KVQ_CUDA(cudaMalloc(&h->d_rowlen, size_t(c.max_seqs) * sizeof(int32_t)));
  h->bytes_workspace = h->part_bytes + size_t(c.max_seqs + 1) * 4 + size_t(c.max_seqs) * 4 + 4;
  return ensure_plan_capacity(h, size_t(1) << 16);
}

}  // namespace

extern "C" {

const char* kvq_last_error(void) { return g_last_error.c_str(); }

kvq_status kvq_layout(const kvq_config* cfg, kvq_layout_info* out) {
  kvq_status st = validate(cfg);
  if (st != KVQ_OK) return st;
  if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is null");
  const kvq::Geo g = make_geo(*cfg);
  out->row_bytes = uint64_t(g.row_bytes);
  out->sub_bytes = uint64_t(g.sub_bytes);
  out->off_v = uint64_t(g.off_V);
  out->off_vmeta = uint64_t(g.off_Vm);
  out->off_kmeta = uint64_t(g.off_Km);
  out->chunk_bytes = uint64_t(g.chunk_bytes);
  out->block_bytes = uint64_t(g.block_bytes);
  out->kslice = uint64_t(g.kslice);
  return KVQ_OK;
}

uint64_t kvq_cache_bytes(int32_t layers, int64_t tokens, int32_t h_kv, int32_t d_h, const kvq_config* cfg) {
  if (!cfg || layers < 0 || tokens < 0 || h_kv < 0 || d_h < 0) return 0;
  if (cfg->bits != 2 && cfg->bits != 4 && cfg->bits != 8 && cfg->bits != 16) return 0;
  if (cfg->g_k <= 0 || cfg->g_v <= 0) return 0;
  // M = 2 L T H_kv d_h b: codes for K and V, plus per-group metadata
  const uint64_t elems = uint64_t(layers) * uint64_t(tokens) * uint64_t(h_kv) * uint64_t(d_h);
  if (cfg->bits == 16) return 2 * elems * 2;   // the BF16 control: b = 2, no metadata
  const uint64_t meta = uint64_t(cfg->scale_fp32 ? 4 : 2) * uint64_t(1 + cfg->asym);
  const uint64_t codes = 2 * elems * uint64_t(cfg->bits) / 8;
  const uint64_t kmeta = (elems * meta + uint64_t(cfg->g_k) - 1) / uint64_t(cfg->g_k);
  const uint64_t vmeta = (elems * meta + uint64_t(cfg->g_v) - 1) / uint64_t(cfg->g_v);
  return codes + kmeta + vmeta;
}

kvq_status kvq_create(const kvq_config* cfg, kvq_handle* out) {
  if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  kvq_status st = validate(cfg);
  if (st != KVQ_OK) return st;
  kvq_handle h = new kvq_handle_s();
  h->cfg = *cfg;
  h->geo = make_geo(*cfg);
  h->len.assign(size_t(cfg->max_seqs), 0);
  h->nblk.assign(size_t(cfg->max_seqs), 0);
  h->refcnt.assign(size_t(cfg->num_blocks), 0);
  h->fp8.assign(size_t(2) * cfg->h_kv, 1.0f);
  h->table.assign(size_t(cfg->max_seqs) * cfg->max_blocks_per_seq, -1);
  // free list: Fisher-Yates over [0, num_blocks) driven by splitmix64(seed)
  std::vector<int32_t> perm(size_t(cfg->num_blocks));
  for (int32_t i = 0; i < cfg->num_blocks; ++i) perm[size_t(i)] = i;
  uint64_t sm = cfg->seed;
  for (int32_t i = cfg->num_blocks - 1; i >= 1; --i) {
    const uint64_t j = splitmix64(sm) % uint64_t(i + 1);
    std::swap(perm[size_t(i)], perm[size_t(j)]);
  }
  h->freelist.assign(perm.begin(), perm.end());
  if (!cfg->host_only) {
    st = create_device(h);
    if (st != KVQ_OK) {
      const std::string msg = g_last_error;
      destroy_device(h);
      delete h;
      return fail(st, msg);
    }
  }
  *out = h;
  return KVQ_OK;
}

void kvq_destroy(kvq_handle h) {
  if (!h) return;
  destroy_device(h);
  delete h;
}

kvq_status kvq_append(kvq_handle h, const void* k_bf16, const void* v_bf16, const int32_t* seq_ids_host,
                      int32_t n, void* stream_) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (n < 0) return fail(KVQ_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return KVQ_OK;
  if (!seq_ids_host) return fail(KVQ_ERR_INVALID_ARG, "seq_ids_host is null");
  if (!h->cfg.host_only) {
    if (!k_bf16 || !v_bf16) return fail(KVQ_ERR_INVALID_ARG, "k/v pointer is null");
    if (!aligned16(k_bf16) || !aligned16(v_bf16)) return fail(KVQ_ERR_INVALID_ARG, "k/v must be 16-byte aligned");
  }
  const kvq_config& c = h->cfg;
  const int S = c.max_seqs, R = c.residual, P = c.page, MB = c.max_blocks_per_seq;

  // ---- admission (no state change on failure) ----------------------------
  std::vector<int64_t> newlen(h->len.begin(), h->len.end());
  for (int32_t i = 0; i < n; ++i) {
    const int32_t s = seq_ids_host[i];
    if (s < 0 || s >= S) return fail(KVQ_ERR_BAD_SEQ, "sequence id " + std::to_string(s) + " out of range");
    ++newlen[size_t(s)];
  }
  int64_t need = 0;
  for (int s = 0; s < S; ++s) {
    if (newlen[size_t(s)] == h->len[size_t(s)]) continue;
    if (newlen[size_t(s)] > INT32_MAX / 2) return fail(KVQ_ERR_INVALID_ARG, "sequence too long");
    const int64_t nb = blocks_for_len(c, newlen[size_t(s)]);
    if (nb > MB) return fail(KVQ_ERR_OOM, "block-table row of sequence " + std::to_string(s) + " is full");
    need += nb - h->nblk[size_t(s)];
  }
  if (need > int64_t(h->freelist.size())) return fail(KVQ_ERR_OOM, "out of free blocks");
  if (c.fail_alloc_after >= 0 && h->alloc_count + need > c.fail_alloc_after)
    return fail(KVQ_ERR_OOM, "allocation refused by fail_alloc_after");

  // ---- plan (state is committed below, after the plan is complete) --------
  Plan pl;
  std::vector<int32_t> first(h->len.begin(), h->len.end());   // length before the call
  std::vector<int32_t> cur(first);
  std::vector<int32_t> nblk(h->nblk);
  // New table entries go straight into h->table (they were -1) and are
  // listed here, so a failure below can put the -1 back; the planner never
  // copies the whole table.
  std::vector<std::pair<int32_t, int32_t>> tab_changes;        // (index, block)
  auto undo_table = [&]() {
    for (const auto& tc : tab_changes) h->table[size_t(tc.first)] = -1;
  };
  std::vector<std::vector<int32_t>> arrivals(static_cast<size_t>(S));  // input rows per sequence
  int64_t allocs = 0;
  auto take = [&]() { return h->freelist[size_t(allocs++)]; };  // front of the free list, in order
  for (int32_t i = 0; i < n; ++i) {
    const int32_t s = seq_ids_host[i];
    const int32_t pos = cur[size_t(s)]++;
    if (R == 0) {
      const int32_t lb = pos / P;
      if (lb == nblk[size_t(s)]) {
        const int32_t b = take();
        tab_changes.push_back({s * MB + lb, b});
        h->table[size_t(s) * MB + lb] = b;
        ++nblk[size_t(s)];
        if (newlen[size_t(s)] < int64_t(lb + 1) * P) pl.zero.push_back(b);
      }
      pl.tok.insert(pl.tok.end(), {i, h->table[size_t(s) * MB + lb], pos % P});
    } else {
      arrivals[size_t(s)].push_back(i);
      if (pos % R == R - 1) {
        const int32_t grp = pos / R, npg = R / P;
        std::vector<int32_t> ent = {s, grp, npg};
        for (int j = 0; j < npg; ++j) {
          const int32_t b = take();
          tab_changes.push_back({s * MB + nblk[size_t(s)], b});
          h->table[size_t(s) * MB + nblk[size_t(s)]] = b;
          ++nblk[size_t(s)];
          ent.push_back(b);
        }
        ent.resize(kvq::kFlushEntryInts, -1);
        pl.flush.insert(pl.flush.end(), ent.begin(), ent.end());
        for (int r = 0; r < R; ++r) {
          const int32_t p = grp * R + r;
          pl.src.push_back(p < first[size_t(s)] ? -1 - (p % R)
                                                : arrivals[size_t(s)][size_t(p - first[size_t(s)])]);
        }
      }
    }
  }
  if (R > 0) {
    for (int s = 0; s < S; ++s) {
      const int32_t L = cur[size_t(s)];
      if (L == first[size_t(s)]) continue;
      const int32_t lo = std::max(first[size_t(s)], (L / R) * R);
      for (int32_t p = lo; p < L; ++p)
        pl.res.insert(pl.res.end(), {arrivals[size_t(s)][size_t(p - first[size_t(s)])], s, p % R});
    }
  }
  for (const auto& tc : tab_changes) pl.tab.insert(pl.tab.end(), {tc.first, tc.second});
  for (int s = 0; s < S; ++s)
    if (cur[size_t(s)] != first[size_t(s)]) pl.lens.insert(pl.lens.end(), {s, cur[size_t(s)]});

  if (!c.host_only) {
    kvq_status st = device_guard(h);
    if (st == KVQ_OK)
      st = run_plan(h, pl, static_cast<const uint16_t*>(k_bf16), static_cast<const uint16_t*>(v_bf16),
                    static_cast<cudaStream_t>(stream_));
    if (st != KVQ_OK) {
      undo_table();
      return st;
    }
  }
  // ---- commit host state -----------------------------------------------------
  h->nblk = nblk;
  for (int64_t j = 0; j < allocs; ++j) h->refcnt[size_t(h->freelist[size_t(j)])] = 1;
  h->freelist.erase(h->freelist.begin(), h->freelist.begin() + allocs);
  h->alloc_count += allocs;
  for (int s = 0; s < S; ++s) h->len[size_t(s)] = cur[size_t(s)];
  return KVQ_OK;
}

namespace {

// Decode over the handle's pool and windows for `batch` rows (tables from the
// caller or the handle's own rows by sequence).
kvq_status launch_handle_decode(kvq_handle h, const void* q_bf16, const int32_t* block_table, int32_t bt_stride,
                                const int32_t* seq_lens, const int32_t* seqmap, int32_t batch, float* out,
                                cudaStream_t stream) {
  kvq::DecodeArgs a{};
  a.pool = h->d_pool;
  a.kres = h->d_kres;
  a.vres = h->d_vres;
  a.table = block_table ? block_table : h->d_table;
  a.table_stride = block_table ? bt_stride : h->cfg.max_blocks_per_seq;
  a.table_by_seq = block_table ? 0 : 1;
  a.seq_lens = seq_lens;
  a.seqmap = seqmap;
  a.stored_len = h->d_len;
  a.q = static_cast<const uint16_t*>(q_bf16);
  a.fp8 = h->d_fp8;
  a.out = out;
  a.partials = h->d_part;
  a.prefix = h->d_prefix;
  a.err = h->d_err;
  a.B = batch;
  a.grid = h->decode_override > 0 ? h->decode_override : h->decode_ctas;
  a.qk_scale = float(1.4426950408889634 / std::sqrt(double(kvq::kD)));
  a.pipe = h->pipe;
  a.g = h->geo;
  KVQ_CUDA(kvq::launch_decode(a, stream, h->decode_event, &h->launches));
  return KVQ_OK;
}

}  // namespace

kvq_status kvq_decode_attn(kvq_handle h, const void* q_bf16, const int32_t* block_table, int32_t bt_stride,
                           const int32_t* seq_lens, const int32_t* seq_ids_host, int32_t batch, float* out,
                           void* stream_) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (batch < 0) return fail(KVQ_ERR_INVALID_ARG, "batch must be >= 0");
  if (batch == 0) return KVQ_OK;
  if (batch > h->cfg.max_seqs) return fail(KVQ_ERR_INVALID_ARG, "batch exceeds max_seqs");
  kvq_status st = device_guard(h);
  if (st != KVQ_OK) return st;
  if (!q_bf16 || !seq_lens || !out) return fail(KVQ_ERR_INVALID_ARG, "q, seq_lens and out are required");
  if (!aligned16(q_bf16) || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "q/out must be 16-byte aligned");
  if (block_table && bt_stride < 1) return fail(KVQ_ERR_INVALID_ARG, "bt_stride must be >= 1");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const int32_t* seqmap = nullptr;
  if (seq_ids_host) {
    for (int32_t i = 0; i < batch; ++i)
      if (seq_ids_host[i] < 0 || seq_ids_host[i] >= h->cfg.max_seqs)
        return fail(KVQ_ERR_BAD_SEQ, "sequence id " + std::to_string(seq_ids_host[i]) + " out of range");
    st = stage_upload(h, seq_ids_host, size_t(batch), h->d_seqmap, stream);
    if (st != KVQ_OK) return st;
    seqmap = h->d_seqmap;
  }
  return launch_handle_decode(h, q_bf16, block_table, bt_stride, seq_lens, seqmap, batch, out, stream);
}

namespace {

// Grows the staging of kvq_step_host to at least `rows` K/V rows and `batch`
// q / output rows.  Earlier steps may still read the old buffers: growing
// waits for the device first.
kvq_status ensure_io(kvq_handle h, int32_t rows, int32_t batch) {
  if (rows <= h->io_rows && batch <= h->io_batch) return KVQ_OK;
  KVQ_CUDA(cudaDeviceSynchronize());
  const int32_t r = std::max(rows, h->io_rows), b = std::max(batch, h->io_batch);
  const kvq_config& c = h->cfg;
  const size_t kv = size_t(r) * c.h_kv * c.d_h, qo = size_t(b) * c.h_q * c.d_h;
  if (h->d_in) KVQ_CUDA(cudaFree(h->d_in));
  if (h->d_out) KVQ_CUDA(cudaFree(h->d_out));
  h->d_in = nullptr;
  h->d_out = nullptr;
  h->bytes_workspace -= (size_t(h->io_rows) * c.h_kv * c.d_h * 4 + size_t(h->io_batch) * c.h_q * c.d_h * 6);
  h->io_rows = h->io_batch = 0;
  KVQ_CUDA(cudaMalloc(&h->d_in, std::max<size_t>(2 * kv + qo, 1) * 2));
  KVQ_CUDA(cudaMalloc(&h->d_out, std::max<size_t>(qo, 1) * 4));
  h->io_rows = r;
  h->io_batch = b;
  h->bytes_workspace += kv * 4 + qo * 6;
  return KVQ_OK;
}

}  // namespace

kvq_status kvq_step_host(kvq_handle h, const void* k_host, const void* v_host, const int32_t* seq_ids_host,
                         int32_t n, const void* q_host, int32_t batch, float* out_host, void* stream_) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (n < 0 || batch < 0) return fail(KVQ_ERR_INVALID_ARG, "n and batch must be >= 0");
  if (batch > h->cfg.max_seqs) return fail(KVQ_ERR_INVALID_ARG, "batch exceeds max_seqs");
  if (n > 0 && (!k_host || !v_host || !seq_ids_host))
    return fail(KVQ_ERR_INVALID_ARG, "k, v and seq_ids are required when n > 0");
  if (batch > 0 && (!q_host || !out_host)) return fail(KVQ_ERR_INVALID_ARG, "q and out are required when batch > 0");
  kvq_status st = device_guard(h);
  if (st != KVQ_OK) return st;
  const kvq_config& c = h->cfg;
  for (int32_t i = 0; i < n; ++i)   // checked here so that a bad id enqueues nothing
    if (seq_ids_host[i] < 0 || seq_ids_host[i] >= c.max_seqs)
      return fail(KVQ_ERR_BAD_SEQ, "sequence id " + std::to_string(seq_ids_host[i]) + " out of range");
  st = ensure_io(h, n, batch);
  if (st != KVQ_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const size_t kv_bytes = size_t(n) * c.h_kv * c.d_h * 2, q_bytes = size_t(batch) * c.h_q * c.d_h * 2;
  // this call's rows back to back in the device staging: K | V | q
  uint8_t* d_k = h->d_in;
  uint8_t* d_v = d_k + kv_bytes;
  uint8_t* d_q = d_v + kv_bytes;
  const uint8_t* hk = static_cast<const uint8_t*>(k_host);
  const uint8_t* hv = static_cast<const uint8_t*>(v_host);
  const uint8_t* hq = static_cast<const uint8_t*>(q_host);
  // a caller whose k, v and q are back to back in host memory gets one copy
  const bool packed = n > 0 && batch > 0 && hv == hk + kv_bytes && hq == hv + kv_bytes;
  // The device address of page-locked host memory the device maps, else null
  // (an unregistered pointer is not an error here).
  auto mapped = [](const void* ptr) -> const void* {
    cudaPointerAttributes pa{};
    if (ptr && cudaPointerGetAttributes(&pa, ptr) == cudaSuccess && pa.type == cudaMemoryTypeHost &&
        pa.devicePointer != nullptr && aligned16(pa.devicePointer))
      return pa.devicePointer;
    (void)cudaGetLastError();
    return nullptr;
  };
  const void* mk = n > 0 ? mapped(k_host) : nullptr;
  const void* mv = n > 0 && !packed ? mapped(v_host) : nullptr;
  const void* mq = batch > 0 && !packed ? mapped(q_host) : nullptr;
  if (packed ? mk != nullptr : ((n == 0 || (mk && mv)) && (batch == 0 || mq))) {
    // mapped inputs: one pull kernel reads them over the bus into the staging
    kvq::PullArgs pa{};
    auto seg = [&](const void* src, void* dst, size_t bytes) {
      pa.src[pa.n] = src;
      pa.dst[pa.n] = dst;
      pa.n16[pa.n] = int64_t(bytes / 16);
      ++pa.n;
    };
    if (packed) {
      seg(mk, d_k, 2 * kv_bytes + q_bytes);
    } else {
      if (n > 0) {
        seg(mk, d_k, kv_bytes);
        seg(mv, d_v, kv_bytes);
      }
      if (batch > 0) seg(mq, d_q, q_bytes);
    }
    KVQ_CUDA(kvq::launch_pull(pa, stream, &h->launches));
  } else if (packed) {
    KVQ_CUDA(cudaMemcpyAsync(d_k, hk, 2 * kv_bytes + q_bytes, cudaMemcpyHostToDevice, stream));
  } else {
    if (n > 0) {
      KVQ_CUDA(cudaMemcpyAsync(d_k, hk, kv_bytes, cudaMemcpyHostToDevice, stream));
      KVQ_CUDA(cudaMemcpyAsync(d_v, hv, kv_bytes, cudaMemcpyHostToDevice, stream));
    }
    if (batch > 0) KVQ_CUDA(cudaMemcpyAsync(d_q, hq, q_bytes, cudaMemcpyHostToDevice, stream));
  }
  if (n > 0) {
    st = kvq_append(h, d_k, d_v, seq_ids_host, n, stream_);
    if (st != KVQ_OK) return st;
  }
  if (batch == 0) return KVQ_OK;
  // page-locked output the device can write (mapped pinned memory) takes the
  // attention output straight from the decode kernel; else one D2H copy
  const void* mo = mapped(out_host);
  float* d_out = mo ? static_cast<float*>(const_cast<void*>(mo)) : h->d_out;
  const bool direct = mo != nullptr;
  st = launch_handle_decode(h, d_q, nullptr, 0, h->d_len, nullptr, batch, d_out, stream);
  if (st != KVQ_OK) return st;
  if (!direct) KVQ_CUDA(cudaMemcpyAsync(out_host, h->d_out, q_bytes * 2, cudaMemcpyDeviceToHost, stream));
  return KVQ_OK;
}

namespace {

// Grows a device buffer of `elem`-byte entries to at least `need` entries
// (earlier launches may still read it: growing waits for the device first).
kvq_status ensure_buffer(kvq_handle h, void** buf, size_t& cap, size_t need, size_t elem) {
  if (need <= cap) return KVQ_OK;
  KVQ_CUDA(cudaDeviceSynchronize());
  if (*buf) KVQ_CUDA(cudaFree(*buf));
  *buf = nullptr;
  const size_t c = std::max(need, cap * 2);
  KVQ_CUDA(cudaMalloc(buf, c * elem));
  h->bytes_workspace += (c - cap) * elem;
  cap = c;
  return KVQ_OK;
}

// Chunked prefill with shared tiles: rows sorted by (sequence, position) form
// blocks of at most 64 / g query tokens of one sequence (32 for the
// tensor-core kernel of the INT4 KIVI format: 128 rows of 4 heads); each
// block is split over the key range into `splits` tasks per kv head, one CTA
// each.
kvq_status prefill_blocks(kvq_handle h, const uint16_t* q, const int32_t* seq_ids, const int32_t* pos,
                          int32_t n, float* out, cudaStream_t stream) {
  const kvq::Geo& g = h->geo;
  const bool tc = kvq::prefill_tc_supported(g) && h->pipe.sup == 64;
  const int G = g.G, QB = tc ? 32 : 4 * (16 / G);
  std::vector<int32_t> order(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) order[size_t(i)] = i;
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
    return seq_ids[x] != seq_ids[y] ? seq_ids[x] < seq_ids[y] : pos[x] < pos[y];
  });
  std::vector<int32_t> rows, blocks, tasks;
  rows.reserve(size_t(n) * 2);
  std::vector<int32_t> nq;   // quantized units per block
  const int sup = h->pipe.sup;
  for (int32_t i = 0; i < n;) {
    const int32_t s = seq_ids[order[size_t(i)]];
    int32_t j = i;
    while (j < n && j - i < QB && seq_ids[order[size_t(j)]] == s) ++j;
    const int32_t Lq = (h->len[size_t(s)] / g.g_k) * g.g_k;
    const int32_t bmax = pos[order[size_t(j - 1)]];
    blocks.insert(blocks.end(), {s, int32_t(rows.size() / 2), j - i, Lq});
    for (int32_t k = i; k < j; ++k) rows.insert(rows.end(), {order[size_t(k)], pos[order[size_t(k)]]});
    nq.push_back((std::min(bmax + 1, Lq) + sup - 1) / sup);
    i = j;
  }
  const int nb = int(nq.size());
  const int cap_units = kvq::kPrefillMaxPages / (sup / g.P);
  int max_nq = 1;
  for (int x : nq) max_nq = std::max(max_nq, x);
  // Pick the split count that minimises the makespan
  // estimate max(waves of resident CTAs x (mean units per task + a task's
  // fixed cost), the longest task + that cost); a task's setup, pipeline fill
  // and records cost about as much as 8 units.  No task may outgrow its
  // block-id cache.
  const int stage_bytes = tc ? kvq::prefill_tc_stage_bytes() : kvq::prefill_stage_bytes(g, sup);
  if (h->pf_ctas_per_sm == 0) h->pf_ctas_per_sm = tc ? kvq::prefill_tc_ctas_per_sm() : kvq::prefill_ctas_per_sm(g, stage_bytes);
  const int slots = h->pf_ctas_per_sm * h->sm_count;
  double units = 0.0;
  for (int x : nq) units += double(x) * g.h_kv;
  const int smin = std::max(1, (max_nq + cap_units - 1) / cap_units);
  const int smax = std::max(smin, std::min(64, max_nq));
  int splits = smin;
  double best = 1e300;
  for (int sp = smin; sp <= smax; ++sp) {
    const int64_t ntask = int64_t(nb) * g.h_kv * sp;
    const double waves = double((ntask + slots - 1) / slots);
    constexpr double kTaskUnits = 8.0;
    const double cost = std::max(waves * (units / double(ntask) + kTaskUnits),
                                 double((max_nq + sp - 1) / sp) + kTaskUnits);
    if (cost < best) {
      best = cost;
      splits = sp;
    }
  }
  struct Task { int32_t b, hk, sp, u0, u1; };
  std::vector<Task> tl;
  tl.reserve(size_t(nb) * g.h_kv * splits);
  for (int b = 0; b < nb; ++b)
    for (int hk = 0; hk < g.h_kv; ++hk)
      for (int sp = 0; sp < splits; ++sp)
        tl.push_back({b, hk, sp, int32_t(int64_t(sp) * nq[size_t(b)] / splits),
                      int32_t(int64_t(sp + 1) * nq[size_t(b)] / splits)});
  // longest tasks first: CTAs start roughly in index order, so this packs the
  // resident slots like a longest-processing-time schedule
  std::stable_sort(tl.begin(), tl.end(), [](const Task& x, const Task& y) { return x.u1 - x.u0 > y.u1 - y.u0; });
  for (const Task& t : tl) tasks.insert(tasks.end(), {t.b, t.hk, t.sp, t.u0, t.u1});
  kvq::PrefillArgs a{};
  a.off_rows = 0;
  a.off_blocks = int32_t(rows.size());
  a.off_tasks = a.off_blocks + int32_t(blocks.size());
  const size_t total = size_t(a.off_tasks) + tasks.size();
  std::vector<int32_t> flat;
  flat.reserve(total);
  for (const auto* sec : {&rows, &blocks, &tasks}) flat.insert(flat.end(), sec->begin(), sec->end());
  kvq_status st = ensure_buffer(h, reinterpret_cast<void**>(&h->d_pfplan), h->pfplan_cap, total, 4);
  if (st != KVQ_OK) return st;
  if (splits > 1) {
    st = ensure_buffer(h, reinterpret_cast<void**>(&h->d_pfpart), h->pfpart_cap,
                       size_t(n) * g.h_q * splits * (kvq::kD + 2), 4);
    if (st != KVQ_OK) return st;
  }
  st = stage_upload(h, flat.data(), total, h->d_pfplan, stream);
  if (st != KVQ_OK) return st;
  a.pool = h->d_pool;
  a.kres = h->d_kres;
  a.vres = h->d_vres;
  a.table = h->d_table;
  a.table_stride = h->cfg.max_blocks_per_seq;
  a.q = q;
  a.out = out;
  a.part = h->d_pfpart;
  a.plan = h->d_pfplan;
  a.n_tasks = int32_t(tasks.size() / 5);
  a.splits = splits;
  a.err = h->d_err;
  a.qk_scale = float(1.4426950408889634 / std::sqrt(double(kvq::kD)));
  a.sup = sup;
  a.lg_sup = h->pipe.lg_sup;
  a.stage_bytes = stage_bytes;
  a.g = g;
  if (tc) KVQ_CUDA(kvq::launch_prefill_tc(a, n, stream, &h->launches));
  else KVQ_CUDA(kvq::launch_prefill(a, n, stream, &h->launches));
  return KVQ_OK;
}

}  // namespace

kvq_status kvq_prefill_attn(kvq_handle h, const void* q_bf16, const int32_t* seq_ids_host,
                            const int32_t* positions_host, int32_t n, float* out, void* stream_) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (n < 0) return fail(KVQ_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return KVQ_OK;
  kvq_status st = device_guard(h);
  if (st != KVQ_OK) return st;
  if (!q_bf16 || !out || !seq_ids_host || !positions_host)
    return fail(KVQ_ERR_INVALID_ARG, "q, out, seq_ids and positions are required");
  if (!aligned16(q_bf16) || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "q/out must be 16-byte aligned");
  const kvq_config& c = h->cfg;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t s = seq_ids_host[i];
    if (s < 0 || s >= c.max_seqs)
      return fail(KVQ_ERR_BAD_SEQ, "sequence id " + std::to_string(s) + " out of range");
    if (positions_host[i] < 0 || positions_host[i] >= h->len[size_t(s)])
      return fail(KVQ_ERR_INVALID_ARG, "position " + std::to_string(positions_host[i]) + " of row " +
                                           std::to_string(i) + " is not a stored position of its sequence");
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (kvq::prefill_supported(h->geo))
    return prefill_blocks(h, static_cast<const uint16_t*>(q_bf16), seq_ids_host, positions_host, n, out, stream);
  // other formats: one decode row per query token, attending its own causal
  // prefix; at most max_seqs rows per launch (the planned batch)
  std::vector<int32_t> rowlen(size_t(std::min<int32_t>(n, c.max_seqs)));
  const int64_t row = int64_t(c.h_q) * c.d_h;
  for (int32_t base = 0; base < n; base += c.max_seqs) {
    const int32_t m = std::min<int32_t>(c.max_seqs, n - base);
    for (int32_t j = 0; j < m; ++j) rowlen[size_t(j)] = positions_host[base + j] + 1;
    st = stage_upload(h, seq_ids_host + base, size_t(m), h->d_seqmap, stream);
    if (st != KVQ_OK) return st;
    st = stage_upload(h, rowlen.data(), size_t(m), h->d_rowlen, stream);
    if (st != KVQ_OK) return st;
    st = launch_handle_decode(h, static_cast<const uint16_t*>(q_bf16) + base * row, nullptr, 0, h->d_rowlen,
                              h->d_seqmap, m, out + base * row, stream);
    if (st != KVQ_OK) return st;
  }
  return KVQ_OK;
}

kvq_status kvq_block_table(kvq_handle h, const int32_t** dev_ptr, int32_t* stride) {
  if (!h || !dev_ptr || !stride) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  *dev_ptr = h->d_table;
  *stride = h->cfg.max_blocks_per_seq;
  return KVQ_OK;
}

kvq_status kvq_block_table_host(kvq_handle h, int32_t seq, int32_t* dst, int32_t max_entries,
                                int32_t* n_entries) {
  if (!h || !n_entries) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (seq < 0 || seq >= h->cfg.max_seqs) return fail(KVQ_ERR_BAD_SEQ, "sequence id out of range");
  const int32_t nb = h->nblk[size_t(seq)];
  *n_entries = nb;
  for (int32_t j = 0; dst && j < std::min(nb, max_entries); ++j)
    dst[j] = h->table[size_t(seq) * h->cfg.max_blocks_per_seq + j];
  return KVQ_OK;
}

kvq_status kvq_seq_len(kvq_handle h, int32_t seq, int32_t* len) {
  if (!h || !len) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (seq < 0 || seq >= h->cfg.max_seqs) return fail(KVQ_ERR_BAD_SEQ, "sequence id out of range");
  *len = h->len[size_t(seq)];
  return KVQ_OK;
}

kvq_status kvq_seq_lens_device(kvq_handle h, const int32_t** dev_ptr) {
  if (!h || !dev_ptr) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  *dev_ptr = h->d_len;
  return KVQ_OK;
}

kvq_status kvq_free_seq(kvq_handle h, int32_t seq, void* stream_) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (seq < 0 || seq >= h->cfg.max_seqs) return fail(KVQ_ERR_BAD_SEQ, "sequence id out of range");
  const int MB = h->cfg.max_blocks_per_seq;
  Plan pl;
  for (int32_t j = 0; j < h->nblk[size_t(seq)]; ++j) pl.tab.insert(pl.tab.end(), {seq * MB + j, -1});
  pl.lens.insert(pl.lens.end(), {seq, 0});
  if (!h->cfg.host_only) {
    kvq_status st = device_guard(h);
    if (st != KVQ_OK) return st;
    st = run_plan(h, pl, nullptr, nullptr, static_cast<cudaStream_t>(stream_));
    if (st != KVQ_OK) return st;
  }
  for (int32_t j = 0; j < h->nblk[size_t(seq)]; ++j) {
    int32_t& e = h->table[size_t(seq) * MB + j];
    if (--h->refcnt[size_t(e)] == 0) h->freelist.push_back(e);   // last holder frees it
    e = -1;
  }
  h->nblk[size_t(seq)] = 0;
  h->len[size_t(seq)] = 0;
  return KVQ_OK;
}

kvq_status kvq_set_fp8_scales(kvq_handle h, const float* k_scales, const float* v_scales) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (!h->cfg.fp8) return fail(KVQ_ERR_INVALID_ARG, "the cache is not in the FP8 format");
  if (!k_scales || !v_scales) return fail(KVQ_ERR_INVALID_ARG, "scales are required");
  for (int32_t L : h->len)
    if (L) return fail(KVQ_ERR_INVALID_ARG, "scales must be set before the first append");
  const int H = h->cfg.h_kv;
  for (int i = 0; i < H; ++i)
    if (!(k_scales[i] > 0.0f) || !(v_scales[i] > 0.0f) || !std::isfinite(k_scales[i]) || !std::isfinite(v_scales[i]))
      return fail(KVQ_ERR_INVALID_ARG, "scales must be positive finite numbers");
  std::vector<float> s(size_t(2) * H);
  std::copy(k_scales, k_scales + H, s.begin());
  std::copy(v_scales, v_scales + H, s.begin() + H);
  if (!h->cfg.host_only) {
    kvq_status st = device_guard(h);
    if (st != KVQ_OK) return st;
    KVQ_CUDA(cudaDeviceSynchronize());   // earlier work may still read the old scales
    KVQ_CUDA(cudaMemcpy(h->d_fp8, s.data(), s.size() * sizeof(float), cudaMemcpyHostToDevice));
  }
  h->fp8 = s;
  return KVQ_OK;
}

kvq_status kvq_share_prefix(kvq_handle h, int32_t src_seq, int32_t dst_seq, int32_t tokens, void* stream_) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  const kvq_config& c = h->cfg;
  if (src_seq < 0 || src_seq >= c.max_seqs || dst_seq < 0 || dst_seq >= c.max_seqs)
    return fail(KVQ_ERR_BAD_SEQ, "sequence id out of range");
  if (src_seq == dst_seq) return fail(KVQ_ERR_INVALID_ARG, "source and destination are the same sequence");
  if (h->len[size_t(dst_seq)] != 0) return fail(KVQ_ERR_INVALID_ARG, "destination sequence is not empty");
  if (tokens < 0 || tokens > h->len[size_t(src_seq)])
    return fail(KVQ_ERR_INVALID_ARG, "tokens must be in [0, source length]");
  // only whole, full blocks are shared: whole pages of a per-token format, whole
  // key groups (which are whole pages) of a per-channel format with a window
  const int32_t unit = c.residual ? c.residual : c.page;
  if (tokens % unit != 0)
    return fail(KVQ_ERR_INVALID_ARG, "tokens must be a multiple of " + std::to_string(unit) +
                                         " (whole blocks / key groups) to be shared");
  const int MB = c.max_blocks_per_seq;
  const int32_t nb = int32_t(blocks_for_len(c, tokens));
  if (nb > MB) return fail(KVQ_ERR_OOM, "block-table row is too short");
  Plan pl;
  for (int32_t j = 0; j < nb; ++j) pl.tab.insert(pl.tab.end(), {dst_seq * MB + j, h->table[size_t(src_seq) * MB + j]});
  pl.lens.insert(pl.lens.end(), {dst_seq, tokens});
  if (!c.host_only) {
    kvq_status st = device_guard(h);
    if (st != KVQ_OK) return st;
    st = run_plan(h, pl, nullptr, nullptr, static_cast<cudaStream_t>(stream_));
    if (st != KVQ_OK) return st;
  }
  for (int32_t j = 0; j < nb; ++j) {
    const int32_t b = h->table[size_t(src_seq) * MB + j];
    h->table[size_t(dst_seq) * MB + j] = b;
    ++h->refcnt[size_t(b)];
  }
  h->nblk[size_t(dst_seq)] = nb;
  h->len[size_t(dst_seq)] = tokens;
  return KVQ_OK;
}

kvq_status kvq_stats(kvq_handle h, kvq_stats_t* out) {
  if (!h || !out) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  const kvq_config& c = h->cfg;
  uint64_t tokens = 0;
  for (int32_t L : h->len) tokens += uint64_t(L);
  out->blocks_free = h->freelist.size();
  out->blocks_used = uint64_t(c.num_blocks) - out->blocks_free;
  out->tokens_stored = tokens;
  out->bytes_pool = c.host_only ? 0 : uint64_t(c.num_blocks) * uint64_t(h->geo.block_bytes);
  out->bytes_residual = c.host_only ? 0 : 2ull * c.max_seqs * c.h_kv * c.residual * c.d_h * 2;
  out->bytes_workspace = c.host_only ? 0 : h->bytes_workspace;
  out->bytes_formula = kvq_cache_bytes(1, int64_t(tokens), c.h_kv, c.d_h, &c);
  out->kernel_launches = uint64_t(h->launches);
  return KVQ_OK;
}

kvq_status kvq_read_pool(kvq_handle h, void* host_dst, uint64_t bytes, void* stream_) {
  if (!h || !host_dst) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  kvq_status st = device_guard(h);
  if (st != KVQ_OK) return st;
  const uint64_t total = uint64_t(h->cfg.num_blocks) * uint64_t(h->geo.block_bytes);
  if (bytes != total) return fail(KVQ_ERR_INVALID_ARG, "bytes must equal num_blocks * block_bytes");
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  KVQ_CUDA(cudaMemcpyAsync(host_dst, h->d_pool, total, cudaMemcpyDeviceToHost, s));
  KVQ_CUDA(cudaStreamSynchronize(s));
  return KVQ_OK;
}

kvq_status kvq_read_residual(kvq_handle h, void* k_host, void* v_host, uint64_t bytes, void* stream_) {
  if (!h || !k_host || !v_host) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  kvq_status st = device_guard(h);
  if (st != KVQ_OK) return st;
  const kvq_config& c = h->cfg;
  const uint64_t total = uint64_t(c.max_seqs) * c.h_kv * c.residual * c.d_h * 2;
  if (bytes != total) return fail(KVQ_ERR_INVALID_ARG, "bytes must equal max_seqs * h_kv * residual * d_h * 2");
  if (total == 0) return KVQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  KVQ_CUDA(cudaMemcpyAsync(k_host, h->d_kres, total, cudaMemcpyDeviceToHost, s));
  KVQ_CUDA(cudaMemcpyAsync(v_host, h->d_vres, total, cudaMemcpyDeviceToHost, s));
  KVQ_CUDA(cudaStreamSynchronize(s));
  return KVQ_OK;
}

kvq_status kvq_sync_status(kvq_handle h, void* stream_, uint32_t* bits_out) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  kvq_status st = device_guard(h);
  if (st != KVQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  KVQ_CUDA(cudaStreamSynchronize(s));
  KVQ_CUDA(cudaGetLastError());
  uint32_t bits = 0;
  KVQ_CUDA(cudaMemcpy(&bits, h->d_err, sizeof(bits), cudaMemcpyDeviceToHost));
  KVQ_CUDA(cudaMemset(h->d_err, 0, sizeof(uint32_t)));
  if (bits_out) *bits_out = bits;
  if (bits) {
    char buf[96];
    std::snprintf(buf, sizeof(buf), "device check fired: error bits 0x%x", bits);
    return fail(KVQ_ERR_DEVICE_CHECK, buf);
  }
  return KVQ_OK;
}

kvq_status kvq_set_decode_event(kvq_handle h, void* event) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  h->decode_event = static_cast<cudaEvent_t>(event);
  return KVQ_OK;
}

kvq_status kvq_pool_device(kvq_handle h, const void** dev_ptr, uint64_t* bytes) {
  if (!h || !dev_ptr || !bytes) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (h->cfg.host_only) return fail(KVQ_ERR_INVALID_ARG, "handle is host-only");
  *dev_ptr = h->d_pool;
  *bytes = uint64_t(h->cfg.num_blocks) * uint64_t(h->geo.block_bytes);
  return KVQ_OK;
}

kvq_status kvq_read_floor(const void* base, const int64_t* offsets, int64_t n_chunks, int64_t span_bytes,
                          int32_t chunk_bytes, int32_t mode, int32_t ctas, int32_t stages, int32_t per_unit,
                          uint32_t* sink, void* stream_) {
  if (!base || !sink) return fail(KVQ_ERR_INVALID_ARG, "base and sink are required");
  if (!aligned16(base) || (reinterpret_cast<uintptr_t>(sink) & 3u))
    return fail(KVQ_ERR_INVALID_ARG, "base must be 16-byte aligned and sink 4-byte aligned");
  if (mode != 0 && mode != 1) return fail(KVQ_ERR_INVALID_ARG, "mode must be 0 (bulk) or 1 (stream)");
  if (ctas < 1 || ctas > 65535) return fail(KVQ_ERR_INVALID_ARG, "ctas must be in [1, 65535]");
  if (span_bytes < 0 || span_bytes % 16) return fail(KVQ_ERR_INVALID_ARG, "span_bytes must be a non-negative multiple of 16");
  if (mode == 0) {
    if (chunk_bytes < 16 || chunk_bytes > 65536 || chunk_bytes % 16)
      return fail(KVQ_ERR_INVALID_ARG, "chunk_bytes must be a multiple of 16 in [16, 65536]");
    if (per_unit < 1 || per_unit > 32) return fail(KVQ_ERR_INVALID_ARG, "per_unit must be in [1, 32]");
    if (stages < 1 || stages > 16) return fail(KVQ_ERR_INVALID_ARG, "stages must be in [1, 16]");
    if (n_chunks < 0) return fail(KVQ_ERR_INVALID_ARG, "n_chunks must be >= 0");
    if (!offsets && n_chunks * int64_t(chunk_bytes) > span_bytes)
      return fail(KVQ_ERR_INVALID_ARG, "n_chunks * chunk_bytes exceeds span_bytes");
    int dev = 0, optin = 0;
    KVQ_CUDA(cudaGetDevice(&dev));
    KVQ_CUDA(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    if (kvq::floor_smem_bytes(chunk_bytes, per_unit, stages) > size_t(optin))
      return fail(KVQ_ERR_INVALID_ARG, "stages * per_unit * chunk_bytes does not fit in shared memory");
  }
  KVQ_CUDA(kvq::launch_floor(base, offsets, n_chunks, span_bytes, chunk_bytes, mode, ctas, stages, per_unit, sink,
                             static_cast<cudaStream_t>(stream_)));
  return KVQ_OK;
}

kvq_status kvq_set_decode_grid(kvq_handle h, int32_t ctas) {
  if (!h) return fail(KVQ_ERR_INVALID_ARG, "handle is null");
  if (ctas < 0 || ctas > kvq::kMaxDecodeGrid) return fail(KVQ_ERR_INVALID_ARG, "ctas must be in [0, 1024]");
  h->decode_override = ctas;
  return KVQ_OK;
}

}  // extern "C"

namespace {

// Decode plans of kvq_decode_attn_noalloc, one per (device, format, max_seqs):
// the first call for a key sizes the pipeline and queries residency, later
// calls reuse the result.
struct NoallocPlan {
  int dev, max_seqs;
  kvq_config fmt;
  kvq::DecodePipe pipe;
  int grid;
};

bool same_format(const kvq_config& a, const kvq_config& b) {
  return a.bits == b.bits && a.asym == b.asym && a.k_axis == b.k_axis && a.g_k == b.g_k && a.g_v == b.g_v &&
         a.scale_fp32 == b.scale_fp32 && a.residual == b.residual && a.page == b.page && a.h_q == b.h_q &&
         a.h_kv == b.h_kv && a.d_h == b.d_h && a.num_blocks == b.num_blocks && a.fp8 == b.fp8;
}

kvq_status noalloc_plan(int dev, const kvq::Geo& g, int max_seqs, kvq::DecodePipe* pipe, int* grid) {
  static std::mutex mu;
  static std::vector<NoallocPlan> plans;
  kvq_config key{};
  key.bits = g.bits; key.asym = g.asym; key.k_axis = g.k_axis; key.g_k = g.g_k; key.g_v = g.g_v;
  key.scale_fp32 = g.scale_fp32; key.residual = g.R; key.page = g.P; key.h_q = g.h_q; key.h_kv = g.h_kv;
  key.d_h = kvq::kD; key.num_blocks = g.num_blocks; key.fp8 = g.fp8;
  std::lock_guard<std::mutex> lock(mu);
  for (const NoallocPlan& p : plans)
    if (p.dev == dev && p.max_seqs == max_seqs && same_format(p.fmt, key)) {
      *pipe = p.pipe;
      *grid = p.grid;
      return KVQ_OK;
    }
  int sms = 0;
  KVQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  kvq::DecodePipe pp{};
  const cudaError_t pe = kvq::plan_decode(g, max_seqs, &pp);
  if (pe == cudaErrorInvalidConfiguration) return fail(KVQ_ERR_UNSUPPORTED, "decode tile does not fit on this device");
  KVQ_CUDA(pe);
  const int gr = std::min(sms * pp.ctas_per_sm, kvq::kMaxDecodeGrid);
  plans.push_back({dev, max_seqs, key, pp, gr});
  *pipe = pp;
  *grid = gr;
  return KVQ_OK;
}

}  // namespace

extern "C" {

// Decode over caller-owned buffers with the library's fixed scratch array:
// allocates nothing (see include/kvq.h).
kvq_status kvq_decode_attn_noalloc(const kvq_config* cfg, const void* pool, const void* k_window,
                                   const void* v_window, const int32_t* block_table, int32_t bt_stride,
                                   const int32_t* stored_lens, const int32_t* seq_lens, const void* q_bf16,
                                   int32_t batch, float* out, uint32_t* error_bits_dev, void* stream_) {
  kvq_status st = validate(cfg);
  if (st != KVQ_OK) return st;
  if (cfg->fp8) return fail(KVQ_ERR_UNSUPPORTED, "the FP8 format is not served without a handle (its scales live there)");
  if (batch < 0 || batch > cfg->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "batch must be in [0, max_seqs]");
  if (batch == 0) return KVQ_OK;
  if (!pool || !block_table || !stored_lens || !seq_lens || !q_bf16 || !out)
    return fail(KVQ_ERR_INVALID_ARG, "pool, block_table, stored_lens, seq_lens, q and out are required");
  if (cfg->residual > 0 && (!k_window || !v_window))
    return fail(KVQ_ERR_INVALID_ARG, "a format with a BF16 window needs k_window and v_window");
  if (bt_stride < 1) return fail(KVQ_ERR_INVALID_ARG, "bt_stride must be >= 1");
  for (const void* p : {pool, q_bf16, static_cast<const void*>(out), k_window, v_window})
    if (p && !aligned16(p)) return fail(KVQ_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  const kvq::Geo g = make_geo(*cfg);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  int dev = 0;
  KVQ_CUDA(cudaGetDevice(&dev));
  kvq::DecodePipe pipe{};
  int grid = 0;
  st = noalloc_plan(dev, g, cfg->max_seqs, &pipe, &grid);
  if (st != KVQ_OK) return st;

  // scratch layout: [error word | pad to 256][prefix (batch + 1) | pad to 256][partials]
  const size_t off_prefix = 256;
  const size_t off_part = off_prefix + align_up(size_t(batch + 1) * 4, 256);
  const size_t part_bytes = kvq::decode_partials_bytes(g, batch, grid);
  if (off_part + part_bytes > kvq::noalloc_scratch_bytes())
    return fail(KVQ_ERR_INVALID_ARG,
                "batch * h_kv too large for the fixed decode scratch of " +
                    std::to_string(kvq::noalloc_scratch_bytes()) + " bytes (needs " +
                    std::to_string(off_part + part_bytes) + ")");
  void* scratch = nullptr;
  KVQ_CUDA(kvq::noalloc_scratch(&scratch));
  uint8_t* base = static_cast<uint8_t*>(scratch);
  KVQ_CUDA(cudaMemsetAsync(base, 0, sizeof(uint32_t), stream));   // error word starts clear

  kvq::DecodeArgs a{};
  a.pool = static_cast<const uint8_t*>(pool);
  a.kres = static_cast<const uint16_t*>(k_window);
  a.vres = static_cast<const uint16_t*>(v_window);
  a.table = block_table;
  a.table_stride = bt_stride;
  a.table_by_seq = 0;
  a.seq_lens = seq_lens;
  a.seqmap = nullptr;            // row i is sequence i of the caller's buffers
  a.stored_len = stored_lens;
  a.q = static_cast<const uint16_t*>(q_bf16);
  a.out = out;
  a.partials = reinterpret_cast<float*>(base + off_part);
  a.prefix = reinterpret_cast<int32_t*>(base + off_prefix);
  a.err = reinterpret_cast<uint32_t*>(base);
  a.B = batch;
  a.grid = grid;
  a.qk_scale = float(1.4426950408889634 / std::sqrt(double(kvq::kD)));
  a.pipe = pipe;
  a.g = g;
  int launches = 0;
  KVQ_CUDA(kvq::launch_decode(a, stream, nullptr, &launches));
  if (error_bits_dev)
    KVQ_CUDA(cudaMemcpyAsync(error_bits_dev, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice, stream));
  return KVQ_OK;
}

}  // extern "C"
