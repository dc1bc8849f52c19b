// kvq_internal.h -- types shared by the host runtime and the CUDA kernels of
// libkvq.so (not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

constexpr int kD = 128;            // head dimension supported by the kernels
constexpr int kDecodeWarps = 4;    // warps per decode CTA; each stages and computes its own units
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kFlushThreads = 256;
constexpr int kMaxPagesPerGroup = 8;
// flush plan entry: seq, group, n_pages, blocks[kMaxPagesPerGroup]
constexpr int kFlushEntryInts = 3 + kMaxPagesPerGroup;

// Byte geometry of a format (the layout described in kvq.h).
struct Geo {
  int bits, asym, k_axis, g_k, g_v, scale_fp32, R, P, h_q, h_kv, G;
  int n;                    // codes per 32-bit word
  int row_bytes;            // key row: D * bits / 8
  int sub_bytes;            // 16-token sub-tile of codes
  int es;                   // bytes per stored scale / zero-point
  int nvg, nkg;             // value groups per row; key groups per row (token axis)
  int kslice;               // channel axis: key-scale entries per block
  int secK, secV, secVm, secKm;
  int off_V, off_Vm, off_Km;
  int chunk_used;           // off_Km + secKm (bytes a decode stage copies per page)
  int64_t chunk_bytes, block_bytes;
  int num_blocks, max_seqs, mbps;
  int tileT;                // tokens per quantized decode tile
  int lg_P, lg_gk, lg_kslice;   // log2 of page, g_k and kslice (powers of two)
  int fp8;                  // 1: FP8 E4M3 elements, one scale per kv head (no metadata)
  int vm16, km16;           // token-axis stage: metadata bytes of 16 rows
  int qtile_bytes;          // bytes staged for one quantized tile
};

// Device view of an append plan: one int32 array with sections.  A plan of
// at most kPlanInline entries travels inside the launch parameters (`inl`,
// `plan` null), so a decode-sized append needs no host-to-device copy; a
// larger one is uploaded first and read through `plan`.
constexpr int kPlanInline = 880;
struct PlanView {
  const int32_t* plan;
  int n_tok, n_flush, n_res, n_tab, n_len, n_zero;
  int off_tok, off_flush, off_src, off_res, off_tab, off_len, off_zero;
  int32_t inl[kPlanInline];
};

struct DevState {
  uint8_t* pool;
  uint16_t* kres;
  uint16_t* vres;
  int32_t* table;
  int32_t* len;
  uint32_t* err;
  const float* fp8;   // FP8 format: [2][h_kv] scales (keys, then values)
};

// Shape of the decode pipeline for a format (see kvq_decode.cu).
struct DecodePipe {
  int sup;          // tokens per quantized work unit (64, or g_k when larger)
  int lg_sup;       // log2(sup)
  int qsub;         // token axis: bytes of one staged 16-token sub-tile
  int stage_bytes;  // one stage: a quantized unit or a 16-token BF16 window tile
  int nstages;
  int ctas_per_sm;  // resident CTAs per SM at the largest batch
  int ws;           // the warp-specialised kernel: 1 INT4 KIVI, 2 INT2 KIVI, 3 INT8 keys per token
};

struct DecodeArgs {
  const uint8_t* pool;
  const uint16_t* kres;
  const uint16_t* vres;
  const int32_t* table;
  int32_t table_stride;
  int32_t table_by_seq;
  const int32_t* seq_lens;
  const int32_t* seqmap;      // may be null: row i = sequence i
  const int32_t* stored_len;
  const uint16_t* q;
  const float* fp8;           // FP8 format: [2][h_kv] scales (keys, then values)
  float* out;
  float* partials;            // [(B * h_kv + grid) * kDecodeWarps * G][D + 2]
  int32_t* prefix;            // [B + 1], written by CTA 0
  uint32_t* err;
  int32_t B;
  int32_t grid;
  float qk_scale;             // log2(e) / sqrt(D)
  DecodePipe pipe;
  Geo g;
};

// Chunked-prefill attention (kvq_prefill.cu).  The plan holds three int32
// sections: rows [n][2] = (row, position) sorted by sequence and position;
// blocks [nb][4] = (sequence, first row entry, rows, quantized length); tasks
// [n_tasks][5] = (block, kv head, split, first unit, end unit), one CTA each.
constexpr int kPrefillMaxPages = 1024;   // block ids one task caches in shared memory
struct PrefillArgs {
  const uint8_t* pool;
  const uint16_t* kres;
  const uint16_t* vres;
  const int32_t* table;       // the handle's block table [max_seqs][table_stride]
  int32_t table_stride;
  const uint16_t* q;          // bf16 [n][h_q][D]
  float* out;                 // fp32 [n][h_q][D]
  float* part;                // with splits > 1: records [n][h_q][splits][D + 2]
  const int32_t* plan;
  int32_t off_rows, off_blocks, off_tasks;
  int32_t n_tasks, splits;
  uint32_t* err;
  float qk_scale;             // log2(e) / sqrt(D)
  int32_t sup, lg_sup;        // tokens per unit (whole key groups) and its log2
  int32_t stage_bytes;
  Geo g;
};
// Formats with a prefill kernel: channel-axis keys with the window, 2/4/8-bit
// codes, fp16 scales.  Others run their chunk as decode rows.
bool prefill_supported(const Geo& g);
int prefill_stage_bytes(const Geo& g, int sup);
size_t prefill_smem_bytes(int stage_bytes);
// Resident prefill CTAs per SM for the format (occupancy API; at least 1).
int prefill_ctas_per_sm(const Geo& g, int stage_bytes);
cudaError_t launch_prefill(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches);
// The split records' log-sum-exp merge of a prefill plan with splits > 1.
cudaError_t launch_prefill_merge(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches);
// The tensor-core (tcgen05) prefill of the INT4 KIVI format with 4 query heads
// per kv head (kvq_prefill_tc.cu): blocks of 32 query tokens, one CTA per task.
bool prefill_tc_supported(const Geo& g);
size_t prefill_tc_smem_bytes();
int prefill_tc_stage_bytes();
int prefill_tc_ctas_per_sm();
cudaError_t launch_prefill_tc(const PrefillArgs& a, int64_t n_rows, cudaStream_t s, int* launches);

// Host-side launchers (defined in the .cu files).
// Each launcher adds the number of kernels it launched to *launches.
// Table, length and zeroing updates of a plan; given k and v it also copies
// the plan's window rows (only for a plan with no token rows whose flushes,
// if any, read none of the slots those rows fill).
cudaError_t launch_apply(const Geo& g, const DevState& d, const PlanView& p, const uint16_t* k,
                         const uint16_t* v, cudaStream_t s, int* launches);
// Flush launch; with `with_apply` it also runs the plan's apply body (and the
// window rows when `fuse_rows` is set) in extra CTAs of the same launch.
cudaError_t launch_flush(const Geo& g, const DevState& d, const PlanView& p,
                         const uint16_t* k, const uint16_t* v, bool with_apply, bool fuse_rows,
                         cudaStream_t s, int* launches);
cudaError_t launch_residual(const Geo& g, const DevState& d, const PlanView& p,
                            const uint16_t* k, const uint16_t* v, cudaStream_t s, int* launches);
cudaError_t launch_quant_token(const Geo& g, const DevState& d, const PlanView& p,
                               const uint16_t* k, const uint16_t* v, cudaStream_t s,
                               int* launches);

// Raises kernel `kern`'s dynamic shared-memory limit on device `dev` to at
// least `smem` bytes; never lowers it (kvq_decode.cu).
cudaError_t raise_smem_limit(int dev, const void* kern, size_t smem);

const void* decode_kernel_ptr(const Geo& g);
// Sizes the pipeline for batches up to max_B on the current device, sets the
// kernel's shared-memory limit and finds its residency.
cudaError_t plan_decode(const Geo& g, int max_B, DecodePipe* out);
size_t decode_smem_bytes(const Geo& g, const DecodePipe& p, int B);
size_t decode_partials_bytes(const Geo& g, int B, int grid);
// Launches the attention kernel and the merge; `between` (optional) is
// recorded between them.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, cudaEvent_t between, int* launches);
// Up to three copies from mapped page-locked host memory (device addresses)
// into device memory, run by one kernel; n16 in 16-byte units.
struct PullArgs {
  const void* src[3];
  void* dst[3];
  int64_t n16[3];
  int n;
};
cudaError_t launch_pull(const PullArgs& a, cudaStream_t s, int* launches);
constexpr int kMaxDecodeGrid = 1024;

// HBM read-floor measurement kernels (kvq_floor.cu).  mode 0: bulk copies of
// chunks into per-warp shared-memory stages; mode 1: a 128-bit load stream
// over [base, base + span).
size_t floor_smem_bytes(int chunk_bytes, int per_unit, int stages);
cudaError_t launch_floor(const void* base, const int64_t* offsets, int64_t n_chunks, int64_t span,
                         int chunk_bytes, int mode, int ctas, int stages, int per_unit, uint32_t* sink,
                         cudaStream_t s);

// Fixed decode scratch of kvq_decode_attn_noalloc (kvq_noalloc.cu).
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch(void** out);

}  // namespace kvq
