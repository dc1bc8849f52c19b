// kvq_internal.h -- types shared by the host runtime and the CUDA kernels of
// libkvq.so (not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

constexpr int kD = 128;            // head dimension supported by the kernels
constexpr int kDecodeWarps = 4;    // warps per decode CTA (independent pipelines)
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
  int vm16, km16;           // token-axis stage: metadata bytes of 16 rows
  int qtile_bytes;          // bytes staged for one quantized tile
};

// Device view of an append plan: one int32 array with sections.
struct PlanView {
  const int32_t* plan;
  int n_tok, n_flush, n_res, n_tab, n_len, n_zero;
  int off_tok, off_flush, off_src, off_res, off_tab, off_len, off_zero;
};

struct DevState {
  uint8_t* pool;
  uint16_t* kres;
  uint16_t* vres;
  int32_t* table;
  int32_t* len;
  uint32_t* err;
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
  float* out;
  float* partials;
  int32_t* prefix;            // [B + 1], written by CTA 0
  uint32_t* err;
  int32_t B;
  int32_t nstages;
  int32_t stage_bytes;
  int32_t pre_bytes;          // dynamic smem bytes of the prefix table
  int32_t nw;                 // total warps of the launch
  float qk_scale;             // log2(e) / sqrt(D)
  Geo g;
};

// Host-side launchers (defined in the .cu files).
// Each launcher adds the number of kernels it launched to *launches.
cudaError_t launch_apply(const Geo& g, const DevState& d, const PlanView& p, cudaStream_t s,
                         int* launches);
cudaError_t launch_flush(const Geo& g, const DevState& d, const PlanView& p,
                         const uint16_t* k, const uint16_t* v, cudaStream_t s, int* launches);
cudaError_t launch_residual(const Geo& g, const DevState& d, const PlanView& p,
                            const uint16_t* k, const uint16_t* v, cudaStream_t s, int* launches);
cudaError_t launch_quant_token(const Geo& g, const DevState& d, const PlanView& p,
                               const uint16_t* k, const uint16_t* v, cudaStream_t s,
                               int* launches);

const void* decode_kernel_ptr(const Geo& g);
cudaError_t launch_decode(const DecodeArgs& a, int grid, size_t smem, cudaStream_t s,
                          cudaEvent_t between, int* launches);
size_t decode_smem_bytes(int B, int nstages, int stage_bytes);
int decode_prefix_bytes(int B);

// Fixed decode scratch of kvq_decode_attn_noalloc (kvq_noalloc.cu).
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch(void** out);

}  // namespace kvq
