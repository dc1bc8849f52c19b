/*
 * kvq.h -- C ABI of libkvq.so: a quantized, paged KV cache with decode
 * attention over the packed low-bit cache, for NVIDIA B200 (sm_100a).
 *
 * The method follows the pages on KV-cache quantization:
 *  - llmdaily.org "KV-cache quantization -- making long-context inference fit
 *    in memory" (day 65): the attention equation and the memory formula
 *    (section "Why the KV cache grows so quickly"), the symmetric quantizer
 *    s = max|x| / (2^(b-1) - 1), q = clip(round(x/s), -Q, Q), x_hat = s q and
 *    the asymmetric zero-point variant (section "From BF16 to INT8, INT4, or
 *    even fewer bits"), one scale per group and different grouping directions
 *    for keys and values (section "Why scales and groups matter"), the BF16
 *    residual window (section "Why some systems keep a full-precision
 *    window"), blocks addressed through block tables (section "How this
 *    connects to paging and prefix caching"), and fused dequantization
 *    (section "Why compression may also improve speed");
 *  - oh-bug.com "KV Cache Quantization in Practice": keys per channel, values
 *    per token (the KIVI paragraph), asymmetric 2-bit (the list under
 *    "4-bit / 3-bit / 2-bit"), the FP8 engineering baseline with per-head
 *    scales ("FP8 / INT8: Engineering Baseline", Step 3), and compatibility
 *    with prefix caching and chunked prefill ("Go-Live Checklist").
 * Besides the quantized formats the cache also holds the pages' unquantized
 * BF16 baseline (bits = 16) on the same paged path, as a control.
 *
 * Conventions for every call:
 *  - Plain pointers and sizes only.  "device" pointers are CUDA global memory
 *    of the handle's device; "host" pointers are ordinary CPU memory.
 *    `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *  - Status codes are returned; nothing is thrown and nothing aborts.  The
 *    text of the last failure on the calling thread is kvq_last_error().
 *  - Work is enqueued asynchronously on `stream`; host-side bookkeeping
 *    (lengths, block tables, free list) is updated before the call returns.
 *    A failing kvq_append leaves all state unchanged.
 *  - Device pointers passed in must be 16-byte aligned (KVQ_ERR_INVALID_ARG).
 *  - Kernels check block ids, lengths and grid coverage themselves and record
 *    failures in a device error word instead of faulting; kvq_sync_status()
 *    reports and clears it.
 *  - A handle may be used from one host thread at a time; different handles
 *    may be used from different threads at once (each kernel's shared-memory
 *    limit is one process-wide setting that calls only ever raise).
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kvq_handle_s* kvq_handle;

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or config field   */
  KVQ_ERR_OOM = 2,           /* no free block, block-table row full, or the
                                fail_alloc_after test hook fired               */
  KVQ_ERR_BAD_SEQ = 3,       /* sequence id outside [0, max_seqs)              */
  KVQ_ERR_CUDA = 4,          /* a CUDA runtime call failed                     */
  KVQ_ERR_DEVICE_CHECK = 5,  /* a kernel's own check fired (see kvq_sync_status)*/
  KVQ_ERR_UNSUPPORTED = 6    /* valid but unsupported combination             */
} kvq_status;

/* Bits of the device error word (kvq_sync_status). */
#define KVQ_DEVERR_BLOCK_ID 0x1u   /* block-table entry outside [0, num_blocks)  */
#define KVQ_DEVERR_SEQ_LEN  0x2u   /* seq_lens[i] < 0 or > the stored length      */
#define KVQ_DEVERR_TIMEOUT  0x4u   /* a bounded wait on a copy gave up            */
#define KVQ_DEVERR_SEQ_ID   0x8u   /* decode row names an invalid sequence        */
/* Debug build only (libkvq_debug.so, compiled with KVQ_DEBUG=1): the kernels
 * check every index they compute against the buffer it addresses and skip
 * the access instead of making it. */
#define KVQ_DEVERR_SMEM     0x10u  /* a shared-memory stage read or copy outside
                                      what the unit's copies filled          */
#define KVQ_DEVERR_INDEX    0x20u  /* a global index (plan entry, window slot,
                                      split-K record, pool chunk) outside its
                                      buffer                                  */

enum { KVQ_AXIS_TOKEN = 0, KVQ_AXIS_CHANNEL = 1 };

/* Storage format and capacity of one layer's cache.
 *   bits        8, 4 or 2 bits per stored element, or 16 for the BF16 control:
 *               the same paged cache holding bf16 rows with no quantization (the
 *               pages' BF16 baseline, "From BF16 to INT8, INT4, or even fewer
 *               bits"); it needs k_axis 0, residual 0, asym 0, scale_fp32 0 and
 *               g_k = g_v = 128, and stores each 16-token sub-tile of keys and of
 *               values as 16 natural bf16 rows.
 *   asym        0: symmetric codes in [-Q, Q], Q = 2^(bits-1) - 1;
 *               1: unsigned codes in [0, 2^bits - 1] with a zero-point.
 *   k_axis      KVQ_AXIS_TOKEN: key groups are g_k consecutive channels of
 *               one token (residual must be 0);
 *               KVQ_AXIS_CHANNEL: key groups are g_k consecutive tokens of one
 *               channel (residual must equal g_k; page divides g_k).
 *   g_k, g_v    group sizes: 16, 32, 64 or 128 (g_k is tokens on the channel
 *               axis).  Values are always grouped per token over g_v channels.
 *   scale_fp32  0: scales and zero-points stored as fp16 (round to nearest
 *               even, saturating at 65504); 1: stored as fp32.
 *   residual    R, the BF16 window length (0 or g_k).
 *   page        P tokens per block: a power of two, at least 16.
 *   h_q, h_kv   query and key/value heads; h_q / h_kv must be 1, 2 or 4.
 *   d_h         head dimension: 128.
 *   max_seqs, num_blocks, max_blocks_per_seq   capacity.  The decode
 *               kernels keep 16 bytes of work-list state per batch row in
 *               shared memory beside their stages, so max_seqs is bounded by
 *               the device's per-CTA shared memory: about 10,000 rows on a
 *               B200 (kvq_create returns KVQ_ERR_UNSUPPORTED beyond it).  The
 *               warp-specialised decode kernels of the INT4 / INT2 KIVI-style
 *               and INT8 per-token formats need two CTAs per SM, which holds
 *               up to about 420 / 1,000 / 700 rows of max_seqs; a handle
 *               planned for more rows decodes every batch with the generic
 *               kernel (same results; 44.7 against 41-44 us of attention on
 *               the 16 x 8192-token INT4 workload when last compared).
 *   seed        seeds the free list: a Fisher-Yates shuffle of
 *               [0, num_blocks) driven by splitmix64(seed); blocks are taken
 *               from its front and freed blocks return to its back.
 *   fail_alloc_after  test hook: allocation number k (0-based, cumulative)
 *               fails when k >= fail_alloc_after; -1 disables it.
 *   host_only   1: no device memory and no kernels (host bookkeeping only,
 *               for tests on machines without a GPU).
 *   device      CUDA device ordinal (ignored when host_only).
 *   fp8         1: the FP8 (E4M3) format, the oh-bug.com page's engineering
 *               baseline ("FP8 / INT8: Engineering Baseline"): each element is
 *               e4m3(x / s) (round to nearest even, saturating at +-448) with
 *               one scale s per kv head for keys and one for values
 *               (kvq_set_fp8_scales; 1.0 until set), no per-group metadata.
 *               Needs bits 8, asym 0, k_axis 0, residual 0, scale_fp32 0,
 *               g_k = g_v = 128.  Key rows keep the key-list order with bytes in
 *               natural order; value lane records hold each operand register's
 *               two tokens in adjacent bytes.  0 otherwise. */
typedef struct kvq_config {
  int32_t bits;
  int32_t asym;
  int32_t k_axis;
  int32_t g_k;
  int32_t g_v;
  int32_t scale_fp32;
  int32_t residual;
  int32_t page;
  int32_t h_q;
  int32_t h_kv;
  int32_t d_h;
  int32_t max_seqs;
  int32_t num_blocks;
  int32_t max_blocks_per_seq;
  uint64_t seed;
  int32_t fail_alloc_after;
  int32_t host_only;
  int32_t device;
  int32_t fp8;
} kvq_config;

/* Byte geometry of the paged format.  A block holds `page` token slots of all
 * h_kv heads; block b, head h starts at b * block_bytes + h * chunk_bytes.  A
 * chunk holds, in order: key codes (page/16 sub-tiles of 16 tokens), value
 * codes (same), value scales [page][d_h/g_v] then zero-points, key metadata
 * (token axis: [page][d_h/g_k] scales then zero-points; channel axis: a slice
 * of kslice entries of the group's scales, then zero-points).  The bit-level
 * placement of codes is given in the project's format notes; the CUDA kernels
 * and the CPU oracle implement it independently. */
typedef struct kvq_layout_info {
  uint64_t row_bytes;    /* key row: d_h * bits / 8                         */
  uint64_t sub_bytes;    /* one 16-token sub-tile of codes                  */
  uint64_t off_v;        /* value codes, from the chunk start               */
  uint64_t off_vmeta;    /* value scales (+ zero-points)                    */
  uint64_t off_kmeta;    /* key scales (+ zero-points)                      */
  uint64_t chunk_bytes;  /* one (block, head): 32-byte multiple             */
  uint64_t block_bytes;  /* h_kv * chunk_bytes                              */
  uint64_t kslice;       /* channel axis: key-scale entries per block       */
} kvq_layout_info;

typedef struct kvq_stats_t {
  uint64_t blocks_used;
  uint64_t blocks_free;
  uint64_t tokens_stored;     /* sum of stored lengths                      */
  uint64_t bytes_pool;        /* device bytes of the block pool             */
  uint64_t bytes_residual;    /* device bytes of the BF16 windows (K + V)   */
  uint64_t bytes_workspace;   /* plans, split partials, prefix, error word  */
  uint64_t bytes_formula;     /* tokens_stored by the memory formula (one
                                 layer), kvq_cache_bytes()                  */
  uint64_t kernel_launches;   /* kernels this handle has launched so far    */
} kvq_stats_t;

/* Validates `cfg`, allocates the pool, residual windows, block table and
 * workspace on cfg->device, zero-fills them, and builds the free list.
 * Ownership: the handle owns every allocation until kvq_destroy().
 * Errors: KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED (config, or a decode plan
 * for max_seqs rows that does not fit the device's shared memory),
 * KVQ_ERR_CUDA. */
kvq_status kvq_create(const kvq_config* cfg, kvq_handle* out);

/* Frees everything the handle owns (synchronizes the device first). */
void kvq_destroy(kvq_handle h);

/* Appends n tokens.  k_bf16, v_bf16: device, bf16 [n][h_kv][d_h] (row-major),
 * caller-owned, read before the enqueued work finishes (keep them alive until
 * the stream reaches that point).  seq_ids_host: host int32 [n]; tokens of one
 * sequence are appended in array order, exactly as if appended one at a time.
 * Token-axis formats quantize each token into its page row at once
 * (chipfoundryservices.com "KV Cache Quantization", per-token quantization).
 * Channel-axis formats keep the newest tokens as BF16 in the residual window
 * and, when it holds R = g_k tokens, quantize keys per channel and values per
 * token into the group's pages (day-65 page, "Why some systems keep a
 * full-precision window"; oh-bug.com, KIVI paragraph).
 * Errors (state unchanged): KVQ_ERR_INVALID_ARG, KVQ_ERR_BAD_SEQ, KVQ_ERR_OOM,
 * KVQ_ERR_CUDA. */
kvq_status kvq_append(kvq_handle h, const void* k_bf16, const void* v_bf16,
                      const int32_t* seq_ids_host, int32_t n, void* stream);

/* Decode attention over the packed cache (day-65 page, "Why the KV cache
 * grows so quickly"): for each batch row i and query head hq,
 *   out[i][hq] = softmax(q[i][hq] K^T / sqrt(d_h)) V
 * over positions [0, seq_lens[i]) of the row's sequence, reading kv head
 * hq / (h_q / h_kv), dequantizing codes inside the kernel.
 *   q_bf16      device bf16 [batch][h_q][d_h].
 *   block_table device int32 [batch][bt_stride] (row i = batch row i), or NULL
 *               to use the handle's own table (row = sequence id).
 *   seq_lens    device int32 [batch]: positions to attend, 0 <= seq_lens[i]
 *               <= the stored length (quantized + residual tokens).
 *   seq_ids_host host int32 [batch] mapping rows to sequence ids, or NULL for
 *               row i = sequence i.
 *   out         device fp32 [batch][h_q][d_h]; empty rows give zeros.
 * The key range of every (row, kv head) is split over a persistent grid; a
 * second kernel merges the split partials by log-sum-exp.  The partials live
 * in the handle's workspace; one call at a time per handle may be in flight
 * on the GPU.
 * Errors: KVQ_ERR_INVALID_ARG, KVQ_ERR_BAD_SEQ, KVQ_ERR_CUDA. */
kvq_status kvq_decode_attn(kvq_handle h, const void* q_bf16,
                           const int32_t* block_table, int32_t bt_stride,
                           const int32_t* seq_lens, const int32_t* seq_ids_host,
                           int32_t batch, float* out, void* stream);

/* One decode step from host memory, all enqueued on `stream`:
 *   1. the n new rows k_host, v_host (host bf16 [n][h_kv][d_h]) go to
 *      library-owned device buffers and are appended to sequences
 *      seq_ids_host[i] exactly as kvq_append does;
 *   2. q_host (host bf16 [batch][h_q][d_h]) goes to the device and row i
 *      attends over every stored token of sequence i (kvq_decode_attn with the
 *      library's own lengths, rows 0..batch-1 = sequences 0..batch-1);
 *   3. the output comes back to out_host (host fp32 [batch][h_q][d_h]).
 * out_host holds the result once the stream reaches that point.  Inputs in
 * page-locked memory the device can address (cudaPointerGetAttributes gives a
 * device pointer) come in through one library kernel that reads them over the
 * bus with every load in flight at once (faster than copy-engine copies at
 * these sizes); other inputs are copied (page-locked ones asynchronously,
 * pageable ones with the copy semantics CUDA gives them).  When k_host, v_host
 * and q_host lie back to back in host memory (v right after the n K rows, q
 * right after the n V rows) that is one transfer instead of three.  When
 * out_host is page-locked memory the device can address, the decode writes the
 * output there directly instead of a device buffer plus a device-to-host copy.
 * n = 0 skips the append, batch = 0 the decode.
 * The device buffers grow on demand (a device synchronize, then a reallocation)
 * and live until kvq_destroy; the host buffers stay the caller's and must
 * stay valid until the stream has reached the end of the step.
 * Errors: KVQ_ERR_INVALID_ARG, KVQ_ERR_BAD_SEQ (nothing enqueued), those of
 * kvq_append (state unchanged) and KVQ_ERR_CUDA. */
kvq_status kvq_step_host(kvq_handle h, const void* k_host, const void* v_host,
                         const int32_t* seq_ids_host, int32_t n, const void* q_host,
                         int32_t batch, float* out_host, void* stream);

/* Library-owned device block table: int32 [max_seqs][*stride], entry
 * [s][j] = physical block of logical block j of sequence s, -1 if none.
 * Valid until kvq_destroy; updated by appends in stream order. */
kvq_status kvq_block_table(kvq_handle h, const int32_t** dev_ptr, int32_t* stride);

/* Host copy of one sequence's block-table row: writes up to max_entries ids
 * to dst (host) and the row's length to *n_entries. */
kvq_status kvq_block_table_host(kvq_handle h, int32_t seq, int32_t* dst,
                                int32_t max_entries, int32_t* n_entries);

/* Stored length of a sequence (quantized + residual tokens). */
kvq_status kvq_seq_len(kvq_handle h, int32_t seq, int32_t* len);

/* Library-owned device array int32 [max_seqs] of stored lengths, updated by
 * appends in stream order (usable as seq_lens when rows are sequences). */
kvq_status kvq_seq_lens_device(kvq_handle h, const int32_t** dev_ptr);

/* Releases a sequence's blocks in logical order and resets its length to 0.
 * A block goes to the back of the free list when the last block-table row
 * holding it lets go (blocks can be shared, see kvq_share_prefix).  `stream`
 * orders the device-side reset. */
kvq_status kvq_free_seq(kvq_handle h, int32_t seq, void* stream);

/* Scales of the FP8 format (config fp8 = 1): k_scales and v_scales are host
 * float arrays of h_kv entries, one per kv head (equal entries give a
 * per-tensor scale).  Stored elements are e4m3(x / s) and read back as
 * s * e4m3.  The pages leave calibration out; a caller typically passes
 * amax / 448 of a sample of each head.  Must be called before the first
 * append (KVQ_ERR_INVALID_ARG otherwise, or for a non-FP8 cache or a scale
 * that is not positive and finite).  Synchronises the device. */
kvq_status kvq_set_fp8_scales(kvq_handle h, const float* k_scales, const float* v_scales);

/* Prefix sharing of quantized blocks (the paging section of the day-65 page,
 * "How this connects to paging and prefix caching": blocks are what prefix
 * caching shares).  Makes the empty sequence dst_seq start with the first
 * `tokens` tokens of src_seq by pointing dst's block-table row at src's
 * physical blocks (no copy; each shared block's holder count goes up).
 * Format check: `tokens` must be a multiple of the page for per-token formats
 * and of g_k (a whole key group, whole pages) for per-channel formats, so
 * only full blocks that no later append writes are shared; dst's window
 * starts empty.  Later appends to either sequence take fresh blocks.
 * Errors (no state change): KVQ_ERR_BAD_SEQ for ids out of range;
 * KVQ_ERR_INVALID_ARG for dst not empty, dst == src, tokens outside
 * [0, len(src)] or not aligned; KVQ_ERR_OOM if dst's row is too short.
 * `stream` orders the device-side table and length update. */
kvq_status kvq_share_prefix(kvq_handle h, int32_t src_seq, int32_t dst_seq, int32_t tokens, void* stream);

/* Capacity and usage counters (day-65 page's memory formula for bytes_formula;
 * oh-bug.com checklist item on monitoring KV-cache usage). */
kvq_status kvq_stats(kvq_handle h, kvq_stats_t* out);

/* The day-65 memory formula M = 2 L T H_kv d_h b with b the bytes per element
 * of the format including its group metadata: keys bits/8 + meta/g_k, values
 * bits/8 + meta/g_v, meta = scale bytes (+ zero-point bytes).  For L=32,
 * T=8192, H_kv=8, d_h=128, 4 bits, fp16 scale per 64: 285,212,672 bytes
 * (272 MiB).  Returns 0 for an invalid config. */
uint64_t kvq_cache_bytes(int32_t layers, int64_t tokens, int32_t h_kv, int32_t d_h,
                         const kvq_config* cfg);

/* Byte geometry of a format (no handle needed). */
kvq_status kvq_layout(const kvq_config* cfg, kvq_layout_info* out);

/* Copies the whole block pool (device) to host_dst: num_blocks * block_bytes
 * bytes; synchronizes `stream`.  For parity checks and debugging. */
kvq_status kvq_read_pool(kvq_handle h, void* host_dst, uint64_t bytes, void* stream);

/* Copies the residual windows (device, bf16 [max_seqs][h_kv][R][d_h]) of keys
 * and values to host; each buffer takes `bytes`; synchronizes `stream`. */
kvq_status kvq_read_residual(kvq_handle h, void* k_host, void* v_host, uint64_t bytes,
                             void* stream);

/* Synchronizes `stream`, reads and clears the device error word.  Returns
 * KVQ_ERR_DEVICE_CHECK (and the word in *bits_out if not NULL) when a kernel's
 * check fired, KVQ_ERR_CUDA on a CUDA error, else KVQ_OK. */
kvq_status kvq_sync_status(kvq_handle h, void* stream, uint32_t* bits_out);

/* Library-owned device view of the block pool: *dev_ptr receives its address
 * and *bytes its size (num_blocks * block_bytes).  Valid until kvq_destroy;
 * for measurement (kvq_read_floor over the pages a decode reads) and
 * debugging.  KVQ_ERR_INVALID_ARG for a host-only handle. */
kvq_status kvq_pool_device(kvq_handle h, const void** dev_ptr, uint64_t* bytes);

/* Measurement hook: the HBM read floor of a decode pass.  Decode over a
 * compressed cache is meant to be bound by memory traffic (llmdaily.org
 * day-65, "Why compression may also improve speed"); this call reads bytes
 * and does nothing else with them, so its device time is the floor a single
 * launch can reach for the same bytes and the same way of reading.
 *   base        device, 16-byte aligned; span_bytes (a multiple of 16)
 *               readable bytes from it.
 *   mode 0      bulk: a grid of `ctas` CTAs of four warps; each CTA takes a
 *               contiguous share of the chunk list and each warp every fourth
 *               unit of `per_unit` chunks (1..32), copying it with
 *               cp.async.bulk into one of its `stages` (1..16) shared-memory
 *               stages, as the decode kernel stages pages.  Chunk i is
 *               chunk_bytes (a multiple of 16, <= 65536) at base + offsets[i]
 *               (offsets: device int64 [n_chunks]) or, with offsets NULL, at
 *               base + i * chunk_bytes.
 *   mode 1      stream: 256-thread CTAs read [base, base + span_bytes) with
 *               128-bit loads, eight in flight per thread (chunk arguments
 *               ignored).
 *   sink        device uint32 [2]: sink[0] receives an XOR checksum of one
 *               word per chunk (mode 0) or of every word (mode 1); sink[1]
 *               gets bit 0 for an offset that is negative, unaligned or past
 *               span_bytes (that unit is skipped) and bit 1 for a copy wait
 *               that gave up after 2 s.  Neither is cleared by the call.
 * Asynchronous on `stream`.  KVQ_ERR_INVALID_ARG for out-of-range arguments or
 * stages that do not fit in shared memory. */
kvq_status kvq_read_floor(const void* base, const int64_t* offsets, int64_t n_chunks, int64_t span_bytes,
                          int32_t chunk_bytes, int32_t mode, int32_t ctas, int32_t stages,
                          int32_t per_unit, uint32_t* sink, void* stream);

/* Overrides the decode kernel's grid (number of CTAs); 0 restores the default
 * (one resident wave on every SM).  Changes how the key range is split across
 * CTAs, never the result beyond rounding. */
kvq_status kvq_set_decode_grid(kvq_handle h, int32_t ctas);

/* Profiling hook: when `event` (a cudaEvent_t) is not NULL, every later
 * kvq_decode_attn records it on its stream between the attention kernel and
 * the kernel that merges split partials, so a caller can time the attention
 * kernel alone with CUDA events.  NULL turns it off.  The event stays owned by
 * the caller and must outlive its use. */
kvq_status kvq_set_decode_event(kvq_handle h, void* event);

/* Decode attention (as kvq_decode_attn) over caller-owned cache buffers,
 * allocating no device memory.  The pages have no counterpart to this call:
 * it serves callers that cannot allocate when they decode -- a runtime that
 * hands the library a pre-sized arena, a process that must allocate everything
 * at start-up, or a serving path where allocation is forbidden.  Its scratch
 * (split-K partials, tile prefix, error word) is a fixed 16 MiB array in the
 * library's device image, held by every GPU that loads the library until the
 * process exits; calls size-check against it and never call cudaMalloc,
 * cudaFree or an allocating library routine.  Each call clears the array's
 * error word with cudaMemsetAsync (no allocation).
 *   cfg          format and capacity; max_seqs bounds batch.  Not a handle.
 *   pool         device, num_blocks * block_bytes in the kvq_layout format.
 *   k_window, v_window  device bf16 [batch][h_kv][residual][d_h] BF16 windows
 *                (may be NULL when residual == 0).
 *   block_table  device int32 [batch][bt_stride], row i = batch row i.
 *   stored_lens  device int32 [batch]: tokens stored for row i (quantized +
 *                window), which fixes where the window starts.
 *   seq_lens     device int32 [batch]: positions to attend, <= stored_lens[i].
 *   q_bf16, out  as in kvq_decode_attn (row i uses window row i).
 *   error_bits_dev  optional device uint32: receives this call's device
 *                check bits (KVQ_DEVERR_*), 0 if none fired.
 * Runs on the current CUDA device.  Every call looks up the scratch array's
 * device address in the current context (cudaGetSymbolAddress).  The first
 * call for a (device, format, max_seqs) sizes the decode pipeline, queries
 * residency and may raise the decode kernel's shared-memory limit (the limit
 * only ever rises, so a small plan never breaks a handle planned for a larger
 * batch); later calls reuse that plan.  Make that first call before any
 * stream capture.  All calls share the one array and it keeps the last
 * call's contents: calls whose work can overlap on the GPU (different streams
 * without ordering) race on it.  Returns KVQ_ERR_INVALID_ARG with a message
 * giving both sizes when batch * h_kv needs more scratch than the array holds;
 * KVQ_ERR_UNSUPPORTED for the FP8 format (its per-head scales live in a handle).
 * The partials take (batch * h_kv + grid) * 4 * G * 520 bytes, G = h_q / h_kv
 * and grid = the resident decode CTAs of the format's kernel (2 or 3 per SM:
 * 296 or 444 on 148 SMs): with G = 4 that allows about 1,500 to 1,700
 * (row, kv head) pairs. */
kvq_status kvq_decode_attn_noalloc(const kvq_config* cfg, const void* pool, const void* k_window,
                                   const void* v_window, const int32_t* block_table,
                                   int32_t bt_stride, const int32_t* stored_lens,
                                   const int32_t* seq_lens, const void* q_bf16, int32_t batch,
                                   float* out, uint32_t* error_bits_dev, void* stream);

/* Attention for a chunk of query tokens over the quantized cache (chunked
 * prefill, which oh-bug.com "KV Cache Quantization in Practice" asks a
 * quantized cache to stay compatible with: "Go-Live Checklist" and Step 1 of
 * its four-step approach).  Row i is the query of a token whose
 * keys and values are already appended: it attends positions 0 ..
 * positions_host[i] of sequence seq_ids_host[i] (causal), with the attention
 * of kvq_decode_attn.
 *   q_bf16          device bf16 [n][h_q][d_h].
 *   seq_ids_host    host int32 [n]; positions_host host int32 [n], each a
 *                   stored position of its sequence.
 *   out             device fp32 [n][h_q][d_h].
 * Channel-axis formats with the window (2/4/8-bit codes, fp16 scales) run
 * a prefill kernel whose query tokens of one sequence share every staged
 * tile: the INT4 format with keys per channel G = 64, values per token G = 64,
 * page 16, window 64 and 4 query heads per kv head on the tensor-core kernel
 * (blocks of 32 tokens, 128 rows of the tcgen05 M dimension), the others on
 * the mma.sync kernel (blocks of 64 / g tokens); the key range is split over
 * CTAs and merged by log-sum-exp.  Other formats run as decode launches of at
 * most max_seqs rows, each row reading its own prefix.  Rows may come in any
 * order; the call uploads a small plan (rows sorted by sequence and position)
 * and may grow a workspace (with a device synchronize).  Errors:
 * KVQ_ERR_BAD_SEQ for an id out of range, KVQ_ERR_INVALID_ARG for a position
 * that is not stored or null / unaligned pointers. */
kvq_status kvq_prefill_attn(kvq_handle h, const void* q_bf16, const int32_t* seq_ids_host,
                            const int32_t* positions_host, int32_t n, float* out, void* stream);

/* Text of the last failure on the calling thread ("" if none). */
const char* kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
