/*
 * v4kv -- single-query decode attention over a paged, heterogeneous,
 * compressed KV cache (DeepSeek-V4-style), for NVIDIA B200 (sm_100a).
 *
 * Source of the method: "DeepSeek-V4 Serving: KV cache and vLLM"
 * (wmrh.cn/news/47220), cited below as P1 with its section numbers.
 *
 * The cache has three parts (P1 §2):
 *   - compressed entries, one shared K = V vector per entry (P1 §2.1): a c4a
 *     layer folds every 4 raw tokens into one entry, a c128a layer every 128;
 *   - a sliding window of the last W (128) raw tokens, uncompressed (P1 §2.3);
 *   - in c4a layers, a small indexer cache whose scores pick the entries a
 *     query reads (P1 §2.2).
 * Every kind is stored in 256-raw-token logical blocks (P1 §3.1.1: 64 c4a
 * entries, 2 c128a entries or 256 raw tokens per block), each block mapped to
 * one physical page of its pool through a per-sequence block table.
 *
 * Conventions for every call:
 *   - Memory: the caller owns all memory. Pointers marked "device" are CUDA
 *     device pointers; the library never allocates, frees or synchronises.
 *     Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns before it runs.
 *   - Alignment: every device data pointer must be 16-byte aligned.
 *   - Errors: a call returns V4KV_OK or an error code after checking its
 *     arguments on the host; nothing is launched when it fails. Problems only
 *     the device can see (a block-table entry outside [0, num_pages), a slot
 *     or index out of range) are never dereferenced: the kernel skips the
 *     access and ORs a V4KV_DEV_* bit into *dev_status (device int32, may be
 *     NULL). Kernels never trap and never wait on other blocks.
 *   - Types: int32 sizes and indices, int64 slots.
 */
#ifndef V4KV_H
#define V4KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t v4kv_status;
#define V4KV_OK 0
#define V4KV_ERR_INVALID_ARG 1 /* null pointer, bad size, misaligned, ... */
#define V4KV_ERR_UNSUPPORTED 2 /* shape or device this build does not run */
#define V4KV_ERR_CUDA 3        /* a CUDA launch or attribute call failed  */

/* bits ORed into *dev_status by kernels */
#define V4KV_DEV_BAD_PAGE 1  /* block-table entry outside [0, num_pages)   */
#define V4KV_DEV_BAD_SLOT 2  /* slot or logical block beyond its table     */
#define V4KV_DEV_BAD_INDEX 4 /* top-k index outside the stored entries     */
#define V4KV_DEV_OVERFLOW 8  /* output array too small for what is needed  */
#define V4KV_DEV_TIMEOUT 16  /* a wait inside a kernel gave up (no progress) */
#define V4KV_DEV_RANGE 32    /* a bf16 value beyond the f16 range met the     */
                             /* 64-head tensor-core path and was clamped      */

typedef enum { V4KV_BF16 = 0, V4KV_FP8_E4M3 = 1, V4KV_FP32 = 2, V4KV_FP4_E2M1 = 3 } v4kv_dtype;

/* One paged pool of one cache kind (P1 §3.1.1, §3.1.3).
 *   data   device, [num_pages, slots_per_page, dim] elements of `dtype`
 *          (fp8-e4m3 codes or bf16; for fp4-e2m1, accepted by the indexer
 *          only, dim / 2 bytes per slot, dim 2i in the low nibble of byte i);
 *          one page = one 256-token logical block.
 *   scales device, [num_pages, slots_per_page] fp32, one absmax scale per
 *          fp8 or fp4 entry (value = float(code) * scale); NULL for bf16.
 *   block_table device, [batch, max_blocks] int32: logical block -> page;
 *          -1 marks a block that has no page (skipped on write, an error on
 *          read). Logical index j of a sequence lives in page
 *          block_table[b][j / slots_per_page], slot j % slots_per_page. */
typedef struct {
  void* data;
  float* scales;
  int32_t num_pages;
  int32_t slots_per_page;
  int32_t dim;
  int32_t dtype;
  const int32_t* block_table;
  int32_t max_blocks;
} v4kv_paged;

/* Rotary embedding on dims [rope_offset, rope_offset + rope_dim): interleaved
 * pairs (off + 2i, off + 2i + 1) rotated by pos * theta^(-2i / rope_dim).
 * rope_dim == 0 disables it. The model uses theta 1e6, 64 dims at offset 448
 * (P1 §2.1: keys carry RoPE, the output gets the inverse). */
typedef struct {
  double theta;
  int32_t rope_dim;
  int32_t rope_offset;
} v4kv_rope;

/* Human-readable name of a status code (static string). */
const char* v4kv_status_string(v4kv_status s);

/* Library ABI version (increases when a signature changes). */
int32_t v4kv_version(void);

/*
 * v4kv_slot_mapping -- physical slots of the logical indices an append
 * touches (P1 §3.1.1: 256-token logical blocks mapped to pages).
 *
 * For sequence b, appending raw tokens [seq_start[b], seq_start[b] + n_new[b])
 * touches logical indices [seq_start/ratio, ceil((seq_start + n_new)/ratio))
 * (none if n_new == 0): compressed entries for ratio 4 or 128, raw tokens for
 * ratio 1. Index j maps to slot
 *     block_table[b][j / slots_per_page] * slots_per_page + j % slots_per_page.
 *   block_table  device [batch, max_blocks] int32
 *   seq_start, n_new  device [batch] int32
 *   cu_out       device [batch + 1] int32, optional: exclusive prefix sums of
 *                the per-sequence counts (sequence b's slots are
 *                slot_out[cu_out[b] .. cu_out[b+1]))
 *   slot_out     device [slot_capacity] int64; a slot whose page is -1 or out
 *                of range is written as -1 and flagged (V4KV_DEV_BAD_PAGE /
 *                V4KV_DEV_BAD_SLOT); indices past slot_capacity are dropped
 *                and flagged V4KV_DEV_OVERFLOW.
 */
v4kv_status v4kv_slot_mapping(const int32_t* block_table, int32_t max_blocks, int32_t batch,
                              const int32_t* seq_start, const int32_t* n_new, int32_t ratio,
                              int32_t slots_per_page, int32_t num_pages, int32_t* cu_out,
                              int64_t* slot_out, int64_t slot_capacity, int32_t* dev_status,
                              void* stream);

/*
 * v4kv_compress_append -- append raw tokens to one layer's cache: compress
 * them into entries, copy the last window_len of them into the window, and
 * keep the unfinished group as compressor state.
 * (P1 §2.1 compression; §2.3 window; §3.1.2 compressor state; §3.2.1 the
 * fused compressor + RoPE + cache-insert kernel.)
 *
 * For every group g touched by the new tokens (see v4kv_slot_mapping), with
 * present tokens t in [g*r, min((g+1)*r, end)), end = seq_start + n_new:
 *     w_t = softmax_t(gate_t + pos_bias[t - g*r])     (fp32, expf)
 *     e   = sum_t w_t * x_t                          (fp32; ratio 4: ascending t;
 *                                                     ratio 128: 8 runs of 16 tokens,
 *                                                     each ascending, added in order)
 *     e   = RoPE(e, position g*r)                    (angles in fp64)
 * then e is stored at slot_mapping[cu_entries[b] + (g - seq_start/r)]:
 * fp8 pools quantise per entry (amax, scale = amax/448 or 1 if amax == 0,
 * code = e4m3_rn_satfinite(e / scale)), bf16 pools round to nearest even.
 * A group not yet complete is stored normalised over its present tokens and
 * rewritten by later appends. Tokens t >= max(seq_start, end - window_len)
 * are also written, RoPE'd at position t, to the window pool (page
 * window->block_table[b][t/256], slot t % 256; a -1 page is skipped).
 *   x            device bf16 [total_tokens, dim], sequence b's chunk is rows
 *                cu_seqlens[b] .. cu_seqlens[b+1]
 *   gate         device fp32 [total_tokens], one logit per raw token
 *   cu_seqlens   device int32 [batch + 1]
 *   seq_start    device int32 [batch], tokens appended before this call
 *   pos_bias     device fp32 [ratio]
 *   ratio        4 or 128; dim a multiple of 8 in [8, 1024]
 *   state_x      device bf16 [batch, ratio, dim], state_gate fp32
 *                [batch, ratio]: rows 0 .. (seq_start % ratio) - 1 hold the
 *                tokens of the unfinished group on entry; updated in place to
 *                rows 0 .. (end % ratio) - 1 on return. Start from any
 *                contents when seq_start == 0.
 *   main_cache   entry pool (slots_per_page = 256 / ratio), dim == `dim`
 *   slot_mapping device int64 and cu_entries device int32 [batch + 1], as
 *                produced by v4kv_slot_mapping(ratio) for this append;
 *                slot_mapping must hold all cu_entries[batch] slots
 *                (total_tokens / ratio + 2 * batch always suffices). Both
 *                NULL: the kernel derives the same slots from
 *                main_cache->block_table itself (one launch instead of two;
 *                batch < 1024, else V4KV_ERR_UNSUPPORTED). Exactly one NULL
 *                is V4KV_ERR_INVALID_ARG.
 *   window       window pool (bf16 or fp8, slots_per_page 256) or NULL
 *   prequant_out device fp32 [cu_entries[batch], dim] or NULL: the fp32
 *                values handed to the quantiser (after RoPE)
 * Rejects dim > 1024, dim % 8, ratio not in {4, 128}, rope dims outside dim.
 */
v4kv_status v4kv_compress_append(const void* x, const float* gate, const int32_t* cu_seqlens,
                                 const int32_t* seq_start, int32_t batch, int32_t total_tokens,
                                 const float* pos_bias, int32_t ratio, v4kv_rope rope,
                                 void* state_x, float* state_gate, const v4kv_paged* main_cache,
                                 const int64_t* slot_mapping, const int32_t* cu_entries,
                                 const v4kv_paged* window, int32_t window_len,
                                 float* prequant_out, int32_t* dev_status, void* stream);

/*
 * v4kv_compress_append_ex -- v4kv_compress_append with the compressor
 * variants the pages describe (P1 §2.1; §3.1.2 "an 8-token overlapping
 * state" for c4a; §3.2.1 RMSNorm in the compressor fusion). opts NULL or all
 * zero is v4kv_compress_append.
 *   overlap          1: entry g folds the present tokens [g*r - r, g*r + r)
 *                    (ratio 4 only, else V4KV_ERR_UNSUPPORTED); pos_bias then
 *                    holds 2r values, token t taking pos_bias[t - (g*r - r)];
 *                    the state holds 2r rows per sequence (state_x
 *                    [batch, 2r, dim], state_gate [batch, 2r]); the RoPE
 *                    position stays g*r
 *   gate_per_channel 1: gate is fp32 [total_tokens, dim], one logit per token
 *                    and dim, and the softmax over an entry's tokens is taken
 *                    per dim; state_gate is then [batch, rows, dim]; gate and
 *                    state_gate 16-byte aligned
 *   norm_weight      fp32 [dim], 16-byte aligned, or NULL: the summed entry
 *                    becomes e * w / sqrt(mean(e^2) + norm_eps) before RoPE
 *                    (norm_eps 0 means 1e-6)
 * With overlap or per-channel gates one block builds each entry (a slower
 * kernel than the plain path); RMSNorm alone keeps the plain kernels.
 */
typedef struct v4kv_compress_opts {
  int32_t overlap;
  int32_t gate_per_channel;
  const float* norm_weight;
  float norm_eps;
} v4kv_compress_opts;

v4kv_status v4kv_compress_append_ex(const void* x, const float* gate, const int32_t* cu_seqlens,
                                    const int32_t* seq_start, int32_t batch, int32_t total_tokens,
                                    const float* pos_bias, int32_t ratio, v4kv_rope rope,
                                    void* state_x, float* state_gate, const v4kv_paged* main_cache,
                                    const int64_t* slot_mapping, const int32_t* cu_entries,
                                    const v4kv_paged* window, int32_t window_len,
                                    float* prequant_out, const v4kv_compress_opts* opts,
                                    int32_t* dev_status, void* stream);

/*
 * v4kv_qk_prepare -- the decode step's query heads and new window row in one
 * launch (P1 §3.2.1, "fused Q norm + KV RoPE + K insert": one warp per query
 * head or K row, no communication between them).
 * For every sequence b and head h:
 *     q_out[b][h] = RoPE(RMSNorm(q_in[b][h]), positions[b])
 * with RMSNorm(v) = v * w / sqrt(mean(v^2) + q_norm_eps) (skipped when
 * q_norm_weight is NULL; q_norm_eps 0 means 1e-6) and RoPE as in
 * v4kv_compress_append (angles in fp64, the rotation in fp32). When k_new and
 * window are given, the new token's K = V row is rotated at positions[b] and
 * stored in the window pool (page window->block_table[b][pos / 256], slot
 * pos % 256; bf16, or fp8 with its own scale; a -1 page is skipped), exactly
 * as the compressor stores its window rows.
 *   q_in          device fp32 [batch, heads, dim], 16-byte aligned
 *   q_out         device [batch, heads, dim], fp32 or bf16 (q_out_dtype)
 *   q_norm_weight device fp32 [dim] or NULL
 *   positions     device int32 [batch], the new token's position (L - 1)
 *   k_new         device bf16 [batch, dim] or NULL
 *   window        window pool (slots_per_page 256) or NULL
 * Rejects dim > 1024 or dim % 8, unaligned buffers, rope dims outside dim.
 * Out-of-range window blocks or pages are flagged in dev_status and skipped.
 */
v4kv_status v4kv_qk_prepare(const float* q_in, int32_t batch, int32_t heads, int32_t dim,
                            const float* q_norm_weight, float q_norm_eps, const int32_t* positions,
                            v4kv_rope rope, void* q_out, int32_t q_out_dtype, const void* k_new,
                            const v4kv_paged* window, int32_t* dev_status, void* stream);

/*
 * v4kv_index_topk -- indexer scores and exact top-k over a c4a layer's
 * visible entries (P1 §2.2 indexer cache; P1 §4.1 sparse attention over
 * the selected c4a entries).
 *
 * q_idx (fp32 [dim]) is quantised per vector like an entry (codes q8, scale
 * qs). For entry j < n_vis = floor(max(0, L - window_len) / ratio):
 *     acc = fp32 fused multiply-add chain over d = 0 .. dim-1 of q8[d]*k8_j[d]
 *     score_j = acc * kscale_j                       (fp32)
 * The min(k, n_vis) best entries by (score descending, index ascending;
 * -0 == +0) are written to topk_out[b] in that order, padded with -1;
 * score_out (optional) receives score_j * qs (0 for padding).
 *   q_idx        device fp32 [batch, dim]
 *   idx_cache    fp8 or fp4 indexer pool, slots_per_page = 256 / ratio,
 *                dim a multiple of 32 in [32, 512] (fp4: P1 §2 keeps the c4a
 *                indexer in fp4; each product of an e4m3 query value and an
 *                e2m1 key value is exact, so the chain is the same)
 *   seq_lens     device int32 [batch], L of each sequence (tokens so far)
 *   max_seq_len  host upper bound of seq_lens (sizes the launch)
 *   k            1 .. 2048
 *   workspace    device scratch of v4kv_workspace_size(V4KV_OP_INDEX_TOPK)
 *                bytes, 256-byte aligned; contents need not be initialised.
 */
v4kv_status v4kv_index_topk(const float* q_idx, const v4kv_paged* idx_cache,
                            const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                            int32_t ratio, int32_t window_len, int32_t k, int32_t* topk_out,
                            float* score_out, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream);

/*
 * v4kv_decode_attention -- one query token per sequence attends to its
 * compressed entries plus its raw-token window; shared K = V; inverse RoPE
 * on the output (P1 §2.1, §2.3; c4a with the indexer's selection, P1 §2.2).
 *
 * J_b = { entries j < n_vis } (topk == NULL) or { topk[b][i] >= 0 }, plus
 * window tokens [max(0, L - window_len), L). With v_j the stored value
 * (fp8 code * scale, or bf16):
 *     s_hj = sm_scale * q_h . v_j,  p = softmax_j(s),  o_h = sum_j p_hj v_j
 *     out  = inverse RoPE of o at position L - 1, rounded to bf16.
 * Numerics: q and p enter the tensor cores as f16 (q scaled per sequence by a
 * power of two), fp8 values convert exactly, accumulation is fp32. With 64
 * heads (the tensor-core path) bf16 entries and window tokens are rounded to
 * f16 as well: magnitudes of 2^16 or more are clamped to 65504 and flagged
 * V4KV_DEV_RANGE; magnitudes below 2^-14 keep an absolute error of at most
 * 2^-25. Other head counts use bf16 values exactly. Any fp8 scale is valid,
 * including zero (the entry's value is 0) and negative scales.
 *   sm_scale     softmax scale; 0 selects the default 1/sqrt(512)
 *   q            device [batch, heads, dim], fp32 or bf16 (q_dtype), with RoPE
 *                already applied at position L - 1
 *   heads        1 .. 128; dim (of q, main_cache and window) must be 512
 *   main_cache   entry pool (fp8 or bf16), slots_per_page = 256 / ratio
 *   window       raw-token pool (bf16 or fp8), slots_per_page = 256
 *   seq_lens     device int32 [batch]; max_seq_len host upper bound
 *   topk         device int32 [batch, k] or NULL
 *   out          device bf16 [batch, heads, dim]
 *   workspace    device scratch of v4kv_workspace_size(V4KV_OP_DECODE)
 *                bytes, 256-byte aligned; contents need not be initialised.
 */
v4kv_status v4kv_decode_attention(const void* q, int32_t q_dtype, int32_t batch, int32_t heads,
                                  const v4kv_paged* main_cache, const v4kv_paged* window,
                                  const int32_t* seq_lens, int32_t max_seq_len, int32_t ratio,
                                  int32_t window_len, const int32_t* topk, int32_t k,
                                  float sm_scale, v4kv_rope rope, void* out, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * v4kv_decode_attention_fp8out -- v4kv_decode_attention with the output
 * quantised to fp8-e4m3 in the same epilogue as the inverse RoPE (P1 §3.2.1:
 * inverse RoPE fused with fp8 quantisation, for a next layer that reads fp8).
 * Each (sequence, head) vector o (fp32, after the inverse RoPE) is quantised
 * like a cache entry: amax = max_d |o_d|, scale = amax / 448 (IEEE fp32
 * division; 1 if amax == 0), code_d = e4m3_rn_satfinite(o_d / scale).
 *   out_codes    device uint8 [batch, heads, 512]
 *   out_scales   device fp32 [batch, heads]
 *   prequant_out device fp32 [batch, heads, 512] or NULL: the fp32 values
 *                handed to the quantiser
 * Every other argument, the workspace (same size) and the errors are those of
 * v4kv_decode_attention.
 */
v4kv_status v4kv_decode_attention_fp8out(const void* q, int32_t q_dtype, int32_t batch,
                                         int32_t heads, const v4kv_paged* main_cache,
                                         const v4kv_paged* window, const int32_t* seq_lens,
                                         int32_t max_seq_len, int32_t ratio, int32_t window_len,
                                         const int32_t* topk, int32_t k, float sm_scale,
                                         v4kv_rope rope, void* out_codes, float* out_scales,
                                         float* prequant_out, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_status,
                                         void* stream);

/*
 * v4kv_decode_attention_noalloc -- v4kv_decode_attention for callers that
 * cannot allocate device memory. The paper has no counterpart: this is a
 * deployment convenience of this library.
 *
 * Some callers cannot call cudaMalloc (or any allocator) where they run
 * decode attention -- for example code that runs inside another framework's
 * memory pool, or a serving thread that must not synchronise or take an
 * allocator lock per request -- so they cannot provide the workspace that
 * v4kv_decode_attention needs. This entry point takes the same arguments
 * without the workspace and uses a fixed scratch array of
 * V4KV_NOALLOC_SCRATCH_BYTES that lives in the library's device memory image:
 * every GPU that loads the library holds it until the process exits. It
 * allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 *   - Sizes: returns V4KV_ERR_INVALID_ARG, launching nothing, when the
 *     workspace v4kv_workspace_size(V4KV_OP_DECODE, ...) reports for these
 *     arguments exceeds V4KV_NOALLOC_SCRATCH_BYTES.
 *   - First call on a device: it looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current, once per device; make
 *     that first call before any stream capture.
 *   - Sharing: all calls on a device share the one scratch array, which keeps
 *     the last call's contents; nothing in it needs to start at zero (a call
 *     writes every partial result it reads). Calls that overlap on the GPU
 *     (other streams, other host threads on the same device) race on the
 *     scratch and must be serialised by the caller.
 */
#define V4KV_NOALLOC_SCRATCH_BYTES (32u << 20)
v4kv_status v4kv_decode_attention_noalloc(const void* q, int32_t q_dtype, int32_t batch,
                                          int32_t heads, const v4kv_paged* main_cache,
                                          const v4kv_paged* window, const int32_t* seq_lens,
                                          int32_t max_seq_len, int32_t ratio, int32_t window_len,
                                          const int32_t* topk, int32_t k, float sm_scale,
                                          v4kv_rope rope, void* out, int32_t* dev_status,
                                          void* stream);

#define V4KV_OP_INDEX_TOPK 1
#define V4KV_OP_DECODE 2

/* Scratch bytes the call `op` needs for these sizes (host only; queries the
 * current device's SM count). For V4KV_OP_DECODE pass the same heads,
 * max_seq_len, ratio, window_len, k (0 when topk is NULL), main dtype
 * (main_dtype) and dim as the decode call. */
v4kv_status v4kv_workspace_size(int32_t op, int32_t batch, int32_t heads, int32_t max_seq_len,
                                int32_t ratio, int32_t window_len, int32_t k, int32_t main_dtype,
                                int32_t dim, size_t* bytes);

/* Cache bytes of one sequence of n_tokens raw tokens (host only; P1 §2):
 * per layer ceil(n/r) entries of (dim * entry_bytes + entry_scale_bytes),
 * plus, for ratio-4 layers, ceil(n/4) indexer keys of (indexer_dim *
 * indexer_bytes + indexer_scale_bytes), plus min(window, n) raw tokens of
 * dim * window_bytes. Element sizes are in bits so that fp4 (4) fits. */
typedef struct {
  int32_t n_layers;
  const int32_t* layer_ratios; /* host [n_layers], 4 or 128 */
  int32_t dim;
  int32_t entry_bits;
  int32_t entry_scale_bytes;
  int32_t indexer_dim;
  int32_t indexer_bits;
  int32_t indexer_scale_bytes;
  int32_t window;
  int32_t window_bits;
} v4kv_footprint_cfg;

uint64_t v4kv_kv_footprint_bytes(uint64_t n_tokens, const v4kv_footprint_cfg* cfg);

/*
 * Unified page pools (host only; P1 §3.1.3, "unifying page sizes").
 *
 * Every cache kind keeps one 256-token logical block per physical page, so
 * its page size is (256 / ratio) x bytes per entry (P1 §3.1.3 writes it as
 * block_size x compress_ratio x per_entry_size). Instead of one pool per kind,
 * the kinds are grouped into a few buckets (three on the page), each a pool of
 * fixed-size pages: the grouping is planned once ("static planning") and
 * requests then take whole pages of their kind's bucket ("dynamic
 * allocation"), with no compaction or migration between pools. These calls
 * only hand out page indices; the caller owns the device memory of each
 * bucket (bucket_bytes[b] x pages) and writes the indices into its block
 * tables. Thread-safe: each pool object serialises its own calls.
 */

/* Page bytes of a kind: (256 / ratio) x (ceil(dim x elem_bits / 8) +
 * scale_bytes); ratio 1 for raw-token pools. 0 for invalid arguments. */
uint64_t v4kv_page_bytes(int32_t ratio, int32_t dim, int32_t elem_bits, int32_t scale_bytes);

/* Group n_kinds page sizes into at most max_buckets buckets. Sizes are split
 * in ascending order into contiguous groups whose page size is the group's
 * largest member, minimising the largest ratio (bucket page / kind page) over
 * the kinds, then the sum of those ratios. Kinds with equal page sizes always
 * share a bucket. Writes bucket_of[n_kinds] (bucket 0 = the largest pages),
 * bucket_bytes[*n_buckets] and *n_buckets (<= max_buckets).
 * V4KV_ERR_INVALID_ARG for a null pointer, a count <= 0 or a zero size. */
v4kv_status v4kv_plan_buckets(int32_t n_kinds, const uint64_t* page_bytes, int32_t max_buckets,
                              int32_t* bucket_of, uint64_t* bucket_bytes, int32_t* n_buckets);

typedef struct v4kv_page_pools v4kv_page_pools; /* opaque host object */

/* Create the pools: pages_per_bucket[b] pages of bucket_bytes[b] each, all
 * free (page indices 0 .. pages_per_bucket[b] - 1, handed out lowest first). */
v4kv_status v4kv_page_pools_create(int32_t n_buckets, const uint64_t* bucket_bytes,
                                   const int32_t* pages_per_bucket, v4kv_page_pools** out);
void v4kv_page_pools_destroy(v4kv_page_pools* pools);

/* Take n pages of `bucket` into pages_out[n]. If fewer than n are free,
 * nothing is taken and V4KV_ERR_UNSUPPORTED is returned. */
v4kv_status v4kv_page_alloc(v4kv_page_pools* pools, int32_t bucket, int32_t n, int32_t* pages_out);

/* Return n pages of `bucket`. All or nothing: a page that is not allocated,
 * out of range or listed twice gives V4KV_ERR_INVALID_ARG and frees none. */
v4kv_status v4kv_page_free(v4kv_page_pools* pools, int32_t bucket, int32_t n, const int32_t* pages);

/* Free pages left in `bucket` (-1 for a bad bucket or pool). */
int64_t v4kv_pages_free(v4kv_page_pools* pools, int32_t bucket);

#ifdef __cplusplus
}
#endif

#endif /* V4KV_H */
