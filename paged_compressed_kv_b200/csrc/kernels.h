// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/v4kv.h"

namespace v4kv {

struct PoolArgs {
  void* data;
  float* scales;
  const int32_t* block_table;
  int num_pages;
  int spb;  // slots per page
  int dim;
  int dtype;
  int max_blocks;
};

constexpr int kRopeTable = 32;  // pairs whose frequency the host precomputes

struct RopeArgs {
  double theta;
  int rope_dim;
  int rope_offset;
  double freq[kRopeTable];  // theta^(-2i / rope_dim), i < min(rope_dim / 2, kRopeTable)
};

struct CompressArgs {
  const uint16_t* x;
  const float* gate;
  const int32_t* cu_seqlens;
  const int32_t* seq_start;
  const float* pos_bias;
  const uint16_t* state_x;
  const float* state_gate;
  uint16_t* state_x_out;  // same memory as state_x (updated in place)
  float* state_gate_out;
  const int64_t* slot_mapping;
  const int32_t* cu_entries;
  float* prequant_out;
  int32_t* dev_status;
  PoolArgs main;
  PoolArgs window;
  RopeArgs rope;
  int batch;
  int ratio;
  int dim;
  int window_len;
  // variants (all off by default)
  int overlap;          // 1: entry g folds tokens [g*r - r, g*r + r) (pos_bias has 2r values)
  int gate_dim;         // 1: one logit per token; dim: one per token and dim
  int state_rows;       // rows of the state per sequence: r, or 2r with the overlap
  const float* norm_w;  // [dim] RMSNorm weights, or null
  float norm_eps;
};

struct QkPrepArgs {
  const float* q_in;        // [batch, heads, dim]
  void* q_out;              // [batch, heads, dim] fp32 or bf16
  int q_out_bf16;
  const float* norm_w;      // [dim] or null
  float norm_eps;
  const uint16_t* k_new;    // [batch, dim] bf16 or null
  const int32_t* positions; // [batch]
  PoolArgs window;          // data null: no K insert
  RopeArgs rope;
  int32_t* dev_status;
  int batch;
  int heads;
  int dim;
};

struct IndexArgs {
  const float* q_idx;
  const int32_t* seq_lens;
  int32_t* topk_out;
  float* score_out;
  float* scores_ws;  // [batch, ws_stride] scratch
  uint32_t* hist_ws; // [batch, 4096] histogram of the top 12 bits of the ranking key
  int32_t* dev_status;
  PoolArgs cache;
  int batch;
  int ratio;
  int window_len;
  int k;
  int max_len;        // host bound on seq_lens; longer sequences are clamped and flagged
  int ws_stride;      // max visible entries (row stride of scores_ws)
  int chunk;          // entries scored per block
};

struct DecodePlan {
  int path;          // 0 = CUDA-core kernel, 1 = tensor-core kernel
  int items_max;     // max attended items (entries + window) of one sequence
  int split;         // items per split
  int n_splits;      // splits per sequence (tensor-core path: blocks of the persistent grid)
  size_t ws_bytes;   // partial results
};

struct DecodeArgs {
  const void* q;
  const int32_t* seq_lens;
  const int32_t* topk;
  void* out;
  float* part_o;  // [batch, n_splits, heads, dim]
  float* part_ml; // [batch, n_splits, heads, 2]  (max in log2 units, sum)
  int32_t* dev_status;
  PoolArgs main;
  PoolArgs window;
  RopeArgs rope;
  int q_dtype;
  int batch;
  int heads;
  int dim;
  int ratio;
  int window_len;
  int k;
  float sm_scale;
  int split;
  int n_splits;
  int max_len;  // host bound on seq_lens; longer sequences are clamped and flagged
  int pad_sel;  // 1: entries are padded to a multiple of 128 items (tensor-core path)
  int out_fp8;          // 0: out is bf16; 1: out is e4m3 codes with one fp32 scale per (b, h)
  float* out_scales;    // [batch, heads] when out_fp8
  float* prequant_out;  // optional [batch, heads, dim] fp32: the values handed to the quantiser
  int32_t* cum; // tensor-core path: [batch + 1] tile prefix sums (workspace)
  uint8_t* qh;  // tensor-core path: [batch] f16 query images, 64 KB each (workspace)
  float* qk0;   // tensor-core path: [batch] score multipliers of the f16 images
  long long* costcum;  // tensor-core path: [batch + 1] cost prefix sums (workspace)
  int32_t* cta_x0;     // tensor-core path: [n_splits + 1] first tile of each block's range
  int4* cta_rec;       // tensor-core path: [n_splits] {x0, x1, b0, lt0}: a block's tile range,
                       // the sequence of its first tile and that tile's index in the sequence
  int32_t* cta_L0;     // tensor-core path: [n_splits] length of that sequence (clamped)
  int2* seq_slots;     // tensor-core path: [batch] first and last block meeting the sequence
  float2* rope_tab;    // tensor-core path: [batch][kRopeTable] (cos, sin) at position L - 1
};

cudaError_t launch_slot_mapping(const int32_t* bt, int max_blocks, int batch,
                                const int32_t* seq_start, const int32_t* n_new, int ratio, int spb,
                                int num_pages, int32_t* cu_out, int64_t* slot_out, long long cap,
                                int32_t* st, cudaStream_t stream);

cudaError_t launch_qk_prepare(const QkPrepArgs& p, cudaStream_t stream);
cudaError_t launch_compress_append(const CompressArgs& a, int max_groups, int total_tokens,
                                   cudaStream_t stream);

size_t index_workspace_bytes(int batch, int max_seq_len, int ratio, int window_len);
cudaError_t launch_index_topk(IndexArgs a, int max_seq_len, cudaStream_t stream);

DecodePlan plan_decode(int batch, int heads, int max_seq_len, int ratio, int window_len, int k,
                       int main_dtype, int dim, int num_sms);
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);  // sweep + merge
size_t decode_tc_workspace_bytes(int batch, int num_sms);
void decode_tc_layout(DecodeArgs& a, void* workspace);  // needs batch, n_splits

// Host-side argument checks of decode attention, without the workspace
// (api.cu); V4KV_OK when the call may proceed.
v4kv_status decode_check_args(const void* q, int32_t q_dtype, int32_t batch, int32_t heads,
                              const v4kv_paged* main_cache, const v4kv_paged* window,
                              const int32_t* seq_lens, int32_t max_seq_len, int32_t ratio,
                              int32_t window_len, const int32_t* topk, int32_t k, float sm_scale,
                              v4kv_rope rope, const void* out);

// Tensor map over `rows` rows of `row_bytes` bytes (uint8, 2-D, 128-byte
// swizzle), boxes of `row_bytes` x `box_rows`. base must be 16-byte aligned.
cudaError_t encode_rows_u8(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes,
                           uint32_t box_rows);

}  // namespace v4kv
