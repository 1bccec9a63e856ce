// C ABI of the v4kv library: argument checks on the host, then launches on
// the caller's stream. Nothing here allocates, frees or synchronises.
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/v4kv.h"
#include "kernels.h"

namespace {

using namespace v4kv;

constexpr int kVersion = 1;
constexpr int kBlock = 256;  // raw tokens per logical block (P1 §3.1.1)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device must be sm_100 (B200). Cached per device ordinal.
v4kv_status check_device(int* num_sms) {
  static int cached_major[64];
  static int cached_sms[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return V4KV_ERR_CUDA;
  if (dev < 0 || dev >= 64) return V4KV_ERR_UNSUPPORTED;
  if (cached_major[dev] == 0) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return V4KV_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return V4KV_ERR_CUDA;
    cached_sms[dev] = sms;
    cached_major[dev] = major;
  }
  if (cached_major[dev] != 10) return V4KV_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = cached_sms[dev];
  return V4KV_OK;
}

v4kv_status to_status(cudaError_t e) { return e == cudaSuccess ? V4KV_OK : V4KV_ERR_CUDA; }

// checks common to every pool; spb must equal `want_spb`
bool pool_ok(const v4kv_paged* p, int want_spb, int want_dim, bool allow_bf16, bool allow_fp8,
             bool allow_fp4 = false) {
  if (!p || !p->data || !p->block_table) return false;
  if (!aligned16(p->data)) return false;
  if (p->num_pages <= 0 || p->max_blocks <= 0) return false;
  if (p->slots_per_page != want_spb) return false;
  if (want_dim > 0 && p->dim != want_dim) return false;
  if (p->dtype == V4KV_FP8_E4M3) {
    if (!allow_fp8 || !p->scales) return false;
  } else if (p->dtype == V4KV_FP4_E2M1) {
    if (!allow_fp4 || !p->scales) return false;
  } else if (p->dtype == V4KV_BF16) {
    if (!allow_bf16) return false;
  } else {
    return false;
  }
  return true;
}

PoolArgs to_args(const v4kv_paged* p) {
  PoolArgs a{};
  if (!p) return a;
  a.data = p->data;
  a.scales = p->scales;
  a.block_table = p->block_table;
  a.num_pages = p->num_pages;
  a.spb = p->slots_per_page;
  a.dim = p->dim;
  a.dtype = p->dtype;
  a.max_blocks = p->max_blocks;
  return a;
}

bool rope_ok(const v4kv_rope& r, int dim) {
  if (r.rope_dim == 0) return true;
  if (r.rope_dim < 0 || (r.rope_dim & 1) || (r.rope_offset & 1) || r.rope_offset < 0) return false;
  if (r.rope_offset + r.rope_dim > dim) return false;
  return r.theta > 0.0 && isfinite(r.theta);
}

RopeArgs to_rope(const v4kv_rope& r) {
  RopeArgs a{};
  a.theta = r.theta;
  a.rope_dim = r.rope_dim;
  a.rope_offset = r.rope_offset;
  for (int i = 0; i < kRopeTable && 2 * i < r.rope_dim; ++i)
    a.freq[i] = std::pow(r.theta, -2.0 * (double)i / (double)r.rope_dim);
  return a;
}

}  // namespace

extern "C" {

const char* v4kv_status_string(v4kv_status s) {
  switch (s) {
    case V4KV_OK: return "ok";
    case V4KV_ERR_INVALID_ARG: return "invalid argument";
    case V4KV_ERR_UNSUPPORTED: return "unsupported shape or device";
    case V4KV_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int32_t v4kv_version(void) { return kVersion; }

v4kv_status v4kv_slot_mapping(const int32_t* block_table, int32_t max_blocks, int32_t batch,
                              const int32_t* seq_start, const int32_t* n_new, int32_t ratio,
                              int32_t slots_per_page, int32_t num_pages, int32_t* cu_out,
                              int64_t* slot_out, int64_t slot_capacity, int32_t* dev_status,
                              void* stream) {
  if (!block_table || !seq_start || !n_new || (!slot_out && slot_capacity > 0)) return V4KV_ERR_INVALID_ARG;
  if (batch <= 0 || max_blocks <= 0 || num_pages <= 0 || slot_capacity < 0) return V4KV_ERR_INVALID_ARG;
  if (ratio <= 0 || ratio > kBlock || kBlock % ratio) return V4KV_ERR_INVALID_ARG;
  if (slots_per_page != kBlock / ratio) return V4KV_ERR_INVALID_ARG;
  v4kv_status st = check_device(nullptr);
  if (st != V4KV_OK) return st;
  return to_status(launch_slot_mapping(block_table, max_blocks, batch, seq_start, n_new, ratio,
                                       slots_per_page, num_pages, cu_out, slot_out, slot_capacity,
                                       dev_status, (cudaStream_t)stream));
}

v4kv_status v4kv_compress_append(const void* x, const float* gate, const int32_t* cu_seqlens,
                                 const int32_t* seq_start, int32_t batch, int32_t total_tokens,
                                 const float* pos_bias, int32_t ratio, v4kv_rope rope,
                                 void* state_x, float* state_gate, const v4kv_paged* main_cache,
                                 const int64_t* slot_mapping, const int32_t* cu_entries,
                                 const v4kv_paged* window, int32_t window_len,
                                 float* prequant_out, int32_t* dev_status, void* stream) {
  return v4kv_compress_append_ex(x, gate, cu_seqlens, seq_start, batch, total_tokens, pos_bias,
                                 ratio, rope, state_x, state_gate, main_cache, slot_mapping,
                                 cu_entries, window, window_len, prequant_out, nullptr, dev_status,
                                 stream);
}

v4kv_status v4kv_compress_append_ex(const void* x, const float* gate, const int32_t* cu_seqlens,
                                    const int32_t* seq_start, int32_t batch, int32_t total_tokens,
                                    const float* pos_bias, int32_t ratio, v4kv_rope rope,
                                    void* state_x, float* state_gate, const v4kv_paged* main_cache,
                                    const int64_t* slot_mapping, const int32_t* cu_entries,
                                    const v4kv_paged* window, int32_t window_len,
                                    float* prequant_out, const v4kv_compress_opts* opts,
                                    int32_t* dev_status, void* stream) {
  if (batch <= 0 || total_tokens < 0) return V4KV_ERR_INVALID_ARG;
  if (ratio != 4 && ratio != 128) return V4KV_ERR_INVALID_ARG;
  const int overlap = opts ? opts->overlap : 0;
  const int per_channel = opts ? opts->gate_per_channel : 0;
  const float* norm_w = opts ? opts->norm_weight : nullptr;
  if ((overlap != 0 && overlap != 1) || (per_channel != 0 && per_channel != 1)) return V4KV_ERR_INVALID_ARG;
  if (overlap && ratio != 4) return V4KV_ERR_UNSUPPORTED;  // the overlapping window is c4a's
  if (norm_w && (!aligned16(norm_w) || !(opts->norm_eps >= 0.f))) return V4KV_ERR_INVALID_ARG;
  if (per_channel && ((gate && !aligned16(gate)) || !aligned16(state_gate))) return V4KV_ERR_INVALID_ARG;
  if (!cu_seqlens || !seq_start || !pos_bias || !state_x || !state_gate) return V4KV_ERR_INVALID_ARG;
  // the slot mapping comes from v4kv_slot_mapping, or (both NULL) is computed
  // inside the kernel from main_cache's block table, for batch < 1024
  if (!slot_mapping != !cu_entries) return V4KV_ERR_INVALID_ARG;
  if (!slot_mapping && batch >= 1024) return V4KV_ERR_UNSUPPORTED;
  if (total_tokens > 0 && (!x || !gate)) return V4KV_ERR_INVALID_ARG;
  if (!main_cache) return V4KV_ERR_INVALID_ARG;
  const int dim = main_cache->dim;
  if (dim < 8 || dim > 1024 || dim % 8) return V4KV_ERR_INVALID_ARG;
  if (!pool_ok(main_cache, kBlock / ratio, dim, true, true)) return V4KV_ERR_INVALID_ARG;
  if (window && !pool_ok(window, kBlock, dim, true, true)) return V4KV_ERR_INVALID_ARG;
  if (window_len < 0) return V4KV_ERR_INVALID_ARG;
  if (!rope_ok(rope, dim)) return V4KV_ERR_INVALID_ARG;
  if ((x && !aligned16(x)) || !aligned16(state_x) || (prequant_out && !aligned16(prequant_out)))
    return V4KV_ERR_INVALID_ARG;
  int sms = 0;
  v4kv_status st = check_device(&sms);
  if (st != V4KV_OK) return st;
  CompressArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.gate = gate;
  a.cu_seqlens = cu_seqlens;
  a.seq_start = seq_start;
  a.pos_bias = pos_bias;
  a.state_x = static_cast<const uint16_t*>(state_x);
  a.state_gate = state_gate;
  a.state_x_out = static_cast<uint16_t*>(state_x);
  a.state_gate_out = state_gate;
  a.slot_mapping = slot_mapping;
  a.cu_entries = cu_entries;
  a.prequant_out = prequant_out;
  a.dev_status = dev_status;
  a.main = to_args(main_cache);
  a.window = to_args(window);
  a.rope = to_rope(rope);
  a.batch = batch;
  a.ratio = ratio;
  a.dim = dim;
  a.window_len = window ? window_len : 0;
  a.overlap = overlap;
  a.gate_dim = per_channel ? dim : 1;
  a.state_rows = overlap ? 2 * ratio : ratio;
  a.norm_w = norm_w;
  a.norm_eps = norm_w ? (opts->norm_eps > 0.f ? opts->norm_eps : 1e-6f) : 0.f;
  // every sequence touches at most ceil(n/r) + 1 groups
  const long long max_groups = (long long)total_tokens / ratio + 2LL * batch;
  if (max_groups > 0x7fffffffLL) return V4KV_ERR_INVALID_ARG;
  return to_status(launch_compress_append(a, (int)max_groups, total_tokens, (cudaStream_t)stream));
}

v4kv_status v4kv_qk_prepare(const float* q_in, int32_t batch, int32_t heads, int32_t dim,
                            const float* q_norm_weight, float q_norm_eps, const int32_t* positions,
                            v4kv_rope rope, void* q_out, int32_t q_out_dtype, const void* k_new,
                            const v4kv_paged* window, int32_t* dev_status, void* stream) {
  if (batch <= 0 || heads <= 0 || !q_in || !q_out || !positions) return V4KV_ERR_INVALID_ARG;
  if (dim < 8 || dim > 1024 || dim % 8) return V4KV_ERR_INVALID_ARG;
  if (q_out_dtype != V4KV_FP32 && q_out_dtype != V4KV_BF16) return V4KV_ERR_INVALID_ARG;
  if (!aligned16(q_in) || !aligned16(q_out) || (q_norm_weight && !aligned16(q_norm_weight)))
    return V4KV_ERR_INVALID_ARG;
  if (q_norm_weight && !(q_norm_eps >= 0.f)) return V4KV_ERR_INVALID_ARG;
  if (k_new && !aligned16(k_new)) return V4KV_ERR_INVALID_ARG;
  if (window && !pool_ok(window, kBlock, dim, true, true)) return V4KV_ERR_INVALID_ARG;
  if (!rope_ok(rope, dim)) return V4KV_ERR_INVALID_ARG;
  if ((long long)heads + 1 > 65535LL * 8) return V4KV_ERR_INVALID_ARG;
  v4kv_status st = check_device(nullptr);
  if (st != V4KV_OK) return st;
  QkPrepArgs p{};
  p.q_in = q_in;
  p.q_out = q_out;
  p.q_out_bf16 = q_out_dtype == V4KV_BF16;
  p.norm_w = q_norm_weight;
  p.norm_eps = q_norm_weight ? (q_norm_eps > 0.f ? q_norm_eps : 1e-6f) : 0.f;
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.positions = positions;
  p.window = to_args(window);
  p.rope = to_rope(rope);
  p.dev_status = dev_status;
  p.batch = batch;
  p.heads = heads;
  p.dim = dim;
  return to_status(launch_qk_prepare(p, (cudaStream_t)stream));
}

v4kv_status v4kv_index_topk(const float* q_idx, const v4kv_paged* idx_cache,
                            const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                            int32_t ratio, int32_t window_len, int32_t k, int32_t* topk_out,
                            float* score_out, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream) {
  if (!q_idx || !seq_lens || !topk_out || batch <= 0 || max_seq_len < 0 || window_len < 0)
    return V4KV_ERR_INVALID_ARG;
  if (ratio != 4 && ratio != 128) return V4KV_ERR_INVALID_ARG;
  if (k < 1 || k > 2048) return V4KV_ERR_INVALID_ARG;
  if (!pool_ok(idx_cache, kBlock / ratio, 0, false, true, true)) return V4KV_ERR_INVALID_ARG;
  if (idx_cache->dim < 16 || idx_cache->dim > 512 || idx_cache->dim % 16) return V4KV_ERR_UNSUPPORTED;
  if (idx_cache->dtype == V4KV_FP4_E2M1 && idx_cache->dim % 32) return V4KV_ERR_UNSUPPORTED;
  const size_t need = index_workspace_bytes(batch, max_seq_len, ratio, window_len);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return V4KV_ERR_INVALID_ARG;
  v4kv_status st = check_device(nullptr);
  if (st != V4KV_OK) return st;
  IndexArgs a{};
  a.q_idx = q_idx;
  a.seq_lens = seq_lens;
  a.topk_out = topk_out;
  a.score_out = score_out;
  a.scores_ws = static_cast<float*>(workspace);
  a.dev_status = dev_status;
  a.cache = to_args(idx_cache);
  a.batch = batch;
  a.ratio = ratio;
  a.window_len = window_len;
  a.k = k;
  return to_status(launch_index_topk(a, max_seq_len, (cudaStream_t)stream));
}

v4kv_status v4kv_workspace_size(int32_t op, int32_t batch, int32_t heads, int32_t max_seq_len,
                                int32_t ratio, int32_t window_len, int32_t k, int32_t main_dtype,
                                int32_t dim, size_t* bytes) {
  if (!bytes || batch <= 0 || max_seq_len < 0 || window_len < 0) return V4KV_ERR_INVALID_ARG;
  if (ratio != 4 && ratio != 128) return V4KV_ERR_INVALID_ARG;
  if (op == V4KV_OP_INDEX_TOPK) {
    *bytes = index_workspace_bytes(batch, max_seq_len, ratio, window_len);
    return V4KV_OK;
  }
  if (op != V4KV_OP_DECODE) return V4KV_ERR_INVALID_ARG;
  if (heads < 1 || heads > 128 || k < 0) return V4KV_ERR_INVALID_ARG;
  int sms = 0;
  v4kv_status st = check_device(&sms);
  if (st != V4KV_OK) return st;
  *bytes = plan_decode(batch, heads, max_seq_len, ratio, window_len, k, main_dtype, dim, sms).ws_bytes;
  return V4KV_OK;
}

}  // extern "C"

namespace v4kv {

// Host-side argument checks of decode attention (everything but the
// workspace), shared by both decode entry points so that they report the
// same status for the same bad argument.
v4kv_status decode_check_args(const void* q, int32_t q_dtype, int32_t batch, int32_t heads,
                              const v4kv_paged* main_cache, const v4kv_paged* window,
                              const int32_t* seq_lens, int32_t max_seq_len, int32_t ratio,
                              int32_t window_len, const int32_t* topk, int32_t k, float sm_scale,
                              v4kv_rope rope, const void* out) {
  if (!q || !seq_lens || !out || batch <= 0 || max_seq_len < 0 || window_len < 0)
    return V4KV_ERR_INVALID_ARG;
  if (q_dtype != V4KV_FP32 && q_dtype != V4KV_BF16) return V4KV_ERR_INVALID_ARG;
  if (heads < 1 || heads > 128) return V4KV_ERR_UNSUPPORTED;
  if (ratio != 4 && ratio != 128) return V4KV_ERR_INVALID_ARG;
  if (topk && (k < 1 || k > 2048)) return V4KV_ERR_INVALID_ARG;
  if (!main_cache || !window) return V4KV_ERR_INVALID_ARG;
  if (main_cache->dim != 512 || window->dim != 512) return V4KV_ERR_UNSUPPORTED;
  if (!pool_ok(main_cache, kBlock / ratio, 512, true, true)) return V4KV_ERR_INVALID_ARG;
  if (!pool_ok(window, kBlock, 512, true, true)) return V4KV_ERR_INVALID_ARG;
  if (!rope_ok(rope, 512)) return V4KV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return V4KV_ERR_INVALID_ARG;
  if (sm_scale != 0.f && (!(sm_scale > 0.f) || !isfinite(sm_scale))) return V4KV_ERR_INVALID_ARG;
  return check_device(nullptr);
}

}  // namespace v4kv

namespace {

// decode attention with the output in bf16 (out_fp8 == 0) or as e4m3 codes
// with one scale per (sequence, head) (out_fp8 == 1)
v4kv_status decode_impl(const void* q, int32_t q_dtype, int32_t batch, int32_t heads,
                        const v4kv_paged* main_cache, const v4kv_paged* window,
                        const int32_t* seq_lens, int32_t max_seq_len, int32_t ratio,
                        int32_t window_len, const int32_t* topk, int32_t k, float sm_scale,
                        v4kv_rope rope, void* out, int out_fp8, float* out_scales,
                        float* prequant_out, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream) {
  v4kv_status st = decode_check_args(q, q_dtype, batch, heads, main_cache, window, seq_lens,
                                     max_seq_len, ratio, window_len, topk, k, sm_scale, rope, out);
  if (st != V4KV_OK) return st;
  if (out_fp8 && (!out_scales || (prequant_out && !aligned16(prequant_out))))
    return V4KV_ERR_INVALID_ARG;
  if (!topk) k = 0;
  if (sm_scale == 0.f) sm_scale = 1.f / sqrtf(512.f);  // the default scale 1/sqrt(dim)
  int sms = 0;
  st = check_device(&sms);
  if (st != V4KV_OK) return st;
  const DecodePlan plan =
      plan_decode(batch, heads, max_seq_len, ratio, window_len, k, main_cache->dtype, 512, sms);
  if (!workspace || workspace_bytes < plan.ws_bytes ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return V4KV_ERR_INVALID_ARG;
  DecodeArgs a{};
  a.q = q;
  a.seq_lens = seq_lens;
  a.topk = topk;
  a.out = out;
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = a.part_o + (size_t)batch * plan.n_splits * heads * 512;
  a.dev_status = dev_status;
  a.main = to_args(main_cache);
  a.window = to_args(window);
  a.rope = to_rope(rope);
  a.q_dtype = q_dtype;
  a.batch = batch;
  a.heads = heads;
  a.dim = 512;
  a.ratio = ratio;
  a.window_len = window_len;
  a.k = k;
  a.sm_scale = sm_scale;
  a.split = plan.split;
  a.n_splits = plan.n_splits;
  a.max_len = max_seq_len;
  a.pad_sel = plan.path == 1;
  a.out_fp8 = out_fp8;
  a.out_scales = out_scales;
  a.prequant_out = out_fp8 ? prequant_out : nullptr;
  if (plan.path == 1) {
    decode_tc_layout(a, workspace);
    return to_status(launch_decode_tc(a, (cudaStream_t)stream));
  }
  cudaError_t e = launch_decode_simt(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return V4KV_ERR_CUDA;
  return to_status(launch_decode_merge(a, (cudaStream_t)stream));
}

}  // namespace

extern "C" {

v4kv_status v4kv_decode_attention(const void* q, int32_t q_dtype, int32_t batch, int32_t heads,
                                  const v4kv_paged* main_cache, const v4kv_paged* window,
                                  const int32_t* seq_lens, int32_t max_seq_len, int32_t ratio,
                                  int32_t window_len, const int32_t* topk, int32_t k,
                                  float sm_scale, v4kv_rope rope, void* out, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return decode_impl(q, q_dtype, batch, heads, main_cache, window, seq_lens, max_seq_len, ratio,
                     window_len, topk, k, sm_scale, rope, out, 0, nullptr, nullptr, workspace,
                     workspace_bytes, dev_status, stream);
}

v4kv_status v4kv_decode_attention_fp8out(const void* q, int32_t q_dtype, int32_t batch,
                                         int32_t heads, const v4kv_paged* main_cache,
                                         const v4kv_paged* window, const int32_t* seq_lens,
                                         int32_t max_seq_len, int32_t ratio, int32_t window_len,
                                         const int32_t* topk, int32_t k, float sm_scale,
                                         v4kv_rope rope, void* out_codes, float* out_scales,
                                         float* prequant_out, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_status,
                                         void* stream) {
  return decode_impl(q, q_dtype, batch, heads, main_cache, window, seq_lens, max_seq_len, ratio,
                     window_len, topk, k, sm_scale, rope, out_codes, 1, out_scales, prequant_out,
                     workspace, workspace_bytes, dev_status, stream);
}

uint64_t v4kv_kv_footprint_bytes(uint64_t n_tokens, const v4kv_footprint_cfg* c) {
  if (!c || !c->layer_ratios || c->n_layers <= 0) return 0;
  // element sizes are in bits; accumulate in bits, round up to bytes per term
  uint64_t total = 0;
  for (int i = 0; i < c->n_layers; ++i) {
    const uint64_t r = (uint64_t)c->layer_ratios[i];
    if (r == 0) return 0;
    const uint64_t entries = (n_tokens + r - 1) / r;
    total += entries * (((uint64_t)c->dim * c->entry_bits + 7) / 8 + (uint64_t)c->entry_scale_bytes);
    if (r == 4 && c->indexer_dim > 0)
      total += entries * (((uint64_t)c->indexer_dim * c->indexer_bits + 7) / 8 +
                          (uint64_t)c->indexer_scale_bytes);
    const uint64_t w = n_tokens < (uint64_t)c->window ? n_tokens : (uint64_t)c->window;
    total += w * (((uint64_t)c->dim * c->window_bits + 7) / 8);
  }
  return total;
}

}  // extern "C"
