// Decode attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run decode attention: code running inside another framework's memory
// pool, or a host thread that must not take the allocator's lock while it
// serves a request. v4kv_decode_attention needs a caller-provided workspace
// for its split-K partial results; this variant instead uses a fixed scratch
// array that lives in the library's own device memory image.
//
// The scratch is a file-scope __device__ array: every GPU that loads the
// library reserves it (V4KV_NOALLOC_SCRATCH_BYTES) until the process exits.
// In host code its name stands for a host-side shadow, not a device address,
// so its device address is looked up with cudaGetSymbolAddress, once per
// device, the first time this entry point runs on that device.
#include <atomic>

#include <cuda_runtime.h>

#include "../../include/v4kv.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[V4KV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// device address of g_decode_scratch on the current device (looked up once)
v4kv_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return V4KV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return V4KV_ERR_UNSUPPORTED;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return V4KV_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return V4KV_OK;
}

}  // namespace

extern "C" v4kv_status v4kv_decode_attention_noalloc(
    const void* q, int32_t q_dtype, int32_t batch, int32_t heads, const v4kv_paged* main_cache,
    const v4kv_paged* window, const int32_t* seq_lens, int32_t max_seq_len, int32_t ratio,
    int32_t window_len, const int32_t* topk, int32_t k, float sm_scale, v4kv_rope rope, void* out,
    int32_t* dev_status, void* stream) {
  // the same argument checks (and statuses) as v4kv_decode_attention first
  v4kv_status st = v4kv::decode_check_args(q, q_dtype, batch, heads, main_cache, window, seq_lens,
                                           max_seq_len, ratio, window_len, topk, k, sm_scale,
                                           rope, out);
  if (st != V4KV_OK) return st;
  size_t need = 0;
  st = v4kv_workspace_size(V4KV_OP_DECODE, batch, heads, max_seq_len, ratio, window_len,
                           topk ? k : 0, main_cache->dtype, 512, &need);
  if (st != V4KV_OK) return st;
  if (need > (size_t)V4KV_NOALLOC_SCRATCH_BYTES) return V4KV_ERR_INVALID_ARG;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != V4KV_OK) return st;
  return v4kv_decode_attention(q, q_dtype, batch, heads, main_cache, window, seq_lens, max_seq_len,
                               ratio, window_len, topk, k, sm_scale, rope, out, scratch,
                               (size_t)V4KV_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
