// Compressor append: softmax-gated group sums -> RoPE -> fp8/bf16 entry,
// raw-token window copy, and the rolling state of the unfinished group.
// (P1 §2.1 c4a / c128a compression, §2.3 window, §3.1.2 compressor state,
//  §3.2.1 compressor + RoPE + cache-insert fusion.)
#include "common.cuh"
#include "kernels.h"

namespace v4kv {

constexpr int kMaxRatio = 128;

struct Vec8 {
  float v[8];
};

// 8 consecutive bf16 elements (16 bytes) -> fp32
__device__ __forceinline__ Vec8 load_bf16x8(const uint16_t* p) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  Vec8 r;
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.v[2 * i] = __uint_as_float(w[i] << 16);
    r.v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
  return r;
}

__device__ __forceinline__ void store_bf16x8(uint16_t* p, const Vec8& x) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = (uint32_t)float_to_bf16_bits(x.v[2 * i]) |
           ((uint32_t)float_to_bf16_bits(x.v[2 * i + 1]) << 16);
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// rotate the pairs of this thread's 8 dims [d0, d0+8) that fall in the rope range
__device__ __forceinline__ void rope8(Vec8& x, int d0, const RopeArgs& rp, long long pos,
                                      bool inverse) {
  if (rp.rope_dim == 0) return;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int d = d0 + 2 * k;
    if (d >= rp.rope_offset && d + 1 < rp.rope_offset + rp.rope_dim) {
      float c, s;
      rope_cs(rp, (d - rp.rope_offset) >> 1, pos, &c, &s);
      if (inverse) s = -s;
      rope_apply(x.v[2 * k], x.v[2 * k + 1], c, s);
    }
  }
}

// quantise (fp8) or round (bf16) one vector spread over the block, 8 dims per
// thread, and store it in `slot` of the pool. `active` marks threads owning dims.
__device__ __forceinline__ void store_entry(const PoolArgs& pool, long long slot, int d0,
                                            bool active, Vec8 e, float* red) {
  if (pool.dtype == V4KV_FP8_E4M3) {
    float m = 0.f;
    if (active)
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(e.v[i]));
    float amax = block_reduce<true>(m, red);
    float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, kE4m3Max);
    if (active) {
      uint16_t c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        c[i] = float2_to_e4m3x2(__fdiv_rn(e.v[2 * i], scale), __fdiv_rn(e.v[2 * i + 1], scale));
      uint2 w = make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16),
                           (uint32_t)c[2] | ((uint32_t)c[3] << 16));
      uint8_t* dst = reinterpret_cast<uint8_t*>(pool.data) + slot * pool.dim + d0;
      *reinterpret_cast<uint2*>(dst) = w;
    }
    if (threadIdx.x == 0) pool.scales[slot] = scale;
  } else {
    if (active) {
      uint16_t* dst = reinterpret_cast<uint16_t*>(pool.data) + slot * pool.dim + d0;
      store_bf16x8(dst, e);
    }
  }
}

__device__ __forceinline__ int find_seq(const int32_t* cu, int batch, int i) {
  int lo = 0, hi = batch - 1;  // largest b with cu[b] <= i
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= i)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// one block per touched group
constexpr int kCuSmem = 1024;  // sequences whose prefix sums fit in shared memory

// largest b with cu[b] <= i, from a shared-memory copy of cu[0..batch] when it fits
__device__ __forceinline__ int find_seq_cached(const int32_t* cu, int batch, int i, int* cu_sh) {
  if (batch + 1 > kCuSmem) return find_seq(cu, batch, i);
  for (int k = threadIdx.x; k <= batch; k += blockDim.x) cu_sh[k] = cu[k];
  __syncthreads();
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu_sh[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void compress_entries_kernel(CompressArgs a) {
  __shared__ float w[kMaxRatio];
  __shared__ float red[32];
  __shared__ int cu_sh[kCuSmem];
  const int i = blockIdx.x;
  const int total = a.cu_entries[a.batch];
  if (i >= total) return;
  const int b = find_seq_cached(a.cu_entries, a.batch, i, cu_sh);
  const int r = a.ratio;
  const int s = a.seq_start[b];
  const int n = a.cu_seqlens[b + 1] - a.cu_seqlens[b];
  const int end = s + n;
  const int g = s / r + (i - a.cu_entries[b]);
  const int t0 = g * r;
  const int t1 = min(t0 + r, end);
  const int np = t1 - t0;
  const int dim = a.dim;
  const int d0 = threadIdx.x * 8;
  const bool active = d0 < dim;

  auto gate_of = [&](int t) -> float {
    return t < s ? a.state_gate[(size_t)b * r + (t - t0)] : a.gate[a.cu_seqlens[b] + (t - s)];
  };
  auto row_of = [&](int t) -> const uint16_t* {
    return t < s ? a.state_x + ((size_t)b * r + (t - t0)) * dim
                 : a.x + (size_t)(a.cu_seqlens[b] + (t - s)) * dim;
  };

  // softmax over the group's present tokens of gate + position bias
  float m = -INFINITY;
  for (int t = threadIdx.x; t < np; t += blockDim.x) {
    float z = gate_of(t0 + t) + a.pos_bias[t];
    w[t] = z;
    m = fmaxf(m, z);
  }
  m = block_reduce<true>(m, red);
  for (int t = threadIdx.x; t < np; t += blockDim.x) w[t] = expf(w[t] - m);
  __syncthreads();
  if (threadIdx.x == 0) {
    float sum = 0.f;
    for (int t = 0; t < np; ++t) sum += w[t];
    red[0] = sum;
  }
  __syncthreads();
  const float sum = red[0];
  __syncthreads();
  for (int t = threadIdx.x; t < np; t += blockDim.x) w[t] = __fdiv_rn(w[t], sum);
  __syncthreads();

  // weighted sum in ascending token order
  Vec8 e;
#pragma unroll
  for (int k = 0; k < 8; ++k) e.v[k] = 0.f;
  if (active) {
    for (int t = 0; t < np; ++t) {
      Vec8 x = load_bf16x8(row_of(t0 + t) + d0);
      const float wt = w[t];
#pragma unroll
      for (int k = 0; k < 8; ++k) e.v[k] = fmaf(wt, x.v[k], e.v[k]);
    }
    rope8(e, d0, a.rope, (long long)t0, false);
    if (a.prequant_out) {
      float* po = a.prequant_out + (size_t)i * dim + d0;
      *reinterpret_cast<float4*>(po) = make_float4(e.v[0], e.v[1], e.v[2], e.v[3]);
      *reinterpret_cast<float4*>(po + 4) = make_float4(e.v[4], e.v[5], e.v[6], e.v[7]);
    }
  }
  long long slot = a.slot_mapping[i];
  const long long cap = (long long)a.main.num_pages * a.main.spb;
  if (slot < 0) return;  // unmapped page (already flagged by the slot mapping)
  if (slot >= cap) {
    if (threadIdx.x == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    return;
  }
  store_entry(a.main, slot, d0, active, e, red);
}

// one block per input token; the last W tokens of each sequence's new ones
// ([max(s, end - W), end)) are written to the window
__global__ void compress_window_kernel(CompressArgs a) {
  __shared__ float red[32];
  __shared__ int cu_sh[kCuSmem];
  const int g = blockIdx.x;
  if (g >= a.cu_seqlens[a.batch]) return;
  const int b = find_seq_cached(a.cu_seqlens, a.batch, g, cu_sh);
  const int s = a.seq_start[b];
  const int n = a.cu_seqlens[b + 1] - a.cu_seqlens[b];
  const int end = s + n;
  const int first = max(s, end - a.window_len);
  const int t = s + (g - a.cu_seqlens[b]);
  if (t < first || t >= end) return;
  const int dim = a.dim;
  const int d0 = threadIdx.x * 8;
  const bool active = d0 < dim;
  const int32_t* row = a.window.block_table + (size_t)b * a.window.max_blocks;
  const int blk = t / kLogicalBlock;
  if (blk >= a.window.max_blocks) {
    if (threadIdx.x == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    return;
  }
  const int p = row[blk];
  if (p < 0) return;  // no page for this block: nothing to keep
  if (p >= a.window.num_pages) {
    if (threadIdx.x == 0) flag(a.dev_status, V4KV_DEV_BAD_PAGE);
    return;
  }
  Vec8 x;
#pragma unroll
  for (int k = 0; k < 8; ++k) x.v[k] = 0.f;
  if (active) {
    x = load_bf16x8(a.x + (size_t)(a.cu_seqlens[b] + (t - s)) * dim + d0);
    rope8(x, d0, a.rope, (long long)t, false);
  }
  const long long slot = (long long)p * kLogicalBlock + (t % kLogicalBlock);
  store_entry(a.window, slot, d0, active, x, red);
}

// after the entries kernel: keep tokens [floor(end/r)*r, end) as state rows
__global__ void compress_state_kernel(CompressArgs a) {
  const int b = blockIdx.x;
  const int r = a.ratio;
  const int s = a.seq_start[b];
  const int n = a.cu_seqlens[b + 1] - a.cu_seqlens[b];
  if (n <= 0) return;
  const int end = s + n;
  const int gs = (end / r) * r;
  const int rows = end - gs;
  const int chunks = a.dim / 8;
  for (int q = threadIdx.x; q < rows * chunks; q += blockDim.x) {
    const int i = q / chunks, c = q % chunks;
    const int t = gs + i;
    if (t < s) continue;  // already in the state from an earlier call
    const uint16_t* src = a.x + (size_t)(a.cu_seqlens[b] + (t - s)) * a.dim + c * 8;
    uint16_t* dst = a.state_x_out + ((size_t)b * r + i) * a.dim + c * 8;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    if (c == 0) a.state_gate_out[(size_t)b * r + i] = a.gate[a.cu_seqlens[b] + (t - s)];
  }
}

cudaError_t launch_compress_append(const CompressArgs& a, int max_groups, int total_tokens,
                                   cudaStream_t stream) {
  const int threads = ((a.dim / 8 + 31) / 32) * 32;
  if (max_groups > 0) compress_entries_kernel<<<max_groups, threads, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (a.window.data && a.window_len > 0 && total_tokens > 0) {
    compress_window_kernel<<<total_tokens, threads, 0, stream>>>(a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  compress_state_kernel<<<a.batch, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace v4kv
