// Indexer scores over c4a entries and exact top-k (P1 §2.2 indexer cache;
// P1 §4.1 sparse attention over the selected c4a entries).
//
// Score of entry j: fp32 fused multiply-add chain over d = 0..dim-1 of
// q8[d] * k8_j[d] (q8 = the query quantised per vector to fp8), times the
// entry's fp32 scale. Ranking: score descending, index ascending, -0 == +0.
#include "common.cuh"
#include "kernels.h"

namespace v4kv {

constexpr int kIdxMaxDim = 512;
constexpr int kScoreThreads = 256;
constexpr int kSelectThreads = 1024;
constexpr int kMaxK = 2048;

__host__ __device__ __forceinline__ int visible(int L, int W, int r) { return max(0, L - W) / r; }

// sequence length, clamped to the host bound the workspace was sized for
__device__ __forceinline__ int seq_len_of(const IndexArgs& a, int b) {
  int L = a.seq_lens[b];
  if (L > a.max_len) {
    if (threadIdx.x == 0) flag(a.dev_status, V4KV_DEV_OVERFLOW);
    L = a.max_len;
  }
  return max(0, L);
}

// quantise q_idx[b] like an entry and leave its fp8 values (as fp32) in qs_f
__device__ void quantise_query(const float* q, int dim, float* q_f, float* red, float* qscale) {
  float m = 0.f;
  for (int d = threadIdx.x; d < dim; d += blockDim.x) m = fmaxf(m, fabsf(q[d]));
  const float amax = block_reduce<true>(m, red);
  const float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, kE4m3Max);
  for (int d = threadIdx.x; d < dim; d += blockDim.x) {
    uint16_t c = float2_to_e4m3x2(__fdiv_rn(q[d], scale), 0.f);
    q_f[d] = e4m3_to_float((uint8_t)(c & 0xff));
  }
  if (qscale && threadIdx.x == 0) *qscale = scale;
  __syncthreads();
}

// grid (chunks, batch): each thread scores one entry at a time
__global__ void __launch_bounds__(kScoreThreads) index_score_kernel(IndexArgs a) {
  __shared__ __align__(16) float q_f[kIdxMaxDim];
  __shared__ float red[32];
  const int b = blockIdx.y;
  const int L = seq_len_of(a, b);
  const int n_vis = visible(L, a.window_len, a.ratio);
  const int j0 = blockIdx.x * a.chunk;
  if (j0 >= n_vis) return;
  const int dim = a.cache.dim;
  quantise_query(a.q_idx + (size_t)b * dim, dim, q_f, red, nullptr);
  const int j1 = min(n_vis, j0 + a.chunk);
  const int32_t* bt = a.cache.block_table + (size_t)b * a.cache.max_blocks;
  const uint8_t* base = reinterpret_cast<const uint8_t*>(a.cache.data);
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
    const int p = page_of(bt, a.cache.max_blocks, j, a.cache.spb, a.cache.num_pages, a.dev_status);
    float score = 0.f;
    if (p >= 0) {
      const long long slot = (long long)p * a.cache.spb + (j % a.cache.spb);
      const uint8_t* key = base + slot * dim;
      float acc = 0.f;
      for (int d = 0; d < dim; d += 16) {
        const uint4 raw = *reinterpret_cast<const uint4*>(key + d);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 lo = __half22float2(e4m3x2_to_half2((uint16_t)(w[i] & 0xffff)));
          const float2 hi = __half22float2(e4m3x2_to_half2((uint16_t)(w[i] >> 16)));
          acc = fmaf(q_f[d + 4 * i + 0], lo.x, acc);
          acc = fmaf(q_f[d + 4 * i + 1], lo.y, acc);
          acc = fmaf(q_f[d + 4 * i + 2], hi.x, acc);
          acc = fmaf(q_f[d + 4 * i + 3], hi.y, acc);
        }
      }
      score = __fmul_rn(acc, a.cache.scales[slot]);
    }
    a.scores_ws[(size_t)b * a.ws_stride + j] = score;
  }
}

// order-preserving map of fp32 onto uint32 (larger float -> larger key)
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.f) u = 0u;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < (int)(blockDim.x >> 5) ? sh[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    sh[lane] = t;  // inclusive prefix over warps
  }
  __syncthreads();
  const uint32_t before = (warp ? sh[warp - 1] : 0u) + x - v;
  *total = sh[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// one block per sequence: radix select of the k-th largest key, collect, sort
__global__ void __launch_bounds__(kSelectThreads) index_select_kernel(IndexArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t scan_sh[32];
  __shared__ unsigned long long sel[kMaxK];
  __shared__ float red[32];
  __shared__ float q_f[kIdxMaxDim];
  __shared__ float qs_sh;
  __shared__ uint32_t n_sel_sh;
  __shared__ uint32_t pick_sh[2];

  const int b = blockIdx.x;
  const int L = seq_len_of(a, b);
  const int n = visible(L, a.window_len, a.ratio);
  const int k = a.k;
  const float* sc = a.scores_ws + (size_t)b * a.ws_stride;
  quantise_query(a.q_idx + (size_t)b * a.cache.dim, a.cache.dim, q_f, red, &qs_sh);

  int kpow = 1;
  while (kpow < k) kpow <<= 1;
  for (int i = threadIdx.x; i < kpow; i += blockDim.x) sel[i] = 0ull;
  if (threadIdx.x == 0) n_sel_sh = 0;
  __syncthreads();

  if (n <= k) {
    for (int j = threadIdx.x; j < n; j += blockDim.x)
      sel[j] = ((unsigned long long)score_key(sc[j]) << 32) | (0xffffffffu - (uint32_t)j);
    __syncthreads();
  } else {
    // radix select, 8 bits per pass from the top: find key T, the k-th largest
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const uint32_t key = score_key(sc[j]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        uint32_t cum = 0, digit = 0;
        for (int d = 255; d >= 0; --d) {
          if (cum + hist[d] >= remaining) {
            digit = (uint32_t)d;
            break;
          }
          cum += hist[d];
        }
        pick_sh[0] = digit;
        pick_sh[1] = remaining - cum;
      }
      __syncthreads();
      prefix |= pick_sh[0] << shift;
      mask |= 255u << shift;
      remaining = pick_sh[1];
      __syncthreads();
    }
    const uint32_t T = prefix;
    // strictly greater keys: any order (sorted below)
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
      const uint32_t key = score_key(sc[j]);
      if (key > T) {
        const uint32_t pos = atomicAdd(&n_sel_sh, 1u);
        sel[pos] = ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)j);
      }
    }
    __syncthreads();
    // ties at T: the `remaining` lowest indices, found in ascending index order
    uint32_t taken = 0;
    const uint32_t base_pos = n_sel_sh;
    for (int j0 = 0; j0 < n && taken < remaining; j0 += blockDim.x) {
      const int j = j0 + threadIdx.x;
      const uint32_t is_tie = (j < n && score_key(sc[j]) == T) ? 1u : 0u;
      uint32_t total;
      const uint32_t before = block_exclusive_scan(is_tie, scan_sh, &total);
      if (is_tie && taken + before < remaining)
        sel[base_pos + taken + before] = ((unsigned long long)T << 32) | (0xffffffffu - (uint32_t)j);
      taken += total;
    }
    __syncthreads();
  }

  // bitonic sort of sel[0 .. kpow) descending (score desc, then index asc)
  for (int size = 2; size <= kpow; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < kpow; i += blockDim.x) {
        const int jx = i ^ stride;
        if (jx > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long x = sel[i], y = sel[jx];
          if (desc ? (x < y) : (x > y)) {
            sel[i] = y;
            sel[jx] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  const int valid = min(n, k);
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    int32_t idx = -1;
    float s = 0.f;
    if (i < valid) {
      idx = (int32_t)(0xffffffffu - (uint32_t)(sel[i] & 0xffffffffull));
      s = __fmul_rn(sc[idx], qs_sh);
    }
    a.topk_out[(size_t)b * k + i] = idx;
    if (a.score_out) a.score_out[(size_t)b * k + i] = s;
  }
}

size_t index_workspace_bytes(int batch, int max_seq_len, int ratio, int window_len) {
  const int nv = visible(max_seq_len, window_len, ratio);
  const size_t stride = ((size_t)max(nv, 1) + 63) / 64 * 64;
  return (size_t)batch * stride * sizeof(float);
}

cudaError_t launch_index_topk(IndexArgs a, int max_seq_len, cudaStream_t stream) {
  const int nv = visible(max_seq_len, a.window_len, a.ratio);
  a.max_len = max_seq_len;
  a.ws_stride = (int)(((size_t)max(nv, 1) + 63) / 64 * 64);
  a.chunk = 4096;
  if (nv > 0) {
    dim3 grid((nv + a.chunk - 1) / a.chunk, a.batch);
    index_score_kernel<<<grid, kScoreThreads, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  index_select_kernel<<<a.batch, kSelectThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace v4kv
