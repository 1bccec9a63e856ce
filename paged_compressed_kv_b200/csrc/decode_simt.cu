// Decode attention on CUDA cores (any head count up to 128), split-K over the
// attended items, and the split merge + inverse RoPE epilogue.
// (P1 §2.1 shared K = V and inverse RoPE on the output; §2.3 window.)
//
// Item list of sequence b: items [0, n_sel) are compressed entries (all
// visible entries in ascending order, or the top-k list), items
// [n_sel, n_sel + n_win) are the window tokens [L - n_win, L). Split s covers
// items [s*split, (s+1)*split). Scores are kept in log2 units (q is
// pre-multiplied by sm_scale * log2(e)) and exponentiated with exp2.
#include "common.cuh"
#include "kernels.h"

namespace v4kv {

constexpr int kDim = 512;
constexpr int kSimtWarps = 8;
constexpr int kSimtHpw = 2;                         // heads per warp
constexpr int kSimtHeads = kSimtWarps * kSimtHpw;   // heads per block
constexpr float kLog2e = 1.4426950408889634f;

struct SeqItems {
  int L, n_vis, n_sel, n_win, w0, n_items;
};

__device__ __forceinline__ SeqItems seq_items(const DecodeArgs& a, int b) {
  SeqItems s;
  int L = a.seq_lens[b];
  if (L > a.max_len) {  // longer than the workspace was sized for: clamp
    if (threadIdx.x == 0) flag(a.dev_status, V4KV_DEV_OVERFLOW);
    L = a.max_len;
  }
  s.L = max(0, L);
  s.n_vis = max(0, s.L - a.window_len) / a.ratio;
  s.n_sel = a.topk ? a.k : s.n_vis;
  s.w0 = max(0, s.L - a.window_len);
  s.n_win = s.L - s.w0;
  s.n_items = (a.pad_sel ? (s.n_sel + 127) / 128 * 128 : s.n_sel) + s.n_win;
  return s;
}

// Resolve item `it` of sequence b to (pool, slot); false if it is skipped
// (a -1 top-k entry, an out-of-range index or an unmapped page).
__device__ __forceinline__ bool resolve_item(const DecodeArgs& a, int b, const SeqItems& si, int it,
                                             bool* is_win, long long* slot) {
  if (it < si.n_sel) {
    long long j = a.topk ? (long long)a.topk[(size_t)b * a.k + it] : (long long)it;
    if (j < 0) return false;
    const long long stored = ((long long)si.L + a.ratio - 1) / a.ratio;
    if (j >= stored) {
      flag(a.dev_status, V4KV_DEV_BAD_INDEX);
      return false;
    }
    const int p = page_of(a.main.block_table + (size_t)b * a.main.max_blocks, a.main.max_blocks, j,
                          a.main.spb, a.main.num_pages, a.dev_status);
    if (p < 0) return false;
    *is_win = false;
    *slot = (long long)p * a.main.spb + j % a.main.spb;
    return true;
  }
  const long long t = si.w0 + (it - si.n_sel);
  const int p = page_of(a.window.block_table + (size_t)b * a.window.max_blocks,
                        a.window.max_blocks, t, a.window.spb, a.window.num_pages, a.dev_status);
  if (p < 0) return false;
  *is_win = true;
  *slot = (long long)p * a.window.spb + t % a.window.spb;
  return true;
}

// 16 consecutive dims [d0, d0+16) of one stored vector, as fp32 values
__device__ __forceinline__ void load16(const PoolArgs& pool, long long slot, int d0, float* v) {
  if (pool.dtype == V4KV_FP8_E4M3) {
    const uint4 raw =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(pool.data) + slot * kDim + d0);
    const float sc = pool.scales[slot];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 lo = __half22float2(e4m3x2_to_half2((uint16_t)(w[i] & 0xffff)));
      const float2 hi = __half22float2(e4m3x2_to_half2((uint16_t)(w[i] >> 16)));
      v[4 * i + 0] = lo.x * sc;
      v[4 * i + 1] = lo.y * sc;
      v[4 * i + 2] = hi.x * sc;
      v[4 * i + 3] = hi.y * sc;
    }
  } else {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(pool.data) + slot * kDim + d0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 raw = *reinterpret_cast<const uint4*>(p + 8 * h);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * h + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * h + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  }
}

// grid (n_splits, ceil(heads / 16), batch); 8 warps, 2 heads each; lane l
// owns dims [16 l, 16 l + 16)
__global__ void __launch_bounds__(kSimtWarps * 32) decode_simt_kernel(DecodeArgs a) {
  __shared__ __align__(16) float vals[kSimtWarps][kDim];
  __shared__ int valid[kSimtWarps];
  const int b = blockIdx.z;
  const int split = blockIdx.x;
  const SeqItems si = seq_items(a, b);
  const int i0 = split * a.split;
  if (i0 >= si.n_items) return;
  const int i1 = min(si.n_items, i0 + a.split);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d0 = lane * 16;

  int heads[kSimtHpw];
  float qf[kSimtHpw][16], of[kSimtHpw][16], m[kSimtHpw], l[kSimtHpw];
  const float qscale = a.sm_scale * kLog2e;
#pragma unroll
  for (int i = 0; i < kSimtHpw; ++i) {
    heads[i] = blockIdx.y * kSimtHeads + i * kSimtWarps + warp;
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      of[i][d] = 0.f;
      float qv = 0.f;
      if (heads[i] < a.heads) {
        const size_t off = ((size_t)b * a.heads + heads[i]) * kDim + d0 + d;
        qv = a.q_dtype == V4KV_FP32 ? reinterpret_cast<const float*>(a.q)[off]
                                    : bf16_bits_to_float(reinterpret_cast<const uint16_t*>(a.q)[off]);
      }
      qf[i][d] = qv * qscale;
    }
  }

  for (int t0 = i0; t0 < i1; t0 += kSimtWarps) {
    // warp w stages item t0 + w
    {
      const int it = t0 + warp;
      bool ok = false, is_win = false;
      long long slot = 0;
      if (it < i1) ok = resolve_item(a, b, si, it, &is_win, &slot);
      if (ok) {
        float v[16];
        load16(is_win ? a.window : a.main, slot, d0, v);
        float4* dst = reinterpret_cast<float4*>(&vals[warp][d0]);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
      if (lane == 0) valid[warp] = ok;
    }
    __syncthreads();
    const int nt = min(kSimtWarps, i1 - t0);
    for (int t = 0; t < nt; ++t) {
      if (!valid[t]) continue;
      float v[16];
      const float4* src = reinterpret_cast<const float4*>(&vals[t][d0]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = src[i];
        v[4 * i] = x.x;
        v[4 * i + 1] = x.y;
        v[4 * i + 2] = x.z;
        v[4 * i + 3] = x.w;
      }
#pragma unroll
      for (int h = 0; h < kSimtHpw; ++h) {
        float part = 0.f;
#pragma unroll
        for (int d = 0; d < 16; ++d) part = fmaf(qf[h][d], v[d], part);
        const float s = warp_sum(part);
        const float mn = fmaxf(m[h], s);
        const float alpha = exp2f(m[h] - mn);
        const float p = exp2f(s - mn);
        l[h] = l[h] * alpha + p;
#pragma unroll
        for (int d = 0; d < 16; ++d) of[h][d] = fmaf(p, v[d], of[h][d] * alpha);
        m[h] = mn;
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int h = 0; h < kSimtHpw; ++h) {
    if (heads[h] >= a.heads) continue;
    const size_t row = ((size_t)b * a.n_splits + split) * a.heads + heads[h];
    float4* dst = reinterpret_cast<float4*>(a.part_o + row * kDim + d0);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_float4(of[h][4 * i], of[h][4 * i + 1], of[h][4 * i + 2], of[h][4 * i + 3]);
    if (lane == 0) {
      a.part_ml[row * 2] = m[h];
      a.part_ml[row * 2 + 1] = l[h];
    }
  }
}

// grid (heads, batch), 128 threads x 4 dims: merge the splits, normalise,
// inverse RoPE at position L - 1, store bf16
__global__ void __launch_bounds__(128) decode_merge_kernel(DecodeArgs a) {
  const int h = blockIdx.x, b = blockIdx.y;
  const SeqItems si = seq_items(a, b);
  const int ns = min(a.n_splits, (si.n_items + a.split - 1) / a.split);
  const int d0 = threadIdx.x * 4;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) {
    const size_t row = ((size_t)b * a.n_splits + s) * a.heads + h;
    M = fmaxf(M, a.part_ml[row * 2]);
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, L = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const size_t row = ((size_t)b * a.n_splits + s) * a.heads + h;
      const float ms = a.part_ml[row * 2];
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      L = fmaf(w, a.part_ml[row * 2 + 1], L);
      const float4 o = *reinterpret_cast<const float4*>(a.part_o + row * kDim + d0);
      acc[0] = fmaf(w, o.x, acc[0]);
      acc[1] = fmaf(w, o.y, acc[1]);
      acc[2] = fmaf(w, o.z, acc[2]);
      acc[3] = fmaf(w, o.w, acc[3]);
    }
  }
  float o[4];
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = acc[i] * inv;
  if (a.rope.rope_dim > 0 && si.L > 0) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int d = d0 + 2 * k;
      if (d >= a.rope.rope_offset && d + 1 < a.rope.rope_offset + a.rope.rope_dim) {
        float c, s;
        rope_cs(a.rope, (d - a.rope.rope_offset) >> 1, (long long)si.L - 1, &c, &s);
        rope_apply(o[2 * k], o[2 * k + 1], c, -s);
      }
    }
  }
  float amax = 0.f;
  if (a.out_fp8) {
    __shared__ float red[32];
    amax = block_reduce<true>(fmaxf(fmaxf(fabsf(o[0]), fabsf(o[1])), fmaxf(fabsf(o[2]), fabsf(o[3]))), red);
  }
  store_output<4>(a, (size_t)b * a.heads + h, d0, o, amax, threadIdx.x == 0);
}

DecodePlan plan_decode(int batch, int heads, int max_seq_len, int ratio, int window_len, int k,
                       int main_dtype, int dim, int num_sms) {
  (void)main_dtype;
  (void)dim;
  DecodePlan p{};
  const int L = max(0, max_seq_len);
  const int n_vis = max(0, L - window_len) / ratio;
  const int n_sel = k > 0 ? k : n_vis;
  const int n_win = min(L, window_len);
  if (heads == 64) {
    // tensor-core kernel: a persistent grid of one block per SM over the tile
    // list of all sequences (entries padded to whole tiles of 128 items)
    p.path = 1;
    p.items_max = (n_sel + 127) / 128 * 128 + n_win;
    p.split = 128;
    p.n_splits = max(1, min(num_sms, 160));  // the merge holds <= 160 weights per sequence
    p.ws_bytes = decode_tc_workspace_bytes(batch, p.n_splits);
    return p;
  }
  p.path = 0;
  p.items_max = n_sel + n_win;
  // aim for about four blocks per SM over all head groups
  const int head_groups = (heads + kSimtHeads - 1) / kSimtHeads;
  const long long target = (long long)num_sms * 4 / max(1, head_groups);
  const long long total = (long long)p.items_max * batch;
  long long split = (total + target - 1) / max(1LL, target);
  split = max(64LL, min(8192LL, ((split + 63) / 64) * 64));
  p.split = (int)split;
  p.n_splits = max(1, (p.items_max + p.split - 1) / p.split);
  p.ws_bytes = (size_t)batch * p.n_splits * heads * (size_t)(kDim + 2) * sizeof(float);
  return p;
}

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream) {
  dim3 grid(a.n_splits, (a.heads + kSimtHeads - 1) / kSimtHeads, a.batch);
  decode_simt_kernel<<<grid, kSimtWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream) {
  dim3 grid(a.heads, a.batch);
  decode_merge_kernel<<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace v4kv
