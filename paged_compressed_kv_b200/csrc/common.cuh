// Device helpers shared by the v4kv kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/v4kv.h"
#include "kernels.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "v4kv kernels are written for sm_100a (B200) only"
#endif

namespace v4kv {

constexpr int kLogicalBlock = 256;  // raw tokens per logical block (P1 §3.1.1)
constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ void flag(int32_t* st, int bit) {
  if (st) atomicOr(st, bit);
}

// ---------------------------------------------------------------- codecs
// fp8-e4m3 pair -> f16 pair, exact (every e4m3 value is an f16 value).
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint16_t two) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return *reinterpret_cast<__half2*>(&r);
}

__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  __half_raw r = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&r));
}

// two fp32 -> two e4m3 codes, round to nearest even, saturating to +-448
__device__ __forceinline__ uint16_t float2_to_e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// ---------------------------------------------------------------- RoPE
// cos / sin of pos * theta^(-2i/rope_dim), formed in fp64 and rounded to fp32.
// cos and sin of pair i's angle at position pos: pos * theta^(-2i/rope_dim)
// in fp64 (the host precomputes the first kRopeTable frequencies), rounded to
// fp32
__device__ __forceinline__ void rope_cs(const RopeArgs& rp, int i, long long pos, float* c,
                                        float* s) {
  const double freq =
      i < kRopeTable ? rp.freq[i] : pow(rp.theta, -2.0 * (double)i / (double)rp.rope_dim);
  const double ang = (double)pos * freq;
  double sd, cd;
  sincos(ang, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

// rotate the pair (a, b) by (c, s) with separately rounded fp32 products
__device__ __forceinline__ void rope_apply(float& a, float& b, float c, float s) {
  float na = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
  float nb = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
  a = na;
  b = nb;
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// block-wide reductions; `red` holds >= 32 floats of shared memory
template <bool kMax>
__device__ __forceinline__ float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = kMax ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float t = lane < nw ? red[lane] : (kMax ? -INFINITY : 0.f);
    t = kMax ? warp_max(t) : warp_sum(t);
    if (lane == 0) red[0] = t;
  }
  __syncthreads();
  float r = red[0];
  __syncthreads();
  return r;
}

// Output epilogue of decode attention for n consecutive values of one
// (sequence, head) vector held by this thread (amax = the vector's absolute
// maximum, reduced by the caller): bf16, or e4m3 codes with the vector's
// scale amax / 448 (1 if amax == 0; IEEE division per element, round to
// nearest even, saturating), optionally also the fp32 values themselves.
template <int N>
__device__ __forceinline__ void store_output(const DecodeArgs& a, size_t row, int d0, const float* v,
                                             float amax, bool scale_writer) {
  const size_t off = row * 512 + d0;
  if (a.prequant_out) {
#pragma unroll
    for (int i = 0; i < N; i += 4)
      *reinterpret_cast<float4*>(a.prequant_out + off + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  }
  if (a.out_fp8) {
    const float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, kE4m3Max);
    uint32_t w[N / 4];
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint16_t lo = float2_to_e4m3x2(__fdiv_rn(v[4 * i], scale), __fdiv_rn(v[4 * i + 1], scale));
      const uint16_t hi = float2_to_e4m3x2(__fdiv_rn(v[4 * i + 2], scale), __fdiv_rn(v[4 * i + 3], scale));
      w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    uint8_t* dst = reinterpret_cast<uint8_t*>(a.out) + off;
    if constexpr (N == 16) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) reinterpret_cast<uint32_t*>(dst)[i] = w[i];
    }
    if (scale_writer) a.out_scales[row] = scale;
  } else {
    uint32_t w[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i)
      w[i] = (uint32_t)float_to_bf16_bits(v[2 * i]) | ((uint32_t)float_to_bf16_bits(v[2 * i + 1]) << 16);
    uint16_t* dst = reinterpret_cast<uint16_t*>(a.out) + off;
#pragma unroll
    for (int i = 0; i < N / 2; i += 2) *reinterpret_cast<uint2*>(dst + 2 * i) = make_uint2(w[i], w[i + 1]);
  }
}

// page of logical index j through a block-table row; -1 if absent
__device__ __forceinline__ int page_of(const int32_t* bt_row, int max_blocks, long long j, int spb,
                                       int num_pages, int32_t* st) {
  long long blk = j / spb;
  if (blk < 0 || blk >= max_blocks) {
    flag(st, V4KV_DEV_BAD_SLOT);
    return -1;
  }
  int p = bt_row[blk];
  if (p < 0 || p >= num_pages) {
    flag(st, V4KV_DEV_BAD_PAGE);
    return -1;
  }
  return p;
}

// launch with programmatic stream serialization: the kernel may start while
// the previous one in the stream finishes; it waits (griddepcontrol.wait)
// before it reads that kernel's results
template <typename... Args>
inline cudaError_t launch_pdl(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace v4kv
