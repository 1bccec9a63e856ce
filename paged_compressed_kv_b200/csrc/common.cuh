// Device helpers shared by the v4kv kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
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
