// Slot mapping: logical index -> physical slot through the block table
// (P1 §3.1.1: one 256-token logical block per page of each cache kind).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace v4kv {

__device__ __forceinline__ void touched(int s, int n, int r, int* first, int* count) {
  if (n <= 0) {
    *first = 0;
    *count = 0;
    return;
  }
  *first = s / r;
  int end = (s + n + r - 1) / r;
  *count = end - *first;
}

// one block per sequence; the block first sums the counts of the sequences
// before it (batch is small: a few thousand at most)
__global__ void slot_mapping_kernel(const int32_t* __restrict__ bt, int max_blocks, int batch,
                                    const int32_t* __restrict__ seq_start,
                                    const int32_t* __restrict__ n_new, int r, int spb,
                                    int num_pages, int32_t* __restrict__ cu_out,
                                    int64_t* __restrict__ slot_out, long long cap,
                                    int32_t* __restrict__ st) {
  tc::pdl_wait();  // the lengths and block tables (earlier work in the stream) are complete
  tc::pdl_launch_dependents();
  const int b = blockIdx.x;
  long long part = 0;
  for (int i = threadIdx.x; i < b; i += blockDim.x) {
    int f, c;
    touched(seq_start[i], n_new[i], r, &f, &c);
    part += c;
  }
  __shared__ long long sred[32];
  {
    long long v = part;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      long long t = 0;
      for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) t += sred[w];
      sred[0] = t;
    }
    __syncthreads();
  }
  const long long base = sred[0];
  int first, count;
  touched(seq_start[b], n_new[b], r, &first, &count);
  if (threadIdx.x == 0 && cu_out) {
    cu_out[b] = (int32_t)base;
    if (b == batch - 1) cu_out[batch] = (int32_t)(base + count);
  }
  const int32_t* row = bt + (size_t)b * max_blocks;
  for (int i = threadIdx.x; i < count; i += blockDim.x) {
    long long o = base + i;
    if (o >= cap) {
      flag(st, V4KV_DEV_OVERFLOW);
      continue;
    }
    long long j = (long long)first + i;
    int p = page_of(row, max_blocks, j, spb, num_pages, st);
    slot_out[o] = p < 0 ? -1 : (long long)p * spb + (j % spb);
  }
}

cudaError_t launch_slot_mapping(const int32_t* bt, int max_blocks, int batch,
                                const int32_t* seq_start, const int32_t* n_new, int ratio, int spb,
                                int num_pages, int32_t* cu_out, int64_t* slot_out, long long cap,
                                int32_t* st, cudaStream_t stream) {
  return launch_pdl(slot_mapping_kernel, dim3(batch), dim3(256), 0, stream, bt, max_blocks, batch,
                    seq_start, n_new, ratio, spb, num_pages, cu_out, slot_out, cap, st);
}

}  // namespace v4kv
