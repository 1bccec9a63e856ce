// Indexer scores over c4a entries and exact top-k (P1 §2.2 indexer cache;
// P1 §4.1 sparse attention over the selected c4a entries).
//
// Score of entry j: fp32 fused multiply-add chain over d = 0..dim-1 of
// q8[d] * k8_j[d] (q8 = the query quantised per vector to fp8), times the
// entry's fp32 scale. Ranking: score descending, index ascending, -0 == +0.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace v4kv {

constexpr int kIdxMaxDim = 512;
constexpr int kScoreThreads = 256;
constexpr int kScoreChunk = 2048;   // entries per scoring block (8 per thread)
constexpr int kSelectThreads = 1024;
constexpr int kMaxK = 2048;
constexpr int kBins = 4096;         // histogram of the top 12 bits of the ranking key
constexpr int kBinShift = 20;
constexpr int kCandCap = 1024;      // entries of the threshold bin sorted directly

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

// acc = fl32(acc + q*k) for four consecutive dims, in ascending order; k4
// holds four fp8 codes (lowest byte first), q01 / q23 the query's f16 pairs.
// Both factors are exact in f16, so each step is the fp32 fused multiply-add
// of the exact product.
__device__ __forceinline__ float fma4_fp8(float acc, uint32_t k4, uint32_t q01, uint32_t q23) {
  const __half2 k01 = e4m3x2_to_half2((uint16_t)(k4 & 0xffffu));
  const __half2 k23 = e4m3x2_to_half2((uint16_t)(k4 >> 16));
  const uint32_t a = *reinterpret_cast<const uint32_t*>(&k01);
  const uint32_t c = *reinterpret_cast<const uint32_t*>(&k23);
  asm("{\n\t.reg .f16 a0, a1, b0, b1, c0, c1, d0, d1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
      "mov.b32 {c0, c1}, %3;\n\tmov.b32 {d0, d1}, %4;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\tfma.rn.f32.f16 %0, a1, b1, %0;\n\t"
      "fma.rn.f32.f16 %0, c0, d0, %0;\n\tfma.rn.f32.f16 %0, c1, d1, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(q01), "r"(c), "r"(q23));
  return acc;
}

// the same chain over eight consecutive dims whose keys are fp4-e2m1 codes
// (k8: four bytes, dim 2i in the low nibble of byte i, lowest byte first);
// q[0..3] the query's f16 pairs of these dims. e2m1 values are exact in f16.
__device__ __forceinline__ float fma8_fp4(float acc, uint32_t k8, const uint32_t* q) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw kr = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((k8 >> (8 * i)) & 0xffu), __NV_E2M1);
    const uint32_t kk = (uint32_t)kr.x | ((uint32_t)kr.y << 16);
    asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %0;\n\tfma.rn.f32.f16 %0, a1, b1, %0;\n\t}"
        : "+f"(acc)
        : "r"(kk), "r"(q[i]));
  }
  return acc;
}

// order-preserving map of fp32 onto uint32 (larger float -> larger key)
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.f) u = 0u;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// grid (chunks of kScoreChunk entries, batch); 256 threads, each scoring two
// entries at a time with all their row loads in flight. Also builds the
// histogram of the top 12 key bits of every sequence (workspace hist[b][]).
__global__ void __launch_bounds__(kScoreThreads) index_score_kernel(IndexArgs a) {
  __shared__ __align__(16) uint32_t q16[kIdxMaxDim / 2];  // query codes as f16 pairs
  __shared__ uint32_t hist[kBins];
  __shared__ float red[32];
  tc::pdl_launch_dependents();  // the select kernel may launch; it waits for this grid's results
  const int b = blockIdx.y;
  const int L = seq_len_of(a, b);
  const int n_vis = visible(L, a.window_len, a.ratio);
  const int j0 = blockIdx.x * kScoreChunk;
  if (j0 >= n_vis) return;
  const int dim = a.cache.dim;
  {
    const float* q = a.q_idx + (size_t)b * dim;
    float m = 0.f;
    for (int d = threadIdx.x; d < dim; d += blockDim.x) m = fmaxf(m, fabsf(q[d]));
    const float amax = block_reduce<true>(m, red);
    const float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, kE4m3Max);
    for (int d = 2 * threadIdx.x; d < dim; d += 2 * blockDim.x) {
      const uint16_t c2 = float2_to_e4m3x2(__fdiv_rn(q[d], scale), __fdiv_rn(q[d + 1], scale));
      const __half2 h = e4m3x2_to_half2(c2);
      q16[d / 2] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  const int j1 = min(n_vis, j0 + kScoreChunk);
  const int32_t* bt = a.cache.block_table + (size_t)b * a.cache.max_blocks;
  const uint8_t* base = reinterpret_cast<const uint8_t*>(a.cache.data);
  const bool fp4 = a.cache.dtype == V4KV_FP4_E2M1;
  const int rowb = fp4 ? dim / 2 : dim;  // bytes per key
  const int nq = rowb / 16;              // 16-byte chunks per key
  for (int jj = j0 + threadIdx.x; jj < j1; jj += 2 * blockDim.x) {
    const int ja = jj, jb = jj + blockDim.x;
    const bool hb = jb < j1;
    const int pa = page_of(bt, a.cache.max_blocks, ja, a.cache.spb, a.cache.num_pages, a.dev_status);
    const int pb = hb ? page_of(bt, a.cache.max_blocks, jb, a.cache.spb, a.cache.num_pages, a.dev_status) : -1;
    const long long sa = pa < 0 ? -1 : (long long)pa * a.cache.spb + ja % a.cache.spb;
    const long long sb = pb < 0 ? -1 : (long long)pb * a.cache.spb + jb % a.cache.spb;
    float acc_a = 0.f, acc_b = 0.f;
    for (int c0 = 0; c0 < nq; c0 += 8) {  // up to 128 dims per round, loads first
      uint4 ra[8], rb[8];
      const int nc = min(8, nq - c0);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        ra[c] = (c < nc && sa >= 0) ? *reinterpret_cast<const uint4*>(base + sa * rowb + 16 * (c0 + c)) : make_uint4(0, 0, 0, 0);
        rb[c] = (c < nc && sb >= 0) ? *reinterpret_cast<const uint4*>(base + sb * rowb + 16 * (c0 + c)) : make_uint4(0, 0, 0, 0);
      }
      if (fp4) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c >= nc) break;
          const uint32_t* qq = &q16[16 * (c0 + c)];  // dims 32 (c0 + c) ..
          acc_a = fma8_fp4(acc_a, ra[c].x, qq);
          acc_a = fma8_fp4(acc_a, ra[c].y, qq + 4);
          acc_a = fma8_fp4(acc_a, ra[c].z, qq + 8);
          acc_a = fma8_fp4(acc_a, ra[c].w, qq + 12);
          acc_b = fma8_fp4(acc_b, rb[c].x, qq);
          acc_b = fma8_fp4(acc_b, rb[c].y, qq + 4);
          acc_b = fma8_fp4(acc_b, rb[c].z, qq + 8);
          acc_b = fma8_fp4(acc_b, rb[c].w, qq + 12);
        }
        continue;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c >= nc) break;
        const uint4 qa = *reinterpret_cast<const uint4*>(&q16[8 * (c0 + c)]);
        const uint4 qb = *reinterpret_cast<const uint4*>(&q16[8 * (c0 + c) + 4]);
        acc_a = fma4_fp8(acc_a, ra[c].x, qa.x, qa.y);
        acc_a = fma4_fp8(acc_a, ra[c].y, qa.z, qa.w);
        acc_a = fma4_fp8(acc_a, ra[c].z, qb.x, qb.y);
        acc_a = fma4_fp8(acc_a, ra[c].w, qb.z, qb.w);
        acc_b = fma4_fp8(acc_b, rb[c].x, qa.x, qa.y);
        acc_b = fma4_fp8(acc_b, rb[c].y, qa.z, qa.w);
        acc_b = fma4_fp8(acc_b, rb[c].z, qb.x, qb.y);
        acc_b = fma4_fp8(acc_b, rb[c].w, qb.z, qb.w);
      }
    }
    const float score_a = sa >= 0 ? __fmul_rn(acc_a, a.cache.scales[sa]) : 0.f;
    a.scores_ws[(size_t)b * a.ws_stride + ja] = score_a;
    atomicAdd(&hist[score_key(score_a) >> kBinShift], 1u);
    if (hb) {
      const float score_b = sb >= 0 ? __fmul_rn(acc_b, a.cache.scales[sb]) : 0.f;
      a.scores_ws[(size_t)b * a.ws_stride + jb] = score_b;
      atomicAdd(&hist[score_key(score_b) >> kBinShift], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh = a.hist_ws + (size_t)b * kBins;
  for (int i = threadIdx.x; i < kBins; i += blockDim.x)
    if (hist[i]) atomicAdd(&gh[i], hist[i]);
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

// ---- 128-byte keys (dim 128) on pages of a multiple of 64 entries.
// Each group of 64 consecutive entries is 8 KB of one page, copied by one TMA
// box with 128-byte swizzle: 16-byte chunk c of row r lands at chunk c ^ (r % 8),
// so the eight threads of a quarter-warp, each reading chunk c of its own row,
// hit eight different bank groups. Stages of 256 entries (four boxes) rotate
// through a three-deep ring; every thread scores one entry of each stage with
// the same ascending-d chain as the generic kernel.
// L2 policy for data read once: evicted first, so that it does not push out
// the scores, which the select reads back
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// tc::tma_load_2d with an L2 cache policy
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const void* tmap, int x, int y, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(tc::smem_u32(bar)), "l"(policy)
      : "memory");
}

constexpr int kTmaBox = 64;                    // rows per box
constexpr int kTmaBatch = 256;                 // entries per stage = threads
constexpr int kTmaStages = 3;
constexpr int kTmaChunk = 2048;                // entries per block
constexpr int kTmaGroups = kTmaChunk / kTmaBox;
constexpr uint32_t kStageBytes = kTmaBatch * 128;
constexpr size_t kTmaSmem = 1024 + kTmaStages * kStageBytes + (kBins / 2) * 4 + 64 * 4 +
                            kTmaGroups * 8 + 32 * 4 + kTmaStages * 8 + 16;

// fp4 keys (64 bytes) use the same machinery on the pool seen as 128-byte
// rows of two keys: a 64-entry group is one box of 32 rows, entry e of a stage
// is half e % 2 of row e / 2.
template <bool kFp4>
__global__ void __launch_bounds__(kTmaBatch) index_score_tma_kernel(const __grid_constant__ CUtensorMap keys,
                                                                    IndexArgs a) {
  constexpr int kRowsPerBox = kFp4 ? kTmaBox / 2 : kTmaBox;  // 128-byte rows per 64-entry group
  extern __shared__ uint8_t dsm_raw[];
  tc::pdl_launch_dependents();  // the select kernel may launch; it waits for this grid's results
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* hist2 = reinterpret_cast<uint32_t*>(stages + kTmaStages * kStageBytes);  // 16-bit pairs
  uint32_t* q16 = hist2 + kBins / 2;
  long long* row0 = reinterpret_cast<long long*>(q16 + 64);  // first slot of each group, -1 if bad
  float* red = reinterpret_cast<float*>(row0 + kTmaGroups);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 32);
  int* abort_sh = reinterpret_cast<int*>(full + kTmaStages);
  const int b = blockIdx.y;
  const int L = seq_len_of(a, b);
  const int n_vis = visible(L, a.window_len, a.ratio);
  const int j0 = blockIdx.x * kTmaChunk;
  if (j0 >= n_vis) return;
  const int t = threadIdx.x;
  const int j1 = min(n_vis, j0 + kTmaChunk);
  const int ngroups = (j1 - j0 + kTmaBox - 1) / kTmaBox;
  const int nb = (j1 - j0 + kTmaBatch - 1) / kTmaBatch;
  const int spb = a.cache.spb;
  if (t < kTmaGroups) {
    long long r = -1;
    if (t < ngroups) {
      const long long g0 = (long long)j0 + (long long)t * kTmaBox;  // first entry of the group
      const long long blk = g0 / spb;
      const int32_t* bt = a.cache.block_table + (size_t)b * a.cache.max_blocks;
      const int p = blk < a.cache.max_blocks ? bt[blk] : -1;
      if (p >= 0 && p < a.cache.num_pages) r = ((long long)p * spb + g0 % spb) / (kFp4 ? 2 : 1);
      else flag(a.dev_status, V4KV_DEV_BAD_PAGE);
    }
    row0[t] = r;
  }
  if (t == 0) {
    for (int s = 0; s < kTmaStages; ++s) tc::mbar_init(&full[s], 1);
    *abort_sh = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  const uint32_t stages_s = tc::smem_u32(stages);
  const uint64_t keys_policy = l2_evict_first_policy();  // keys are read once
  auto issue = [&](int bi) {  // thread 0: the boxes of stage bi
    const int s = bi % kTmaStages;
    uint32_t bytes = 0;
    for (int k = 0; k < kTmaBatch / kTmaBox; ++k) {
      const int g = bi * (kTmaBatch / kTmaBox) + k;
      if (g < ngroups && row0[g] >= 0) bytes += kRowsPerBox * 128;
    }
    tc::mbar_arrive_expect_tx(&full[s], bytes);
    for (int k = 0; k < kTmaBatch / kTmaBox; ++k) {
      const int g = bi * (kTmaBatch / kTmaBox) + k;
      if (g < ngroups && row0[g] >= 0)
        tma_load_2d_hint(stages_s + s * kStageBytes + k * kRowsPerBox * 128, &keys, 0, (int)row0[g], &full[s],
                         keys_policy);
    }
  };
  int issued = 0;  // thread 0: stages issued so far
  if (t == 0)
    for (; issued < min(nb, kTmaStages); ++issued) issue(issued);
  // query codes and histogram while the first boxes are in flight
  {
    const float* q = a.q_idx + (size_t)b * 128;
    float m = 0.f;
    if (t < 128) m = fabsf(q[t]);
    const float amax = block_reduce<true>(m, red);
    const float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, kE4m3Max);
    if (t < 64) {
      const uint16_t c2 = float2_to_e4m3x2(__fdiv_rn(q[2 * t], scale), __fdiv_rn(q[2 * t + 1], scale));
      const __half2 h = e4m3x2_to_half2(c2);
      q16[t] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  for (int i = t; i < kBins / 2; i += kTmaBatch) hist2[i] = 0u;
  __syncthreads();
  const int sw = (t & 7) * 16;  // swizzle of this thread's row (stage bases are 1024-aligned)
  for (int bi = 0; bi < nb; ++bi) {
    const int s = bi % kTmaStages;
    const int e = bi * kTmaBatch + t;  // entry offset within the chunk
    const int j = j0 + e;
    const long long r = j < j1 ? row0[e / kTmaBox] : -1;
    const long long slot = r >= 0 ? r * (kFp4 ? 2 : 1) + (e % kTmaBox) : -1;
    const float ks = slot >= 0 ? a.cache.scales[slot] : 0.f;
    if (!tc::mbar_wait(&full[s], (uint32_t)(bi / kTmaStages) & 1u, abort_sh)) {
      flag(a.dev_status, V4KV_DEV_TIMEOUT);
      *abort_sh = 1;
    }
    if (j < j1) {
      float score = 0.f;
      if (slot >= 0 && kFp4) {
        // row t / 2 of the stage (its swizzle phase (t / 2) % 8), half t % 2
        const uint8_t* row = stages + s * kStageBytes + (t >> 1) * 128;
        const int swr = ((t >> 1) & 7) * 16;
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 kv = *reinterpret_cast<const uint4*>(row + ((16 * (4 * (t & 1) + c)) ^ swr));
          const uint32_t* qq = &q16[16 * c];
          acc = fma8_fp4(acc, kv.x, qq);
          acc = fma8_fp4(acc, kv.y, qq + 4);
          acc = fma8_fp4(acc, kv.z, qq + 8);
          acc = fma8_fp4(acc, kv.w, qq + 12);
        }
        score = __fmul_rn(acc, ks);
      } else if (slot >= 0) {
        const uint8_t* row = stages + s * kStageBytes + t * 128;
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 kv = *reinterpret_cast<const uint4*>(row + ((16 * c) ^ sw));
          const uint4 qa = *reinterpret_cast<const uint4*>(&q16[8 * c]);
          const uint4 qb = *reinterpret_cast<const uint4*>(&q16[8 * c + 4]);
          acc = fma4_fp8(acc, kv.x, qa.x, qa.y);
          acc = fma4_fp8(acc, kv.y, qa.z, qa.w);
          acc = fma4_fp8(acc, kv.z, qb.x, qb.y);
          acc = fma4_fp8(acc, kv.w, qb.z, qb.w);
        }
        score = __fmul_rn(acc, ks);
      }
      a.scores_ws[(size_t)b * a.ws_stride + j] = score;
      const uint32_t bin = score_key(score) >> kBinShift;
      atomicAdd(&hist2[bin >> 1], 1u << (16 * (bin & 1)));
    }
    __syncthreads();  // stage s is free again
    if (t == 0 && issued < nb && !*abort_sh) issue(issued++);
  }
  if (*abort_sh && t == 0) {
    // let copies still in flight land before the block's shared memory is released
    for (int bi = max(0, issued - kTmaStages); bi < issued; ++bi)
      tc::mbar_wait(&full[bi % kTmaStages], (uint32_t)(bi / kTmaStages) & 1u, nullptr);
  }
  uint32_t* gh = a.hist_ws + (size_t)b * kBins;
  for (int i = t; i < kBins / 2; i += kTmaBatch) {
    const uint32_t w = hist2[i];
    if (w & 0xffffu) atomicAdd(&gh[2 * i], w & 0xffffu);
    if (w >> 16) atomicAdd(&gh[2 * i + 1], w >> 16);
  }
}

// Composite sort key: ranking key in the high word, bitwise-inverted index in
// the low word, so that a descending sort gives (score desc, index asc).
__device__ __forceinline__ unsigned long long comp_key(uint32_t key, int j) {
  return ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)j);
}

// bitonic sort of v[0 .. n) (n a power of two) in descending order
// number of the n keys v[] (distinct) larger than `mine`; every thread reads
// the same keys at a time (shared-memory broadcast), two per 16-byte load, so
// a warp's scan costs one shared-memory wavefront per two keys. v is 16-byte
// aligned.
__device__ __forceinline__ int rank_of(unsigned long long mine, const unsigned long long* v, int n) {
  const ulonglong2* v2 = reinterpret_cast<const ulonglong2*>(v);
  int r = 0;
  int j = 0;
  for (; j + 4 <= n; j += 4) {
    const ulonglong2 x = v2[j >> 1], y = v2[(j >> 1) + 1];
    r += (x.x > mine) + (x.y > mine) + (y.x > mine) + (y.y > mine);
  }
  for (; j < n; ++j) r += v[j] > mine;
  return r;
}


// Exact radix select, 8 bits per pass from the top: the keys above the k-th
// largest in any order, then the ties at it by ascending index. Used when the
// histogram's threshold bin holds more than kCandCap entries.
__device__ void radix_select_exact(const float* sc, int n, int k, unsigned long long* sel,
                                   uint32_t* hist, uint32_t* scan_sh, uint32_t* pick_sh,
                                   uint32_t* n_sel_sh) {
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
  if (threadIdx.x == 0) *n_sel_sh = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const uint32_t key = score_key(sc[j]);
    if (key > T) sel[atomicAdd(n_sel_sh, 1u)] = comp_key(key, j);
  }
  __syncthreads();
  uint32_t taken = 0;
  const uint32_t base_pos = *n_sel_sh;
  for (int j0 = 0; j0 < n && taken < remaining; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    const uint32_t is_tie = (j < n && score_key(sc[j]) == T) ? 1u : 0u;
    uint32_t total;
    const uint32_t before = block_exclusive_scan(is_tie, scan_sh, &total);
    if (is_tie && taken + before < remaining) sel[base_pos + taken + before] = comp_key(T, j);
    taken += total;
  }
  __syncthreads();
}

// One block per sequence. The histogram of the top 12 key bits (built while
// scoring) gives the bin holding the k-th largest key; one pass keeps every
// entry above that bin and collects the bin's own entries, which are sorted
// to take the rest. The k results are then sorted (score desc, index asc).
__global__ void __launch_bounds__(kSelectThreads) index_select_kernel(IndexArgs a) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t scan_sh[32];
  __shared__ __align__(16) unsigned long long sel[kMaxK];
  __shared__ __align__(16) unsigned long long cand[kCandCap];
  __shared__ float red[32];
  __shared__ float q_f[kIdxMaxDim];
  __shared__ float qs_sh;
  __shared__ uint32_t n_sel_sh, n_cand_sh, bin_sh, above_sh, n_hit_sh;
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
  if (threadIdx.x == 0) {
    n_sel_sh = 0;
    n_cand_sh = 0;
    n_hit_sh = 0;
    bin_sh = 0xffffffffu;  // "not found" -> exact path
    above_sh = 0;
  }
  __syncthreads();
  // everything above reads only the call's inputs, so it overlaps the scoring
  // kernel's tail (programmatic dependent launch); the scores and the
  // histogram are complete from here on
  tc::pdl_wait();

  if (n <= k) {
    for (int j = threadIdx.x; j < n; j += blockDim.x) sel[j] = comp_key(score_key(sc[j]), j);
    __syncthreads();
  } else {
    // threshold bin: count(bins above) < k <= count(bins at or above)
    const uint32_t* gh = a.hist_ws + (size_t)b * kBins;
    uint32_t local = 0, cnt[kBins / kSelectThreads];
#pragma unroll
    for (int i = 0; i < kBins / kSelectThreads; ++i) {
      cnt[i] = gh[kBins - 1 - (threadIdx.x * (kBins / kSelectThreads) + i)];  // descending bins
      local += cnt[i];
    }
    uint32_t total;
    const uint32_t before = block_exclusive_scan(local, scan_sh, &total);
    if (before < (uint32_t)k && (uint32_t)k <= before + local) {
      uint32_t run = before;
#pragma unroll
      for (int i = 0; i < kBins / kSelectThreads; ++i) {
        if (run + cnt[i] >= (uint32_t)k) {
          bin_sh = kBins - 1 - (threadIdx.x * (kBins / kSelectThreads) + i);
          above_sh = run;
          break;
        }
        run += cnt[i];
      }
    }
    __syncthreads();
    const uint32_t tb = bin_sh, above = above_sh;
    if (tb != 0xffffffffu) {
      // four scores per 16-byte load, four loads in flight per thread (the
      // score rows are 256-byte aligned; entries past n are skipped)
      auto take = [&](float f, int j) {
        if (j >= n) return;
        const uint32_t key = score_key(f);
        const uint32_t bin = key >> kBinShift;
        if (bin > tb) {
          const uint32_t p = atomicAdd(&n_sel_sh, 1u);
          if (p < (uint32_t)k) sel[p] = comp_key(key, j);
        } else if (bin == tb) {
          const uint32_t p = atomicAdd(&n_cand_sh, 1u);
          if (p < (uint32_t)kCandCap) cand[p] = comp_key(key, j);
        }
      };
      // a float below f0, the smallest float whose key reaches the threshold
      // bin, has a key below it (the key is monotone in the float order), so a
      // load of four such scores needs no per-score work (a NaN fails every
      // comparison and takes the exact test)
      const uint32_t k0 = tb << kBinShift;
      const float f0 = __uint_as_float((k0 & 0x80000000u) ? (k0 & 0x7fffffffu) : ~k0);
      const float4* sc4 = reinterpret_cast<const float4*>(sc);
      const int n4 = (n + 3) / 4;
      // pass 1: the float4 loads holding a score at or above the threshold bin
      // (about one in twenty) are listed in shared memory (`hist`, free until
      // the exact path), one atomic per warp and round; pass 2 takes their
      // scores, spread over all threads
      uint32_t* hitq = hist;
      const int lane = threadIdx.x & 31;
      const uint32_t below = (1u << lane) - 1u;
      for (int q0 = threadIdx.x - lane; q0 < n4; q0 += 4 * blockDim.x) {  // warp-uniform
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = q0 + lane + u * blockDim.x;
          v[u] = q < n4 ? sc4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = q0 + lane + u * blockDim.x;
          const bool hit = q < n4 && !(v[u].x < f0 && v[u].y < f0 && v[u].z < f0 && v[u].w < f0);
          const uint32_t m = __ballot_sync(0xffffffffu, hit);
          if (m == 0u) continue;
          const int leader = __ffs(m) - 1;
          uint32_t base = 0;
          if (lane == leader) base = atomicAdd(&n_hit_sh, (uint32_t)__popc(m));
          base = __shfl_sync(0xffffffffu, base, leader);
          const uint32_t pos = base + __popc(m & below);
          if (hit && pos < (uint32_t)kBins) hitq[pos] = (uint32_t)q;
        }
      }
      __syncthreads();
      const uint32_t nh = min(n_hit_sh, (uint32_t)kBins);  // more: the counts below disagree, exact path
      for (uint32_t h = threadIdx.x; h < nh; h += blockDim.x) {
        const int q = (int)hitq[h];
        const float4 x = sc4[q];
        take(x.x, 4 * q);
        take(x.y, 4 * q + 1);
        take(x.z, 4 * q + 2);
        take(x.w, 4 * q + 3);
      }
    }
    __syncthreads();
    const uint32_t nc = n_cand_sh;
    if (tb == 0xffffffffu || nc > (uint32_t)kCandCap || n_sel_sh != above || n_hit_sh > (uint32_t)kBins) {
      // too many entries share the threshold bin: exact radix path
      for (int i = threadIdx.x; i < kpow; i += blockDim.x) sel[i] = 0ull;
      __syncthreads();
      radix_select_exact(sc, n, k, sel, hist, scan_sh, pick_sh, &n_sel_sh);
    } else {
      // the threshold bin's best k - above candidates: a candidate's rank is
      // the number of candidates with a larger key (keys are distinct)
      const int need = k - (int)above;
      for (int c = threadIdx.x; c < (int)nc; c += blockDim.x) {
        const unsigned long long mine = cand[c];
        const int r = rank_of(mine, cand, (int)nc);
        if (r < need) sel[above + r] = mine;
      }
      __syncthreads();
    }
  }

  // output position of each selected key = its rank among the selected keys
  const int valid = min(n, k);
  for (int i = threadIdx.x; i < valid; i += blockDim.x) {
    const unsigned long long mine = sel[i];
    const int32_t idx = (int32_t)(0xffffffffu - (uint32_t)(mine & 0xffffffffull));
    const float raw = a.score_out ? sc[idx] : 0.f;  // requested before the ranking
    const int r = rank_of(mine, sel, valid);
    a.topk_out[(size_t)b * k + r] = idx;
    if (a.score_out) a.score_out[(size_t)b * k + r] = __fmul_rn(raw, qs_sh);
  }
  for (int i = valid + threadIdx.x; i < k; i += blockDim.x) {
    a.topk_out[(size_t)b * k + i] = -1;
    if (a.score_out) a.score_out[(size_t)b * k + i] = 0.f;
  }
}

static size_t score_stride(int nv) { return ((size_t)max(nv, 1) + 63) / 64 * 64; }

size_t index_workspace_bytes(int batch, int max_seq_len, int ratio, int window_len) {
  const int nv = visible(max_seq_len, window_len, ratio);
  return (size_t)batch * score_stride(nv) * sizeof(float) + (size_t)batch * kBins * sizeof(uint32_t);
}

cudaError_t launch_index_topk(IndexArgs a, int max_seq_len, cudaStream_t stream) {
  const int nv = visible(max_seq_len, a.window_len, a.ratio);
  a.max_len = max_seq_len;
  a.ws_stride = (int)score_stride(nv);
  a.chunk = kScoreChunk;
  a.hist_ws = reinterpret_cast<uint32_t*>(a.scores_ws + (size_t)a.batch * a.ws_stride);
  cudaError_t e = cudaMemsetAsync(a.hist_ws, 0, (size_t)a.batch * kBins * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  // 128-dim keys (128 bytes fp8, 64 bytes fp4) on pages of whole 64-entry
  // groups go through TMA boxes of 128-byte rows
  const bool fp4 = a.cache.dtype == V4KV_FP4_E2M1;
  const bool tma = a.cache.dim == 128 && a.cache.spb % kTmaBox == 0 &&
                   (reinterpret_cast<uintptr_t>(a.cache.data) & 15) == 0 &&
                   (long long)a.cache.num_pages * a.cache.spb <= 0x7fffffffLL;
  if (nv > 0 && tma) {
    CUtensorMap keys;
    const uint64_t rows = (uint64_t)a.cache.num_pages * a.cache.spb / (fp4 ? 2 : 1);
    e = encode_rows_u8(&keys, a.cache.data, rows, 128, fp4 ? kTmaBox / 2 : kTmaBox);
    if (e != cudaSuccess) return e;
    auto kern = fp4 ? index_score_tma_kernel<true> : index_score_tma_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTmaSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((nv + kTmaChunk - 1) / kTmaChunk, a.batch);
    kern<<<grid, kTmaBatch, kTmaSmem, stream>>>(keys, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else if (nv > 0) {
    dim3 grid((nv + kScoreChunk - 1) / kScoreChunk, a.batch);
    index_score_kernel<<<grid, kScoreThreads, 0, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(index_select_kernel, dim3(a.batch), dim3(kSelectThreads), 0, stream, a);
}

}  // namespace v4kv
