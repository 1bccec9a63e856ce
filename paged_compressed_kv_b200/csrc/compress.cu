// Compressor append: softmax-gated group sums -> RoPE -> fp8/bf16 entry,
// raw-token window copy, and the rolling state of the unfinished group.
// (P1 §2.1 c4a / c128a compression, §2.3 window, §3.1.2 compressor state,
//  §3.2.1 compressor + RoPE + cache-insert fusion.)
//
// One launch does all three. Its first blocks copy window rows (one warp per
// token). The rest build entries:
//   ratio 4: one warp per group, eight groups per block, the group's rows
//            staged in shared memory with cp.async;
//   ratio 128: one block per group, each warp summing a run of rows,
//              the eight partial sums added in warp order.
// Every row is an 8-dim chunk per lane (chunk c = lane + 32k), so a lane
// always touches the same columns of every row it reads or writes.
//
// The state of sequence b (its unfinished group's rows and gates) is
// rewritten by the warp or block that builds b's first entry of the call,
// after it has consumed the old state. That group is the only reader of the
// old state, so no other block can observe a half-written state.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace v4kv {
namespace {

constexpr int kMaxRatio = 128;
constexpr int kWarps = 8;       // warps per block
constexpr int kCuSmem = 1024;   // sequences whose entry prefix sums fit in shared memory

__device__ __forceinline__ void unpack_bf16x8(uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <int KC>
__device__ __forceinline__ void load_row(const uint16_t* row, int lane, int nch, uint4 (&q)[KC]) {
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const int c = lane + 32 * k;
    q[k] = c < nch ? __ldcs(reinterpret_cast<const uint4*>(row + 8 * c)) : make_uint4(0, 0, 0, 0);
  }
}

// (cos, sin) of rope pair `lane` at position `pos` (identity past the last
// pair): the first 32 pairs' values, one per lane, which rope_warp uses
__device__ __forceinline__ void rope_pair_lane(const RopeArgs& rp, int lane, long long pos, float* c,
                                               float* s) {
  *c = 1.f;
  *s = 0.f;
  if (lane < (rp.rope_dim >> 1)) rope_cs(rp, lane, pos, c, s);
}

// rotate the rope pairs among this lane's dims at position `pos`. Pair p's
// (cos, sin) is evaluated once per warp, by lane p % 32, and fetched with
// shuffles, so every lane must call this. (c0, s0) are this lane's values
// for the first 32 pairs (rope_pair_lane), evaluated by the caller, which
// can then do it while it waits for memory.
template <int KC>
__device__ __forceinline__ void rope_warp(float (&e)[KC][8], int lane, int nch, const RopeArgs& rp,
                                          long long pos, float c0, float s0) {
  if (rp.rope_dim == 0) return;
  const int npairs = rp.rope_dim >> 1;
  for (int base = 0; base < npairs; base += 32) {
    float c = c0, s = s0;
    if (base > 0) {
      c = 1.f;
      s = 0.f;
      if (base + lane < npairs) rope_cs(rp, base + lane, pos, &c, &s);
    }
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      // chunks 32k .. 32k + 31 hold dims [256k, 256k + 256): skip them (the
      // whole warp) when none is rotated
      if (256 * k >= rp.rope_offset + rp.rope_dim || 256 * (k + 1) <= rp.rope_offset) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = 8 * (lane + 32 * k) + 2 * j;
        const int p = (d - rp.rope_offset) >> 1;
        const float cc = __shfl_sync(0xffffffffu, c, p & 31);
        const float ss = __shfl_sync(0xffffffffu, s, p & 31);
        if (lane + 32 * k < nch && d >= rp.rope_offset && p >= base && p < base + 32 && p < npairs)
          rope_apply(e[k][2 * j], e[k][2 * j + 1], cc, ss);
      }
    }
  }
}

template <int KC>
__device__ __forceinline__ void rope_warp(float (&e)[KC][8], int lane, int nch, const RopeArgs& rp,
                                          long long pos) {
  if (rp.rope_dim == 0) return;
  float c0, s0;
  rope_pair_lane(rp, lane, pos, &c0, &s0);
  rope_warp<KC>(e, lane, nch, rp, pos, c0, s0);
}

// e4m3 codes of v / scale from the product q = v * y, y = 1 / scale rounded to
// nearest. The product is within 2 fp32 ulps of v / scale (two roundings of
// relative size 2^-24 each), and the correctly rounded quotient within half an
// ulp of it, so both give the same e4m3 code unless v / scale lies near the
// midpoint between two neighbouring codes. The code of a normal-range value
// (binades 2^-6 .. 2^8) depends only on the 3 leading mantissa bits and the
// rounding bit below them, so a midpoint is a pattern of 0x80000 in the 20 low
// mantissa bits. quotient_needs_ieee(q) is true within 8 ulps of such a
// pattern, below the normal e4m3 range, and for infinities and NaNs: there the
// IEEE quotient is formed instead, so the codes are those of
// float2_to_e4m3x2(v / scale).
__device__ __forceinline__ bool quotient_needs_ieee(float q) {
  const uint32_t u = __float_as_uint(q) & 0x7fffffffu;
  // outside [2^-6, inf): the unsigned difference wraps past the range
  const bool outside = u - 0x3c800000u >= 0x7f800000u - 0x3c800000u;
  // low 20 mantissa bits within 8 of 0x80000
  const bool near_mid = ((u + 8u - 0x80000u) & 0xfffffu) <= 16u;
  return outside || near_mid;
}

// quantise (fp8: absmax over the warp's whole vector) or round (bf16) one
// vector held by a warp, and store it in `slot` of the pool
template <int KC>
__device__ __forceinline__ void store_entry_warp(const PoolArgs& pool, long long slot, int lane,
                                                 int nch, const float (&e)[KC][8]) {
  if (pool.dtype == V4KV_FP8_E4M3) {
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < KC; ++k)
      if (lane + 32 * k < nch)
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(e[k][i]));
    const float amax = warp_max(m);
    const float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, kE4m3Max);
    const float y = __frcp_rn(scale);
    uint8_t* base = reinterpret_cast<uint8_t*>(pool.data) + slot * pool.dim;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      // the products; the IEEE quotient only where one needs it (one vote per
      // chunk row, so the common case has no per-value branch)
      float qv[8];
      bool ieee = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        qv[i] = __fmul_rn(e[k][i], y);
        ieee |= quotient_needs_ieee(qv[i]);
      }
      ieee = ieee && c < nch;
      if (__any_sync(0xffffffffu, ieee) && ieee) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (quotient_needs_ieee(qv[i])) qv[i] = __fdiv_rn(e[k][i], scale);
      }
      if (c >= nch) continue;
      uint16_t q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = float2_to_e4m3x2(qv[2 * i], qv[2 * i + 1]);
      *reinterpret_cast<uint2*>(base + 8 * c) =
          make_uint2((uint32_t)q[0] | ((uint32_t)q[1] << 16), (uint32_t)q[2] | ((uint32_t)q[3] << 16));
    }
    if (lane == 0) pool.scales[slot] = scale;
  } else {
    uint16_t* base = reinterpret_cast<uint16_t*>(pool.data) + slot * pool.dim;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      if (c >= nch) continue;
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = (uint32_t)float_to_bf16_bits(e[k][2 * i]) |
               ((uint32_t)float_to_bf16_bits(e[k][2 * i + 1]) << 16);
      *reinterpret_cast<uint4*>(base + 8 * c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// one window row: token first + u of sequence b, RoPE'd at its own position
template <int KC>
__device__ __forceinline__ void window_row(const CompressArgs& a, int b, int u, int lane, int nch) {
  const int s = a.seq_start[b];
  const int n = a.cu_seqlens[b + 1] - a.cu_seqlens[b];
  const int end = s + n;
  const int t = max(s, end - a.window_len) + u;
  if (t >= end) return;
  const int32_t* row = a.window.block_table + (size_t)b * a.window.max_blocks;
  const int blk = t / kLogicalBlock;
  if (blk >= a.window.max_blocks) {
    if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    return;
  }
  const int p = row[blk];
  if (p < 0) return;  // no page for this block: nothing to keep
  if (p >= a.window.num_pages) {
    if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_PAGE);
    return;
  }
  uint4 q[KC];
  load_row<KC>(a.x + (size_t)(a.cu_seqlens[b] + (t - s)) * a.dim, lane, nch, q);
  float e[KC][8];
#pragma unroll
  for (int k = 0; k < KC; ++k) unpack_bf16x8(q[k], e[k]);
  rope_warp<KC>(e, lane, nch, a.rope, (long long)t);
  store_entry_warp<KC>(a.window, (long long)p * kLogicalBlock + (t % kLogicalBlock), lane, nch, e);
}

// RMSNorm of one vector held by a warp: e * w / sqrt(mean(e^2) + eps)
template <int KC>
__device__ __forceinline__ void rms_norm_warp(float (&e)[KC][8], int lane, int nch, const float* w,
                                              float eps, int dim) {
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < KC; ++k)
    if (lane + 32 * k < nch)
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(e[k][i], e[k][i], ss);
  ss = warp_sum(ss);
  const float inv = __fdiv_rn(1.f, __fsqrt_rn(__fdiv_rn(ss, (float)dim) + eps));
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const int c = lane + 32 * k;
    if (c >= nch) continue;
    const float4 w0 = *reinterpret_cast<const float4*>(w + 8 * c);
    const float4 w1 = *reinterpret_cast<const float4*>(w + 8 * c + 4);
    const float ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) e[k][i] = e[k][i] * inv * ww[i];
  }
}

// slot of entry i (group t0 / r of sequence b): from the slot mapping, or
// (none passed) from the block table; -1 when there is nothing to store
// (an unmapped page, flagged by the slot mapping, or a bad slot, flagged here)
__device__ __forceinline__ long long entry_slot(const CompressArgs& a, int i, int b, int t0, int lane) {
  long long slot;
  if (a.slot_mapping) {
    slot = a.slot_mapping[i];
  } else {
    const long long g = t0 / a.ratio;
    const int p = page_of(a.main.block_table + (size_t)b * a.main.max_blocks, a.main.max_blocks, g,
                          a.main.spb, a.main.num_pages, lane == 0 ? a.dev_status : nullptr);
    slot = p < 0 ? -1 : (long long)p * a.main.spb + g % a.main.spb;
  }
  if (slot >= (long long)a.main.num_pages * a.main.spb) {
    if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    return -1;
  }
  return slot < 0 ? -1 : slot;
}

// RMSNorm (when weights are given), RoPE at the group's first position
// (rope_c, rope_s: rope_pair_lane at t0), optional pre-quantisation copy, and
// the store into `slot` (entry_slot)
template <int KC>
__device__ __forceinline__ void finish_entry(const CompressArgs& a, int i, int t0, int lane, int nch,
                                             float (&e)[KC][8], float rope_c, float rope_s,
                                             long long slot) {
  if (a.norm_w) rms_norm_warp<KC>(e, lane, nch, a.norm_w, a.norm_eps, a.dim);
  rope_warp<KC>(e, lane, nch, a.rope, (long long)t0, rope_c, rope_s);
  if (a.prequant_out) {
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      if (c >= nch) continue;
      float* po = a.prequant_out + (size_t)i * a.dim + 8 * c;
      *reinterpret_cast<float4*>(po) = make_float4(e[k][0], e[k][1], e[k][2], e[k][3]);
      *reinterpret_cast<float4*>(po + 4) = make_float4(e[k][4], e[k][5], e[k][6], e[k][7]);
    }
  }
  if (slot >= 0) store_entry_warp<KC>(a.main, slot, lane, nch, e);
}

// finish_entry with the slot and the rope values evaluated here
template <int KC>
__device__ __forceinline__ void finish_entry(const CompressArgs& a, int i, int b, int t0, int lane,
                                             int nch, float (&e)[KC][8]) {
  float c0 = 1.f, s0 = 0.f;
  if (a.rope.rope_dim) rope_pair_lane(a.rope, lane, (long long)t0, &c0, &s0);
  finish_entry<KC>(a, i, t0, lane, nch, e, c0, s0, entry_slot(a, i, b, t0, lane));
}

// state rows [lo, hi) of sequence b after this call: tokens gs + i of the
// unfinished group that arrived in this call (earlier ones are already there)
template <int KC, int RB>
__device__ __forceinline__ void copy_state(const CompressArgs& a, int b, int s, int end, int lo,
                                           int hi, int lane, int nch) {
  const int r = a.ratio;
  const int gs = (end / r) * r;
  lo = max(lo, s - gs);
  hi = min(hi, end - gs);
  for (int i = lo; i < hi; i += RB) {
    uint4 q[RB][KC];
#pragma unroll
    for (int j = 0; j < RB; ++j)
      if (i + j < hi) load_row<KC>(a.x + (size_t)(a.cu_seqlens[b] + (gs + i + j - s)) * a.dim, lane, nch, q[j]);
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      if (i + j >= hi) break;
      uint16_t* dst = a.state_x_out + ((size_t)b * r + (i + j)) * a.dim;
#pragma unroll
      for (int k = 0; k < KC; ++k)
        if (lane + 32 * k < nch) *reinterpret_cast<uint4*>(dst + 8 * (lane + 32 * k)) = q[j][k];
    }
  }
  for (int i = lo + lane; i < hi; i += 32)
    a.state_gate_out[(size_t)b * r + i] = a.gate[a.cu_seqlens[b] + (gs + i - s)];
}

// largest b with cu[b] <= i
__device__ __forceinline__ int seq_of(const int32_t* cu, int batch, int i) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The entry prefix sums of the call (entries touched per sequence), in cu_sh
// when they fit or are computed here (no slot mapping given); returns the
// array to use. All threads of the block call it.
__device__ __forceinline__ const int32_t* entry_prefix(const CompressArgs& a, int* cu_sh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool cached = a.batch + 1 <= kCuSmem;
  if (!a.cu_entries) {
    // no slot mapping given: the entry counts (groups touched by each
    // sequence's new tokens) and their prefix sums, computed here
    __shared__ int wsum[kWarps];
    int carry = 0;
    for (int base = 0; base < a.batch; base += kWarps * 32) {
      const int bb = base + threadIdx.x;
      int n = 0;
      if (bb < a.batch) {
        const int s0 = a.seq_start[bb], m = a.cu_seqlens[bb + 1] - a.cu_seqlens[bb];
        n = m > 0 ? (s0 + m + a.ratio - 1) / a.ratio - s0 / a.ratio : 0;
      }
      int x = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) wsum[warp] = x;
      __syncthreads();
      int before = carry;
      for (int w2 = 0; w2 < warp; ++w2) before += wsum[w2];
      if (bb < a.batch) cu_sh[bb] = before + x - n;
      for (int w2 = 0; w2 < kWarps; ++w2) carry += wsum[w2];
      __syncthreads();
    }
    if (threadIdx.x == 0) cu_sh[a.batch] = carry;
    __syncthreads();
    return cu_sh;
  }
  if (cached) {
    for (int k = threadIdx.x; k <= a.batch; k += blockDim.x) cu_sh[k] = a.cu_entries[k];
    __syncthreads();
    return cu_sh;
  }
  return a.cu_entries;
}

// cp.async of one 16-byte chunk into this thread's shared memory (cached in
// L2 only); the thread that copies a chunk is the one that reads it back,
// after cp_async_wait_all
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

constexpr int kGroupRows = 4;  // rows of a group on the warp-per-group path (ratio 4)

// Per-call tables in shared memory for the kernels with a compile-time ratio
// kR: the entry prefix sums (cu_sh, batch + 1 values) and, per sequence, its
// seq_start and cu_seqlens (meta_sh[b] = {seq_start[b], cu_seqlens[b]},
// meta_sh[batch].y = cu_seqlens[batch]). With batch <= 32 one warp builds
// them while the others wait at the barrier. Returns false when batch + 1 >
// kCuSmem: then the slot mapping's prefix sums and the global arrays serve.
template <int kR>
__device__ __forceinline__ bool seq_tables(const CompressArgs& a, int* cu_sh, int2* meta_sh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.batch + 1 > kCuSmem) return false;
  if (a.batch <= 32) {
    if (warp == 0) {
      int n = 0;
      if (lane < a.batch) {
        const int s0 = a.seq_start[lane], c0 = a.cu_seqlens[lane], c1 = a.cu_seqlens[lane + 1];
        const int m = c1 - c0;
        n = m > 0 ? (s0 + m + kR - 1) / kR - s0 / kR : 0;
        meta_sh[lane] = make_int2(s0, c0);
        if (lane == a.batch - 1) meta_sh[a.batch] = make_int2(0, c1);
      }
      if (a.cu_entries) {
        if (lane < a.batch) cu_sh[lane] = a.cu_entries[lane];
        if (lane == 0) cu_sh[a.batch] = a.cu_entries[a.batch];
      } else {
        int x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane < a.batch) cu_sh[lane] = x - n;
        if (lane == a.batch - 1) cu_sh[a.batch] = x;
      }
    }
    __syncthreads();
    return true;
  }
  for (int k = threadIdx.x; k <= a.batch; k += blockDim.x)
    meta_sh[k] = make_int2(k < a.batch ? a.seq_start[k] : 0, a.cu_seqlens[k]);
  if (a.cu_entries) {
    for (int k = threadIdx.x; k <= a.batch; k += blockDim.x) cu_sh[k] = a.cu_entries[k];
    __syncthreads();
    return true;
  }
  __shared__ int wsum[kWarps];
  int carry = 0;
  for (int base = 0; base < a.batch; base += kWarps * 32) {
    const int bb = base + threadIdx.x;
    int n = 0;
    if (bb < a.batch) {
      const int s0 = a.seq_start[bb], m = a.cu_seqlens[bb + 1] - a.cu_seqlens[bb];
      n = m > 0 ? (s0 + m + kR - 1) / kR - s0 / kR : 0;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int before = carry;
    for (int w2 = 0; w2 < warp; ++w2) before += wsum[w2];
    if (bb < a.batch) cu_sh[bb] = before + x - n;
    for (int w2 = 0; w2 < kWarps; ++w2) carry += wsum[w2];
    __syncthreads();
  }
  if (threadIdx.x == 0) cu_sh[a.batch] = carry;
  __syncthreads();
  return true;
}

// Ratio 4: one warp per group, eight groups per block; the leading blocks
// copy window rows. The group's rows go into the warp's shared memory with
// cp.async (lane l copies and later reads chunks l, l + 32, ...). Then, while
// they are in flight, the warp issues the loads of the gates, the position
// bias and the entry's block-table entry, evaluates the RoPE cos / sin at the
// group's position, and only then consumes the loads: the group costs one
// memory latency after the per-call tables. KC: 8-dim chunks per lane (dim <=
// 256 * KC); kFull: dim == 256 * KC (no partial chunk rows). Dynamic shared
// memory: kWarps * kGroupRows * KC * 512 B.
template <int KC, bool kFull>
__global__ void __launch_bounds__(kWarps * 32, KC <= 2 ? 4 : 2)
    compress_group_warp_kernel(CompressArgs a, int window_blocks, int window_blocks_per_seq) {
  constexpr int r = kGroupRows;
  constexpr int spb = kLogicalBlock / kGroupRows;  // entries per page
  extern __shared__ uint4 rows_sh[];  // [kWarps][kGroupRows][KC][32]
  __shared__ int cu_sh[kCuSmem];
  __shared__ int2 meta_sh[kCuSmem];
  tc::pdl_wait();  // the slot mapping (and whatever produced x) is complete from here on
  tc::pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = kFull ? 32 * KC : a.dim >> 3;
  if ((int)blockIdx.x < window_blocks) {
    window_row<KC>(a, blockIdx.x / window_blocks_per_seq,
                   (blockIdx.x % window_blocks_per_seq) * kWarps + warp, lane, nch);
    return;
  }
  const bool cached = seq_tables<r>(a, cu_sh, meta_sh);
  const int32_t* cu = cached ? cu_sh : a.cu_entries;
  const int total = cu[a.batch];
  const int i = (blockIdx.x - window_blocks) * kWarps + warp;
  if (i >= total) return;  // uniform over the warp
  const int b = seq_of(cu, a.batch, i);
  const int s = cached ? meta_sh[b].x : a.seq_start[b];
  const int c0 = cached ? meta_sh[b].y : a.cu_seqlens[b];
  const int end = s + ((cached ? meta_sh[b + 1].y : a.cu_seqlens[b + 1]) - c0);
  const int g = s / r + (i - cu[b]);  // the entry's group index in the sequence
  const int t0 = g * r;
  const int np = min(t0 + r, end) - t0;

  // 1. the rows, into shared memory
  uint4* stage = rows_sh + (size_t)warp * kGroupRows * KC * 32;
#pragma unroll
  for (int j = 0; j < kGroupRows; ++j) {
    if (j < np) {
      const int tt = t0 + j;
      const uint16_t* row = tt < s ? a.state_x + ((size_t)b * r + j) * a.dim
                                   : a.x + (size_t)(c0 + (tt - s)) * a.dim;
#pragma unroll
      for (int k = 0; k < KC; ++k)
        if (kFull || lane + 32 * k < nch)
          cp_async16(stage + (j * KC + k) * 32 + lane, row + 8 * (lane + 32 * k));
    }
  }
  // 2. gate, position bias and page loads, consumed after the RoPE values
  float gate = 0.f, bias = 0.f;
  if (lane < np) {
    const int tt = t0 + lane;
    gate = tt < s ? a.state_gate[(size_t)b * r + lane] : a.gate[c0 + (tt - s)];
    bias = a.pos_bias[lane];
  }
  const int blk = g / spb;
  long long slot = -1;
  int page = -1;
  if (a.slot_mapping) slot = a.slot_mapping[i];
  else if (blk < a.main.max_blocks) page = a.main.block_table[(size_t)b * a.main.max_blocks + blk];
  float rc = 1.f, rs = 0.f;
  if (a.rope.rope_dim) rope_pair_lane(a.rope, lane, (long long)t0, &rc, &rs);
  if (!a.slot_mapping) {
    if (blk >= a.main.max_blocks) {
      if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    } else if (page < 0 || page >= a.main.num_pages) {
      if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_PAGE);
    } else {
      slot = (long long)page * spb + g % spb;
    }
  }
  if (slot >= (long long)a.main.num_pages * spb) {
    if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    slot = -1;
  }
  // 3. the gate softmax over the np present tokens (lanes 0 .. 3, reduced
  // among themselves); lane j holds w[j]
  const float z = lane < np ? gate + bias : -INFINITY;
  float m = fmaxf(z, __shfl_xor_sync(0xffffffffu, z, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const float ez = lane < np ? expf(z - m) : 0.f;
  float sum = ez + __shfl_xor_sync(0xffffffffu, ez, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  const float wl = lane < np ? __fdiv_rn(ez, sum) : 0.f;

  float acc[KC][8];
#pragma unroll
  for (int k = 0; k < KC; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
  cp_async_wait_all();
#pragma unroll
  for (int j = 0; j < kGroupRows; ++j) {
    const float wt = __shfl_sync(0xffffffffu, wl, j);
    if (j >= np) break;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      if (!kFull && lane + 32 * k >= nch) continue;
      float v[8];
      unpack_bf16x8(stage[(j * KC + k) * 32 + lane], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(wt, v[e], acc[k][e]);
    }
  }
  finish_entry<KC>(a, i, t0, lane, nch, acc, rc, rs, slot);
  // this warp consumed every old state row and gate it read (the sums and
  // the softmax reductions depend on them), so the state may be rewritten
  if (i == cu[b]) copy_state<KC, kGroupRows>(a, b, s, end, 0, r, lane, nch);
}

// Ratio 128: one block per group; the leading blocks copy window rows. Warp
// w sums rows [16w, 16w + 16) of the group: the first eight go into its
// shared memory with cp.async, the other eight into registers, all sixteen
// requested at once, before the gate loads; warp 0 also issues the entry's
// block-table load and evaluates the RoPE cos / sin while they are in
// flight. The eight partial sums are added in warp order. KC: 8-dim chunks
// per lane (dim <= 256 * KC); kFull: dim == 256 * KC. Dynamic shared memory:
// kWarps * 8 * KC * 512 B.
constexpr int kBlockRatio = 128;
constexpr int kStagedRows = 8;  // rows per warp through shared memory (the rest in registers)

template <int KC, bool kFull>
__global__ void __launch_bounds__(kWarps * 32, KC <= 2 ? 2 : 1)
    compress_group_block_kernel(CompressArgs a, int window_blocks, int window_blocks_per_seq) {
  constexpr int r = kBlockRatio;
  constexpr int spb = kLogicalBlock / kBlockRatio;
  constexpr int rpw = r / kWarps;                 // 16 rows per warp
  constexpr int kRegRows = rpw - kStagedRows;     // 8
  constexpr int kNQ = r / 32;                     // gates per lane
  extern __shared__ uint4 rows_sh[];  // [kWarps][kStagedRows][KC][32]; then the partial sums
  __shared__ int cu_sh[kCuSmem];
  __shared__ int2 meta_sh[kCuSmem];
  tc::pdl_wait();  // the slot mapping (and whatever produced x) is complete from here on
  tc::pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = kFull ? 32 * KC : a.dim >> 3;
  if ((int)blockIdx.x < window_blocks) {
    window_row<KC>(a, blockIdx.x / window_blocks_per_seq,
                   (blockIdx.x % window_blocks_per_seq) * kWarps + warp, lane, nch);
    return;
  }
  const bool cached = seq_tables<r>(a, cu_sh, meta_sh);
  const int32_t* cu = cached ? cu_sh : a.cu_entries;
  const int total = cu[a.batch];
  const int i = blockIdx.x - window_blocks;
  if (i >= total) return;  // uniform over the block
  const int b = seq_of(cu, a.batch, i);
  const int s = cached ? meta_sh[b].x : a.seq_start[b];
  const int c0 = cached ? meta_sh[b].y : a.cu_seqlens[b];
  const int end = s + ((cached ? meta_sh[b + 1].y : a.cu_seqlens[b + 1]) - c0);
  const int g = s / r + (i - cu[b]);
  const int t0 = g * r;
  const int np = min(t0 + r, end) - t0;
  const int lo = min(np, warp * rpw), mid = min(np, lo + kStagedRows), hi = min(np, lo + rpw);

  // 1. this warp's rows: [lo, mid) into shared memory, [mid, hi) into registers
  uint4* stage = rows_sh + (size_t)warp * kStagedRows * KC * 32;
  auto row_ptr = [&](int j) {
    const int tt = t0 + j;
    return tt < s ? a.state_x + ((size_t)b * r + j) * a.dim : a.x + (size_t)(c0 + (tt - s)) * a.dim;
  };
  for (int j = lo; j < mid; ++j) {
    const uint16_t* row = row_ptr(j);
#pragma unroll
    for (int k = 0; k < KC; ++k)
      if (kFull || lane + 32 * k < nch)
        cp_async16(stage + ((j - lo) * KC + k) * 32 + lane, row + 8 * (lane + 32 * k));
  }
  uint4 q[kRegRows][KC];
#pragma unroll
  for (int j = 0; j < kRegRows; ++j)
    if (mid + j < hi) load_row<KC>(row_ptr(mid + j), lane, nch, q[j]);
  // 2. gates and position bias (every warp forms the whole softmax); warp 0:
  // the page and the RoPE values
  float gate[kNQ], bias[kNQ];
#pragma unroll
  for (int u = 0; u < kNQ; ++u) {
    const int t = lane + 32 * u;
    gate[u] = 0.f;
    bias[u] = 0.f;
    if (t < np) {
      const int tt = t0 + t;
      gate[u] = tt < s ? a.state_gate[(size_t)b * r + t] : a.gate[c0 + (tt - s)];
      bias[u] = a.pos_bias[t];
    }
  }
  long long slot = -1;
  float rc = 1.f, rs = 0.f;
  if (warp == 0) {
    const int blk = g / spb;
    int page = -1;
    if (a.slot_mapping) slot = a.slot_mapping[i];
    else if (blk < a.main.max_blocks) page = a.main.block_table[(size_t)b * a.main.max_blocks + blk];
    if (a.rope.rope_dim) rope_pair_lane(a.rope, lane, (long long)t0, &rc, &rs);
    if (!a.slot_mapping) {
      if (blk >= a.main.max_blocks) {
        if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
      } else if (page < 0 || page >= a.main.num_pages) {
        if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_PAGE);
      } else {
        slot = (long long)page * spb + g % spb;
      }
    }
    if (slot >= (long long)a.main.num_pages * spb) {
      if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
      slot = -1;
    }
  }
  // 3. softmax weights: w[t] held by lane t % 32 in wq[t / 32]
  float z[kNQ], m = -INFINITY;
#pragma unroll
  for (int u = 0; u < kNQ; ++u) {
    z[u] = lane + 32 * u < np ? gate[u] + bias[u] : -INFINITY;
    m = fmaxf(m, z[u]);
  }
  m = warp_max(m);
  float part_sum = 0.f;
#pragma unroll
  for (int u = 0; u < kNQ; ++u) {
    z[u] = lane + 32 * u < np ? expf(z[u] - m) : 0.f;
    part_sum += z[u];
  }
  const float sum = warp_sum(part_sum);
  float wq[kNQ];
#pragma unroll
  for (int u = 0; u < kNQ; ++u) wq[u] = __fdiv_rn(z[u], sum);
  auto weight = [&](int t) {  // t warp-uniform
    float v = wq[0];
#pragma unroll
    for (int u = 1; u < kNQ; ++u)
      if ((t >> 5) == u) v = wq[u];
    return __shfl_sync(0xffffffffu, v, t & 31);
  };

  float acc[KC][8];
#pragma unroll
  for (int k = 0; k < KC; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
  cp_async_wait_all();
  for (int j = lo; j < mid; ++j) {
    const float wt = weight(j);
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      if (!kFull && lane + 32 * k >= nch) continue;
      float v[8];
      unpack_bf16x8(stage[((j - lo) * KC + k) * 32 + lane], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(wt, v[e], acc[k][e]);
    }
  }
#pragma unroll
  for (int j = 0; j < kRegRows; ++j) {
    if (mid + j >= hi) break;
    const float wt = weight(mid + j);
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      float v[8];
      unpack_bf16x8(q[j][k], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(wt, v[e], acc[k][e]);
    }
  }
  __syncwarp();  // every lane has read its staged rows: the partial sum may overwrite them
  float* part = reinterpret_cast<float*>(stage);
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    float* p = part + 8 * (lane + 32 * k);
    *reinterpret_cast<float4*>(p) = make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(acc[k][4], acc[k][5], acc[k][6], acc[k][7]);
  }
  __syncthreads();  // partial sums in place; every read of the old state is done
  if (warp == 0) {
    constexpr int kWarpFloats = kStagedRows * KC * 32 * 4;
    const float* parts = reinterpret_cast<const float*>(rows_sh);
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int d = 8 * (lane + 32 * k);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float4 t = *reinterpret_cast<const float4*>(parts + d + 4 * h);
        for (int ww = 1; ww < kWarps; ++ww) {
          const float4 u = *reinterpret_cast<const float4*>(parts + ww * kWarpFloats + d + 4 * h);
          t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        acc[k][4 * h] = t.x; acc[k][4 * h + 1] = t.y; acc[k][4 * h + 2] = t.z; acc[k][4 * h + 3] = t.w;
      }
    }
    finish_entry<KC>(a, i, t0, lane, nch, acc, rc, rs, slot);
  }
  if (i == cu[b]) copy_state<KC, KC <= 2 ? 8 : 4>(a, b, s, end, warp * rpw, (warp + 1) * rpw, lane, nch);
}

// ---------------------------------------------------------------- variants
// c128a with per-channel gates: one block per entry. Token k of the entry's span (k = t - start, start =
// g*r, or g*r - r with the overlapping window) belongs to warp k / rpw, rpw =
// ceil(span / 8); for every dim the softmax over the present tokens runs in
// two passes through shared memory (the maxima, then the weighted sums, each
// warp over its tokens in ascending order, added in warp order), so the
// arithmetic depends only on a token's place in the span. Per-token gates are
// the case of one logit for all dims.

// logit of token tt (of sequence b, seq_start s) for dims 8c .. 8c + 7
__device__ __forceinline__ void gate_chunk(const CompressArgs& a, int b, int s, int old_base, int tt, int c,
                                           float (&z)[8]) {
  const int rows = a.state_rows;
  if (a.gate_dim == 1) {
    const float g = tt < s ? a.state_gate[(size_t)b * rows + (tt - old_base)]
                           : a.gate[a.cu_seqlens[b] + (tt - s)];
#pragma unroll
    for (int i = 0; i < 8; ++i) z[i] = g;
  } else {
    const float* row = tt < s ? a.state_gate + ((size_t)b * rows + (tt - old_base)) * a.dim
                              : a.gate + (size_t)(a.cu_seqlens[b] + (tt - s)) * a.dim;
    const float4 u = *reinterpret_cast<const float4*>(row + 8 * c);
    const float4 v = *reinterpret_cast<const float4*>(row + 8 * c + 4);
    z[0] = u.x; z[1] = u.y; z[2] = u.z; z[3] = u.w; z[4] = v.x; z[5] = v.y; z[6] = v.z; z[7] = v.w;
  }
}

template <int KC>
__device__ void variant_entry(const CompressArgs& a, int i, int b, const int32_t* cu, float* sh_m,
                              float* sh_s, float* sh_v) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = a.dim >> 3;
  const int r = a.ratio;
  const int s = a.seq_start[b];
  const int end = s + (a.cu_seqlens[b + 1] - a.cu_seqlens[b]);
  const int t0 = (s / r + (i - cu[b])) * r;
  const int span = a.overlap ? 2 * r : r;
  const int start = t0 - (a.overlap ? r : 0);
  const int lo = max(0, start), hi = min(t0 + r, end);
  const int old_base = (s / r) * r - (a.overlap ? r : 0);
  const int rpw = (span + kWarps - 1) / kWarps;
  const int k0 = max(warp * rpw, lo - start), k1 = min((warp + 1) * rpw, hi - start);
  // pass 1: this warp's maxima per dim
  float m[KC][8];
#pragma unroll
  for (int k = 0; k < KC; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) m[k][e] = -INFINITY;
  for (int kk = k0; kk < k1; ++kk) {
    const float bias = a.pos_bias[kk];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      if (c >= nch) continue;
      float z[8];
      gate_chunk(a, b, s, old_base, start + kk, c, z);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[k][e] = fmaxf(m[k][e], z[e] + bias);
    }
  }
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const int c = lane + 32 * k;
    if (c >= nch) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e) sh_m[warp * a.dim + 8 * c + e] = m[k][e];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const int c = lane + 32 * k;
    if (c >= nch) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float mm = -INFINITY;
      for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, sh_m[w * a.dim + 8 * c + e]);
      m[k][e] = mm;
    }
  }
  // pass 2: this warp's sums of exp(z - m) and of exp(z - m) * x per dim
  float su[KC][8], sv[KC][8];
#pragma unroll
  for (int k = 0; k < KC; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) su[k][e] = sv[k][e] = 0.f;
  for (int kk = k0; kk < k1; ++kk) {
    const int tt = start + kk;
    const float bias = a.pos_bias[kk];
    const uint16_t* xrow = tt < s ? a.state_x + ((size_t)b * a.state_rows + (tt - old_base)) * a.dim
                                  : a.x + (size_t)(a.cu_seqlens[b] + (tt - s)) * a.dim;
    uint4 q[KC];
    load_row<KC>(xrow, lane, nch, q);
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      if (c >= nch) continue;
      float z[8], x[8];
      gate_chunk(a, b, s, old_base, tt, c, z);
      unpack_bf16x8(q[k], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float u = expf(z[e] + bias - m[k][e]);
        su[k][e] += u;
        sv[k][e] = fmaf(u, x[e], sv[k][e]);
      }
    }
  }
  __syncthreads();  // every warp has read the maxima
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const int c = lane + 32 * k;
    if (c >= nch) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sh_s[warp * a.dim + 8 * c + e] = su[k][e];
      sh_v[warp * a.dim + 8 * c + e] = sv[k][e];
    }
  }
  __syncthreads();
  if (warp == 0) {
    float acc[KC][8];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float S = 0.f, V = 0.f;
        if (c < nch)
          for (int w = 0; w < kWarps; ++w) {
            S += sh_s[w * a.dim + 8 * c + e];
            V += sh_v[w * a.dim + 8 * c + e];
          }
        acc[k][e] = c < nch ? __fdiv_rn(V, S) : 0.f;
      }
    }
    finish_entry<KC>(a, i, b, t0, lane, nch, acc);
  }
  __syncthreads();  // the scratch is free again
}

// state rows after the call: the tokens [max(0, base), end), base = the last
// group start (minus r with the overlapping window), at row t - base; a token
// from before the call moves from its old row t - old_base >= t - base, so
// rows are copied in ascending order by one warp
template <int KC>
__device__ void variant_state(const CompressArgs& a, int b) {
  const int lane = threadIdx.x & 31;
  const int nch = a.dim >> 3;
  const int r = a.ratio;
  const int s = a.seq_start[b];
  const int end = s + (a.cu_seqlens[b + 1] - a.cu_seqlens[b]);
  const int ov = a.overlap ? r : 0;
  const int base = (end / r) * r - ov, old_base = (s / r) * r - ov;
  for (int tt = max(0, base); tt < end; ++tt) {
    const int row = tt - base;
    const uint16_t* src = tt < s ? a.state_x + ((size_t)b * a.state_rows + (tt - old_base)) * a.dim
                                 : a.x + (size_t)(a.cu_seqlens[b] + (tt - s)) * a.dim;
    uint4 q[KC];
    load_row<KC>(src, lane, nch, q);
    float gsc = 0.f;
    float4 gv[KC][2];
    if (a.gate_dim == 1) {
      gsc = tt < s ? a.state_gate[(size_t)b * a.state_rows + (tt - old_base)]
                   : a.gate[a.cu_seqlens[b] + (tt - s)];
    } else {
      const float* grow = tt < s ? a.state_gate + ((size_t)b * a.state_rows + (tt - old_base)) * a.dim
                                 : a.gate + (size_t)(a.cu_seqlens[b] + (tt - s)) * a.dim;
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        const int c = lane + 32 * k;
        if (c < nch) {
          gv[k][0] = *reinterpret_cast<const float4*>(grow + 8 * c);
          gv[k][1] = *reinterpret_cast<const float4*>(grow + 8 * c + 4);
        }
      }
    }
    __syncwarp();  // every lane has read the source row before it is overwritten
    uint16_t* dst = a.state_x_out + ((size_t)b * a.state_rows + row) * a.dim;
#pragma unroll
    for (int k = 0; k < KC; ++k)
      if (lane + 32 * k < nch) *reinterpret_cast<uint4*>(dst + 8 * (lane + 32 * k)) = q[k];
    if (a.gate_dim == 1) {
      if (lane == 0) a.state_gate_out[(size_t)b * a.state_rows + row] = gsc;
    } else {
      float* gdst = a.state_gate_out + ((size_t)b * a.state_rows + row) * a.dim;
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        const int c = lane + 32 * k;
        if (c < nch) {
          *reinterpret_cast<float4*>(gdst + 8 * c) = gv[k][0];
          *reinterpret_cast<float4*>(gdst + 8 * c + 4) = gv[k][1];
        }
      }
    }
    __syncwarp();
  }
}

template <int KC>
__global__ void __launch_bounds__(kWarps * 32) compress_variant_kernel(CompressArgs a, int window_blocks,
                                                                      int window_blocks_per_seq) {
  extern __shared__ float vsm[];  // 3 x kWarps x dim: maxima, sums, weighted sums
  __shared__ int cu_sh[kCuSmem];
  tc::pdl_wait();  // x, the gates and the state (earlier work in the stream) are complete
  tc::pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = a.dim >> 3;
  if ((int)blockIdx.x < window_blocks) {
    window_row<KC>(a, blockIdx.x / window_blocks_per_seq,
                   (blockIdx.x % window_blocks_per_seq) * kWarps + warp, lane, nch);
    return;
  }
  const int32_t* cu = entry_prefix(a, cu_sh);
  const int i = blockIdx.x - window_blocks;
  if (i >= cu[a.batch]) return;
  const int b = seq_of(cu, a.batch, i);
  // The old state is read by the sequence's first entry of the call, and with
  // the overlapping window also by its second: one block builds both and then
  // rewrites the state.
  if (a.overlap && i == cu[b] + 1) return;
  float* sh_m = vsm;
  float* sh_s = vsm + kWarps * a.dim;
  float* sh_v = vsm + 2 * kWarps * a.dim;
  variant_entry<KC>(a, i, b, cu, sh_m, sh_s, sh_v);
  if (i == cu[b]) {
    if (a.overlap && i + 1 < cu[b + 1]) variant_entry<KC>(a, i + 1, b, cu, sh_m, sh_s, sh_v);
    if (warp == 0) variant_state<KC>(a, b);
  }
}


// c4a variants, one warp per entry. The span's rows (4 tokens, or 8 with the
// overlapping window) go into the warp's shared memory with cp.async (lane l
// copies and later reads chunks l, l + 32, ...); with per-token gates the
// gate, bias and block-table loads and the RoPE cos / sin are issued while the
// rows are in flight. Per-token gates: the weights once per token (lane t),
// added in ascending t; per-channel gates: per dim, the maximum over the
// tokens, then the sums of exp(z - m) and of exp(z - m) * x in ascending t.
constexpr int kVariantSpan = 2 * kGroupRows;

__host__ __device__ inline size_t variant_warp_smem(int kc, int batch) {
  const size_t tables = batch + 1 <= kCuSmem ? (size_t)((batch + 4) & ~3) * 4 + (size_t)(batch + 1) * 8 : 0;
  return (size_t)kWarps * kVariantSpan * kc * 32 * 16 + tables;
}

template <int KC, bool kFull>
__device__ void warp_variant_entry(const CompressArgs& a, int i, int b, const int32_t* cu,
                                   const int2* meta, uint4* stage) {
  constexpr int r = kGroupRows;
  constexpr int spb = kLogicalBlock / kGroupRows;
  const int lane = threadIdx.x & 31;
  const int nch = kFull ? 32 * KC : a.dim >> 3;
  const int s = meta ? meta[b].x : a.seq_start[b];
  const int c0 = meta ? meta[b].y : a.cu_seqlens[b];
  const int end = s + ((meta ? meta[b + 1].y : a.cu_seqlens[b + 1]) - c0);
  const int g = s / r + (i - cu[b]);
  const int t0 = g * r;
  const int start = t0 - (a.overlap ? r : 0);
  const int lo = max(0, start), hi = min(t0 + r, end);
  const int np = hi - lo, k0 = lo - start;
  const int old_base = (s / r) * r - (a.overlap ? r : 0);
#pragma unroll
  for (int j = 0; j < kVariantSpan; ++j) {
    if (j < np) {
      const int tt = lo + j;
      const uint16_t* row = tt < s ? a.state_x + ((size_t)b * a.state_rows + (tt - old_base)) * a.dim
                                   : a.x + (size_t)(c0 + (tt - s)) * a.dim;
#pragma unroll
      for (int k = 0; k < KC; ++k)
        if (kFull || lane + 32 * k < nch) cp_async16(stage + (j * KC + k) * 32 + lane, row + 8 * (lane + 32 * k));
    }
  }
  // per-token gates: lane t < np holds token lo + t's logit and bias
  float gate = 0.f, bias = 0.f;
  if (a.gate_dim == 1 && lane < np) {
    const int tt = lo + lane;
    gate = tt < s ? a.state_gate[(size_t)b * a.state_rows + (tt - old_base)] : a.gate[c0 + (tt - s)];
    bias = a.pos_bias[k0 + lane];
  }
  long long slot = -1;
  int page = -1;
  if (a.slot_mapping) slot = a.slot_mapping[i];
  else if (g / spb < a.main.max_blocks) page = a.main.block_table[(size_t)b * a.main.max_blocks + g / spb];
  float rc = 1.f, rs = 0.f;
  if (a.rope.rope_dim) rope_pair_lane(a.rope, lane, (long long)t0, &rc, &rs);
  if (!a.slot_mapping) {
    if (g / spb >= a.main.max_blocks) {
      if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    } else if (page < 0 || page >= a.main.num_pages) {
      if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_PAGE);
    } else {
      slot = (long long)page * spb + g % spb;
    }
  }
  if (slot >= (long long)a.main.num_pages * spb) {
    if (lane == 0) flag(a.dev_status, V4KV_DEV_BAD_SLOT);
    slot = -1;
  }
  float acc[KC][8];
  if (a.gate_dim == 1) {
    const float z = lane < np ? gate + bias : -INFINITY;
    const float m = warp_max(z);
    const float u = lane < np ? expf(z - m) : 0.f;
    const float sum = warp_sum(u);
    const float w = lane < np ? __fdiv_rn(u, sum) : 0.f;
#pragma unroll
    for (int k = 0; k < KC; ++k)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
    cp_async_wait_all();
#pragma unroll
    for (int j = 0; j < kVariantSpan; ++j) {
      const float wt = __shfl_sync(0xffffffffu, w, j);
      if (j >= np) break;
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        if (!kFull && lane + 32 * k >= nch) continue;
        float v[8];
        unpack_bf16x8(stage[(j * KC + k) * 32 + lane], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(wt, v[e], acc[k][e]);
      }
    }
  } else {
    cp_async_wait_all();
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      float m[8], su[8], sv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        m[e] = -INFINITY;
        su[e] = sv[e] = 0.f;
      }
      if (kFull || c < nch) {
#pragma unroll
        for (int j = 0; j < kVariantSpan; ++j) {
          if (j >= np) break;
          float z[8];
          gate_chunk(a, b, s, old_base, lo + j, c, z);
          const float bj = a.pos_bias[k0 + j];
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], z[e] + bj);
        }
#pragma unroll
        for (int j = 0; j < kVariantSpan; ++j) {
          if (j >= np) break;
          float z[8], v[8];
          gate_chunk(a, b, s, old_base, lo + j, c, z);
          unpack_bf16x8(stage[(j * KC + k) * 32 + lane], v);
          const float bj = a.pos_bias[k0 + j];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float u = expf(z[e] + bj - m[e]);
            su[e] += u;
            sv[e] = fmaf(u, v[e], sv[e]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] = (kFull || c < nch) ? __fdiv_rn(sv[e], su[e]) : 0.f;
    }
  }
  __syncwarp();  // every lane has read its rows before the stage is reused
  finish_entry<KC>(a, i, t0, lane, nch, acc, rc, rs, slot);
}

template <int KC, bool kFull>
__global__ void __launch_bounds__(kWarps * 32, KC <= 2 ? 3 : 1)
    compress_variant_warp_kernel(CompressArgs a, int window_blocks, int window_blocks_per_seq) {
  extern __shared__ uint4 dyn_sh[];  // [kWarps][kVariantSpan][KC][32], then the tables
  int* cu_sh = reinterpret_cast<int*>(dyn_sh + kWarps * kVariantSpan * KC * 32);
  int2* meta_sh = reinterpret_cast<int2*>(cu_sh + ((a.batch + 4) & ~3));
  tc::pdl_wait();  // x, the gates and the state (earlier work in the stream) are complete
  tc::pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = kFull ? 32 * KC : a.dim >> 3;
  if ((int)blockIdx.x < window_blocks) {
    window_row<KC>(a, blockIdx.x / window_blocks_per_seq,
                   (blockIdx.x % window_blocks_per_seq) * kWarps + warp, lane, nch);
    return;
  }
  const bool cached = seq_tables<kGroupRows>(a, cu_sh, meta_sh);
  const int32_t* cu = cached ? cu_sh : a.cu_entries;
  const int2* meta = cached ? meta_sh : nullptr;
  const int i = (blockIdx.x - window_blocks) * kWarps + warp;
  if (i >= cu[a.batch]) return;  // uniform over the warp
  const int b = seq_of(cu, a.batch, i);
  // the warp of the sequence's first entry also builds the second (both read
  // the old state with the overlapping window) and then rewrites the state
  if (a.overlap && i == cu[b] + 1) return;
  uint4* stage = dyn_sh + (size_t)warp * kVariantSpan * KC * 32;
  warp_variant_entry<KC, kFull>(a, i, b, cu, meta, stage);
  if (i == cu[b]) {
    if (a.overlap && i + 1 < cu[b + 1]) warp_variant_entry<KC, kFull>(a, i + 1, b, cu, meta, stage);
    variant_state<KC>(a, b);
  }
}

template <int KC>
cudaError_t launch_variant_kc(const CompressArgs& a, int max_groups, int window_blocks, int per_seq,
                              cudaStream_t stream) {
  if (a.ratio == kGroupRows) {  // c4a: one warp per entry
    const size_t smem = variant_warp_smem(KC, a.batch);
    cudaError_t e = cudaFuncSetAttribute(compress_variant_warp_kernel<KC, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(compress_variant_warp_kernel<KC, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(window_blocks + (max_groups + kWarps - 1) / kWarps), block(kWarps * 32);
    if (a.dim == 256 * KC)
      return launch_pdl(compress_variant_warp_kernel<KC, true>, grid, block, smem, stream, a, window_blocks,
                        per_seq);
    return launch_pdl(compress_variant_warp_kernel<KC, false>, grid, block, smem, stream, a, window_blocks,
                      per_seq);
  }
  const size_t smem = (size_t)3 * kWarps * a.dim * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(compress_variant_kernel<KC>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(compress_variant_kernel<KC>, dim3(window_blocks + max_groups), dim3(kWarps * 32),
                    smem, stream, a, window_blocks, per_seq);
}

template <int KC>
cudaError_t launch_kc(const CompressArgs& a, int max_groups, int window_blocks, int per_seq,
                      cudaStream_t stream) {
  if (a.ratio != kGroupRows) {
    if (a.ratio != kBlockRatio) return cudaErrorInvalidValue;
    const dim3 grid(window_blocks + max_groups), block(kWarps * 32);
    // with the static arrays (12 KB) the total passes 48 KB: opt in
    const size_t smem = (size_t)kWarps * kStagedRows * KC * 32 * sizeof(uint4);
    cudaError_t e = cudaFuncSetAttribute(compress_group_block_kernel<KC, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(compress_group_block_kernel<KC, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (a.dim == 256 * KC)
      return launch_pdl(compress_group_block_kernel<KC, true>, grid, block, smem, stream, a, window_blocks,
                        per_seq);
    return launch_pdl(compress_group_block_kernel<KC, false>, grid, block, smem, stream, a, window_blocks,
                      per_seq);
  }
  const dim3 grid(window_blocks + (max_groups + kWarps - 1) / kWarps), block(kWarps * 32);
  const size_t smem = (size_t)kWarps * kGroupRows * KC * 32 * sizeof(uint4);
  if (smem > 32 * 1024) {  // with the static arrays (12 KB) past 48 KB: opt in
    cudaError_t e = cudaFuncSetAttribute(compress_group_warp_kernel<KC, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(compress_group_warp_kernel<KC, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (a.dim == 256 * KC)
    return launch_pdl(compress_group_warp_kernel<KC, true>, grid, block, smem, stream, a, window_blocks,
                      per_seq);
  return launch_pdl(compress_group_warp_kernel<KC, false>, grid, block, smem, stream, a, window_blocks,
                    per_seq);
}


// ---------------------------------------------------------------- Q/K preparation
// The decode step's query heads and new window row in one launch, one warp per
// item (horizontal fusion): warp j < heads RMS-normalises head j of sequence b
// (when weights are given) and rotates it by RoPE at positions[b]; warp j ==
// heads rotates the new K = V row and stores it in the window (bf16, or fp8
// per token), the same arithmetic as the compressor's window rows.
template <int KC>
__global__ void __launch_bounds__(kWarps * 32) qk_prepare_kernel(QkPrepArgs p) {
  tc::pdl_wait();  // q and the new rows (earlier work in the stream) are complete
  tc::pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x, j = blockIdx.y * kWarps + warp;
  const int nch = p.dim >> 3;
  const long long pos = p.positions[b];
  if (j < p.heads) {
    const float* src = p.q_in + ((size_t)b * p.heads + j) * p.dim;
    float e[KC][8];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
#pragma unroll
      for (int i = 0; i < 8; ++i) e[k][i] = 0.f;
      if (c < nch) {
        const float4 u = *reinterpret_cast<const float4*>(src + 8 * c);
        const float4 v = *reinterpret_cast<const float4*>(src + 8 * c + 4);
        e[k][0] = u.x; e[k][1] = u.y; e[k][2] = u.z; e[k][3] = u.w;
        e[k][4] = v.x; e[k][5] = v.y; e[k][6] = v.z; e[k][7] = v.w;
      }
    }
    if (p.norm_w) rms_norm_warp<KC>(e, lane, nch, p.norm_w, p.norm_eps, p.dim);
    rope_warp<KC>(e, lane, nch, p.rope, pos);
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      if (c >= nch) continue;
      const size_t o = ((size_t)b * p.heads + j) * p.dim + 8 * c;
      if (p.q_out_bf16) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = (uint32_t)float_to_bf16_bits(e[k][2 * i]) | ((uint32_t)float_to_bf16_bits(e[k][2 * i + 1]) << 16);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.q_out) + o) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        float* dst = static_cast<float*>(p.q_out) + o;
        *reinterpret_cast<float4*>(dst) = make_float4(e[k][0], e[k][1], e[k][2], e[k][3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(e[k][4], e[k][5], e[k][6], e[k][7]);
      }
    }
  } else if (j == p.heads && p.k_new && p.window.data) {
    const int32_t* row = p.window.block_table + (size_t)b * p.window.max_blocks;
    const long long blk = pos / kLogicalBlock;
    if (pos < 0 || blk >= p.window.max_blocks) {
      if (lane == 0) flag(p.dev_status, V4KV_DEV_BAD_SLOT);
      return;
    }
    const int pg = row[blk];
    if (pg < 0) return;  // no page for this block: nothing to keep
    if (pg >= p.window.num_pages) {
      if (lane == 0) flag(p.dev_status, V4KV_DEV_BAD_PAGE);
      return;
    }
    uint4 q[KC];
    load_row<KC>(p.k_new + (size_t)b * p.dim, lane, nch, q);
    float e[KC][8];
#pragma unroll
    for (int k = 0; k < KC; ++k) unpack_bf16x8(q[k], e[k]);
    rope_warp<KC>(e, lane, nch, p.rope, pos);
    store_entry_warp<KC>(p.window, (long long)pg * kLogicalBlock + (pos % kLogicalBlock), lane, nch, e);
  }
}
}  // namespace

cudaError_t launch_compress_append(const CompressArgs& a, int max_groups, int total_tokens,
                                   cudaStream_t stream) {
  if (a.ratio > kMaxRatio) return cudaErrorInvalidValue;
  // window rows: per sequence the last min(n, W) new tokens, W <= total new tokens
  int per_seq = 0;
  if (a.window.data && a.window_len > 0 && total_tokens > 0)
    per_seq = (min(a.window_len, total_tokens) + kWarps - 1) / kWarps;
  const long long wb = (long long)per_seq * a.batch;
  if (wb + max_groups > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (wb + max_groups == 0) return cudaSuccess;
  const int kc = (a.dim + 255) / 256;
  if (a.overlap || a.gate_dim != 1) {
    // the variant kernel (one block per entry); RMSNorm alone runs in the
    // regular kernels
    if (kc <= 1) return launch_variant_kc<1>(a, max_groups, (int)wb, per_seq, stream);
    if (kc <= 2) return launch_variant_kc<2>(a, max_groups, (int)wb, per_seq, stream);
    return launch_variant_kc<4>(a, max_groups, (int)wb, per_seq, stream);
  }
  if (kc <= 1) return launch_kc<1>(a, max_groups, (int)wb, per_seq, stream);
  if (kc <= 2) return launch_kc<2>(a, max_groups, (int)wb, per_seq, stream);
  return launch_kc<4>(a, max_groups, (int)wb, per_seq, stream);
}

}  // namespace v4kv

namespace v4kv {

cudaError_t launch_qk_prepare(const QkPrepArgs& p, cudaStream_t stream) {
  const dim3 grid(p.batch, (p.heads + 1 + kWarps - 1) / kWarps), block(kWarps * 32);
  const int kc = (p.dim + 255) / 256;
  if (kc <= 1) return launch_pdl(qk_prepare_kernel<1>, grid, block, 0, stream, p);
  if (kc <= 2) return launch_pdl(qk_prepare_kernel<2>, grid, block, 0, stream, p);
  return launch_pdl(qk_prepare_kernel<4>, grid, block, 0, stream, p);
}

}  // namespace v4kv
