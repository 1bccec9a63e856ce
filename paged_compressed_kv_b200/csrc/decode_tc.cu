// Decode attention on the tcgen05 tensor cores for 64 query heads sharing one
// K = V vector per item (P1 §2.1: shared K/V; §2.3: raw-token window).
//
// Per tile of 128 items (entries or window tokens) of one sequence:
//   S^T[128 x 64] = V[128 x 512] . Q^T          (M = items, N = heads, K = dims)
//   P' = 2^(S^T * c_j + log2 ks_j - m_h)        (CUDA cores, one thread per item)
//   O^T[512 x 64] += V^T[512 x 128] . P'^T      (M = dims in 4 tiles of 128)
// V sits once in shared memory as f16 in 128-byte-swizzled atoms; it is the
// K-major A operand of the first product and the MN-major A operand of the
// second. fp8 codes convert to f16 exactly; the entry's fp32 scale ks_j enters
// the score multiplier c_j and, through log2 ks_j, the exponent, so P' is the
// weight of the raw code vector. The normaliser is sum_j P'_hj / ks_j.
// q is scaled per sequence by a power of two into f16 range. m_h is a
// reference maximum per head, raised only when a score exceeds it by more
// than 2^8 (P' <= 256), at which point O^T and the partial sums are rescaled.
//
// Warp roles (352 threads): warps 0-7 are workers. Each runs the softmax of
// one tile row (its TMEM lane) for 32 of the 64 heads, then gathers and
// converts 16 rows of the next tile (16-byte coalesced page loads) as the
// second product releases each V chunk. Warp 8 allocates tensor memory and
// one of its threads issues the MMAs; warps 9 and 10 resolve the rows of the
// even and odd tiles up to kRing - 1 ahead and prefetch them into L2. The
// partial normalisers of each row (one per head) live in tensor memory.
//
// Schedule: the kernel is persistent. The tiles of all sequences form one
// list (each sequence: its entries padded to whole tiles, then its window);
// the prep kernel gives block c of G the range of tiles where the estimated
// cost prefix runs from c/G to (c+1)/G of the total, or, when every sequence
// fits one block cheaply, sequence c whole. A block writes one partial result
// (O, m, l) per sequence it touches into slot b + c, which is unique because
// b + c increases strictly along the tile list; the merge kernel combines the
// slots of each sequence. A block that runs every tile of a sequence writes
// that sequence's output itself and the merge skips it.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace v4kv {

namespace {

constexpr int kH = 64;          // heads (MMA N)
constexpr int kD = 512;         // dims
constexpr int kT = 128;         // items per tile (MMA M of the first product)
constexpr int kThreads = 352;
constexpr float kTau = 8.f;     // rescale when a score exceeds the reference by 2^8
constexpr float kNone = -1e30f; // reference maximum before any item

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kVOff = 0;                    // 8 dim atoms x 128 rows x 128 B
constexpr uint32_t kQOff = 131072;               // 8 dim atoms x 64 rows x 128 B
constexpr uint32_t kPOff = 196608;               // 128 rows x 128 B (64 heads f16)
constexpr int kRing = 6;        // tiles of row addresses the address warp keeps ready
constexpr uint32_t kMetaOff = 212992;                 // [kRing][128] fp32 item scales
constexpr uint32_t kPtrOff = kMetaOff + kRing * 512;  // [kRing][128] item row addresses (null = skip)
constexpr uint32_t kMrefOff = kPtrOff + kRing * 1024;  // [64] reference max per head
constexpr uint32_t kAlphaOff = kMrefOff + 256;   // [64] rescale factors
constexpr uint32_t kRedOff = kAlphaOff + 256;    // [8][32] per-warp reductions
constexpr uint32_t kBarOff = kRedOff + 1024;     // mbarriers
constexpr uint32_t kInfoOff = kBarOff + 256;     // [kRing] tile info words
constexpr uint32_t kMiscOff = kInfoOff + 64;     // tmem address, flags, range
constexpr uint32_t kSmemBytes = kMiscOff + 64 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per block");

// TMEM columns: S double buffer [0, 128), O^T 4 x 64 at [128, 384), partial
// normalisers of each lane (64 heads) at [384, 448)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 128;
constexpr uint32_t kLCol = 384;

struct Bars {
  uint64_t addr_ready[kRing];
  uint64_t addr_free[kRing];
  uint64_t v_full[4];
  uint64_t v_empty[4];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t q_ready;
  uint64_t drain;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

// tile info word written by the address warp
constexpr uint32_t kInfoFp8 = 1;    // rows are fp8 codes (else bf16)
constexpr uint32_t kInfoFirst = 2;  // first tile of a segment (new sequence)

// 2^x on the special-function unit (ftz: results below 2^-126 become 0)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_and(int id, int n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, %2, %3, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool named_or(int id, int n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, %2, %3, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

struct Seq {
  int L, n_sel, n_sel_pad, n_win, w0, n_items;
};

// the tile plan of a sequence of length L (already clamped to [0, max_len])
__device__ __forceinline__ Seq seq_from_len(const DecodeArgs& a, int L) {
  Seq s;
  s.L = L;
  const int n_vis = max(0, s.L - a.window_len) / a.ratio;
  s.n_sel = a.topk ? a.k : n_vis;
  s.n_sel_pad = (s.n_sel + kT - 1) / kT * kT;
  s.w0 = max(0, s.L - a.window_len);
  s.n_win = s.L - s.w0;
  s.n_items = s.n_sel_pad + s.n_win;
  return s;
}

__device__ __forceinline__ Seq seq_of(const DecodeArgs& a, int b, int32_t* st) {
  int L = a.seq_lens[b];
  if (L > a.max_len) {
    if (threadIdx.x == 0) flag(st, V4KV_DEV_OVERFLOW);
    L = a.max_len;
  }
  return seq_from_len(a, max(0, L));
}

// one bulk L2 prefetch of `bytes` (a multiple of 16, 16-byte aligned) through
// the copy engine
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Address warp: lane l resolves rows l, l+32, l+64, l+96 of the tile that
// starts at item tile0 into the row-address and scale tables (nullptr / 0 for
// a skipped item). The loads go in phases (top-k indices, block-table
// entries, scales), each phase's four loads independent of one another, so a
// tile costs three memory latencies rather than twelve. Problems are flagged
// as V4KV_DEV_* bits.
__device__ __forceinline__ void resolve_tile(const DecodeArgs& a, int b, const Seq& s, int tile0,
                                             int lane, const uint8_t** rp, float* ms) {
  const bool main_tile = tile0 < s.n_sel_pad;  // a tile is all entries or all window
  const int spb = main_tile ? a.main.spb : a.window.spb;
  const int max_blocks = main_tile ? a.main.max_blocks : a.window.max_blocks;
  const int num_pages = main_tile ? a.main.num_pages : a.window.num_pages;
  const int32_t* bt = (main_tile ? a.main.block_table : a.window.block_table) + (size_t)b * max_blocks;
  const bool fp8 = (main_tile ? a.main.dtype : a.window.dtype) == V4KV_FP8_E4M3;
  const float* scales = main_tile ? a.main.scales : a.window.scales;
  const uint8_t* data = reinterpret_cast<const uint8_t*>(main_tile ? a.main.data : a.window.data);
  const long long n_stored = ((long long)s.L + a.ratio - 1) / a.ratio;
  int err = 0;
  // phase 1: item indices (top-k entries are read from the selection)
  long long j[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int it = tile0 + lane + 32 * r;
    j[r] = -1;
    if (main_tile) {
      if (it < s.n_sel) j[r] = a.topk ? (long long)a.topk[(size_t)b * a.k + it] : (long long)it;
    } else {
      const int w = it - s.n_sel_pad;
      if (w < s.n_win) j[r] = s.w0 + w;
    }
  }
  // phase 2: block-table entries
  int pg[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    pg[r] = -1;
    if (j[r] < 0) continue;
    if (main_tile && j[r] >= n_stored) {
      err |= V4KV_DEV_BAD_INDEX;
      j[r] = -1;
      continue;
    }
    const long long blk = j[r] / spb;
    if (blk >= max_blocks) {
      err |= V4KV_DEV_BAD_SLOT;
      j[r] = -1;
      continue;
    }
    pg[r] = bt[blk];
  }
  // phase 3: slots, scales, row addresses
  const uint8_t* p[4];
  float ks[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    p[r] = nullptr;
    ks[r] = 0.f;
    if (j[r] < 0) continue;
    if (pg[r] < 0 || pg[r] >= num_pages) {
      err |= V4KV_DEV_BAD_PAGE;
      continue;
    }
    const long long slot = (long long)pg[r] * spb + j[r] % spb;
    ks[r] = fp8 ? scales[slot] : 1.f;
    p[r] = data + slot * (fp8 ? kD : 2 * kD);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    rp[lane + 32 * r] = p[r];
    ms[lane + 32 * r] = ks[r];
  }
  if (err) flag(a.dev_status, err);
}

__device__ __forceinline__ uint4 ldg_stream(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// 16 fp8 codes -> 16 f16 values as two 16-byte halves
__device__ __forceinline__ void fp8x16_to_f16(uint4 raw, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = h2u(e4m3x2_to_half2((uint16_t)(w[i] & 0xffffu)));
    o[2 * i + 1] = h2u(e4m3x2_to_half2((uint16_t)(w[i] >> 16)));
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 8 bf16 -> 8 f16 (round to nearest, saturating to the f16 range). `wide`
// is set when a value's magnitude is 2^16 or more (or not finite): such a
// value does not fit the f16 operands of the tensor cores and is clamped.
__device__ __forceinline__ uint4 bf16x8_to_f16(uint4 raw, bool& wide) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    wide |= (w[i] & 0x7fffu) >= 0x4780u || ((w[i] >> 16) & 0x7fffu) >= 0x4780u;
    const float a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xffff0000u);
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    o[i] = r;
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}


__device__ __forceinline__ int tiles_of(const Seq& s) {
  return s.n_sel_pad / kT + (s.n_win + kT - 1) / kT;
}

// Estimated cost of a sequence's tiles in the sweep (units of a quarter of an
// fp8 tile): fp8 tiles 4, bf16 tiles 8 (twice the bytes and a slower
// conversion), and 4 for opening a segment (query copy, epilogue).
constexpr int kCostFp8 = 4, kCostBf16 = 8, kCostSeg = 4;
// estimated cost of splitting a sequence over blocks: the partial results'
// stores and the merge (about three fp8 tiles)
constexpr int kCostMerge = 12;

__device__ __forceinline__ long long seq_cost(const DecodeArgs& a, const Seq& s) {
  const int nm = s.n_sel_pad / kT, nw = (s.n_win + kT - 1) / kT;
  if (nm + nw == 0) return 0;
  const int cm = a.main.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  const int cw = a.window.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  return kCostSeg + (long long)nm * cm + (long long)nw * cw;
}

// tile of sequence s at which `off` cost units (from the sequence's start)
// fall, clamped to the sequence's tiles
__device__ __forceinline__ int tile_at_cost(const DecodeArgs& a, const Seq& s, long long off) {
  const int nm = s.n_sel_pad / kT, nw = (s.n_win + kT - 1) / kT;
  const int cm = a.main.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  const int cw = a.window.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  off -= kCostSeg;
  if (off <= 0) return 0;
  if (off < (long long)nm * cm) return (int)(off / cm);
  const long long k = nm + (off - (long long)nm * cm) / cw;
  return (int)min(k, (long long)(nm + nw - 1));
}

// Walks the global tile list: sequence b, tile lt of nt in that sequence.
struct Cursor {
  int b, lt, nt;
  Seq s;
};

__device__ __forceinline__ void cursor_set(Cursor& c, const DecodeArgs& a, int b, int lt, int L) {
  c.b = b;
  c.lt = lt;
  c.s = seq_from_len(a, L);
  c.nt = tiles_of(c.s);
}

__device__ __forceinline__ void cursor_next(Cursor& c, const DecodeArgs& a) {
  ++c.lt;
  while (c.lt >= c.nt && c.b + 1 < a.batch) {
    ++c.b;
    c.lt = 0;
    c.s = seq_of(a, c.b, nullptr);
    c.nt = tiles_of(c.s);
  }
}

constexpr uint32_t kQBytes = kH * kD * 2;  // one query image (f16)
constexpr int kMaxSplits = 160;            // sweep blocks at most (the plan caps the grid)
constexpr int kMergeWarps = 4;             // heads per merge block (a warp each)
constexpr int kPrepCache = 2048;           // batches whose prefix sums the prep keeps in shared memory

// Start the bulk copy of sequence b's query image into shared memory; the
// copy completes phase by transaction count on `bar`.
__device__ __forceinline__ void issue_q(const DecodeArgs& a, int b, uint32_t qdst, uint64_t* bar) {
  tc::mbar_arrive_expect_tx(bar, kQBytes);
  const uint8_t* src = a.qh + (size_t)b * kQBytes;
#pragma unroll
  for (int k = 0; k < 4; ++k) tc::bulk_load(qdst + k * (kQBytes / 4), src + k * (kQBytes / 4), kQBytes / 4, bar);
}

// Sum (or maximum, kMax) of 32 per-lane values over the 32 lanes of a warp
// (reduce-scatter): lane l ends with the result for the value whose index the
// lane bits pick (bit 4: the upper 16 values, bit 3: 8, ... bit 0: 1), and
// returns that index. 31 shuffles per lane.
template <bool kMax>
__device__ __forceinline__ int warp_reduce_scatter32(float* v, int lane, float* out1) {
  int base = 0;
#pragma unroll
  for (int level = 0; level < 5; ++level) {
    const int off = 16 >> level;   // shuffle distance
    const int n = 16 >> level;     // values kept after this level
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < n; ++k) {
      const float mine = upper ? v[n + k] : v[k];
      const float other = upper ? v[k] : v[n + k];
      const float x = __shfl_xor_sync(0xffffffffu, other, off);
      v[k] = kMax ? fmaxf(mine, x) : mine + x;
    }
    if (upper) base += n;
  }
  out1[0] = v[0];
  return base;
}

// A block writes the output of a sequence whose every tile it ran itself
// (and the merge kernel skips such a sequence) when the output is bf16 and the
// rope pairs' cos/sin are all in the prep kernel's table.
__device__ __forceinline__ bool direct_output(const DecodeArgs& a) {
  return !a.out_fp8 && a.rope.rope_dim <= 2 * kRopeTable;
}

// That output (called by a softmax thread at the segment's end, O^T complete
// in tensor memory): O^T rows of this thread's lane (dims 128 mt + row,
// mt = 2 hh, 2 hh + 1) times inv_l per head, the inverse RoPE at position
// L - 1 on the rope pairs (the pair's other dim is in the neighbouring lane),
// bf16 into out16 (the sequence's [64 heads][512 dims]). This is the merge
// kernel's arithmetic for a sequence with one partial result (weight 1).
__device__ __noinline__ void write_whole_output(uint16_t* out16, const float2* cs_tab, int rope_dim,
                                                int rope_offset, uint32_t lane_base, int hh, int row,
                                                const float* inv_l) {
#pragma unroll 1
  for (int m2 = 0; m2 < 2; ++m2) {
    const int mt = 2 * hh + m2;
    const int d = 128 * mt + row, de = d & ~1;
    const bool rot = cs_tab && de >= rope_offset && de + 1 < rope_offset + rope_dim;
    float c = 1.f, sn = 0.f;
    if (rot) {
      const float2 cs = cs_tab[(de - rope_offset) >> 1];
      c = cs.x;
      sn = cs.y;
    }
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      uint32_t r32[32];
      tc::tmem_ld32(lane_base + kOCol + kH * mt + 32 * half, r32);
      tc::tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        float v = __uint_as_float(r32[h]) * inv_l[32 * half + h];
        const float p = __shfl_xor_sync(0xffffffffu, v, 1);
        if (rot)
          v = (d & 1) ? __fadd_rn(__fmul_rn(p, -sn), __fmul_rn(v, c))
                      : __fsub_rn(__fmul_rn(v, c), __fmul_rn(p, -sn));
        out16[(size_t)(32 * half + h) * kD + d] = float_to_bf16_bits(v);
      }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = tc::smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t* sm = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  Bars* bars = reinterpret_cast<Bars*>(sm + kBarOff);
  float* meta = reinterpret_cast<float*>(sm + kMetaOff);
  const uint8_t** rowptr = reinterpret_cast<const uint8_t**>(sm + kPtrOff);
  uint32_t* info = reinterpret_cast<uint32_t*>(sm + kInfoOff);
  float* mref = reinterpret_cast<float*>(sm + kMrefOff);
  float* alpha = reinterpret_cast<float*>(sm + kAlphaOff);
  float* red = reinterpret_cast<float*>(sm + kRedOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kMiscOff + 4);
  int* range = reinterpret_cast<int*>(sm + kMiscOff + 16);  // x0, x1, b0, lt0, L0

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

  // barriers and tensor memory first: this overlaps the query-preparation
  // kernel still running ahead of this one
  if (tid == 0) {
    for (int k = 0; k < kRing; ++k) {
      tc::mbar_init(&bars->addr_ready[k], 32);
      tc::mbar_init(&bars->addr_free[k], 256);
    }
    for (int c = 0; c < 4; ++c) {
      tc::mbar_init(&bars->v_full[c], 256);
      tc::mbar_init(&bars->v_empty[c], 1);
    }
    tc::mbar_init(&bars->s_full[0], 1);
    tc::mbar_init(&bars->s_full[1], 1);
    tc::mbar_init(&bars->p_full, 256);
    tc::mbar_init(&bars->pv_done, 1);
    tc::mbar_init(&bars->q_ready, 1);
    tc::mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 8) tc::tmem_alloc(tmem_slot, kTmemCols);
  if (tid < kH) mref[tid] = kNone;
  tc::pdl_wait();  // the tile prefix sums and query images are complete from here on
  tc::pdl_launch_dependents();

  // ---- this block's tile range [x0, x1) and the sequence of its first tile
  // (the prep kernel balanced the ranges by estimated cost)
  if (tid == 0) {
    // one record per block (independent loads): no chain of dependent loads
    // before the first tile's addresses can be resolved
    const int4 rec = a.cta_rec[cta];
    range[0] = rec.x;
    range[1] = rec.y;
    range[2] = rec.z;
    range[3] = rec.w;
    range[4] = a.cta_L0[cta];
    if (rec.x < rec.y) issue_q(a, rec.z, sbase + kQOff, &bars->q_ready);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const int x0 = range[0], x1 = range[1];
  const int n_tiles = x1 - x0;
  const int b0 = range[2], lt0 = range[3], L0 = range[4];
  const uint32_t tmem = *tmem_slot;
  if (x0 >= x1) {
    // nothing to do: release tensor memory and leave
    if (warp == 8) tc::tmem_free(tmem, kTmemCols);
    return;
  }

  if (warp >= 9) {
    // ======================= address resolution + L2 prefetch, up to kRing - 1 tiles ahead
    // (warp 9 the even tiles, warp 10 the odd ones)
    const int aw = warp - 9;
    Cursor cu;
    cursor_set(cu, a, b0, lt0, L0);
    if (aw) cursor_next(cu, a);
    for (int t = aw; t < n_tiles; t += 2) {
      const int buf = t % kRing;
      if (t >= kRing && !tc::mbar_wait(&bars->addr_free[buf], ((t - kRing) / kRing) & 1, abort_flag)) break;
      if (t > 0 && cu.lt == 0) {
        // a new sequence starts: pull its query image into L2 as well
        const uint8_t* qp = a.qh + (size_t)cu.b * kQBytes;
        if (lane < 4) prefetch_l2_bulk(qp + lane * (kQBytes / 4), kQBytes / 4);
      }
      const int tile0 = cu.lt * kT;
      resolve_tile(a, cu.b, cu.s, tile0, lane, rowptr + buf * kT, meta + buf * kT);
      if (t >= 2) {
        // rows into L2 for the workers' loads, one bulk prefetch per row (a
        // per-line prefetch issues four times the instructions, which hold up
        // the softmax's shared- and tensor-memory operations). Tiles 0 and 1
        // are loaded at once by the workers; prefetching them too would only
        // add to the burst of requests every block makes at its start.
        const bool main_tile = tile0 < cu.s.n_sel_pad;
        const bool fp8 = (main_tile ? a.main.dtype : a.window.dtype) == V4KV_FP8_E4M3;
        const uint8_t* const* rp = rowptr + buf * kT;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint8_t* pr = rp[lane + 32 * r];
          if (pr)
            prefetch_l2_bulk(pr, fp8 ? kD : 2 * kD);
        }
      }
      if (lane == 0) {
        const bool main_tile = tile0 < cu.s.n_sel_pad;
        const bool fp8 = (main_tile ? a.main.dtype : a.window.dtype) == V4KV_FP8_E4M3;
        info[buf] = (fp8 ? kInfoFp8 : 0u) | ((t == 0 || cu.lt == 0) ? kInfoFirst : 0u);
      }
      __syncwarp();
      tc::mbar_arrive(&bars->addr_ready[buf]);
      cursor_next(cu, a);
      cursor_next(cu, a);
    }
  } else if (warp == 8) {
    // ======================= MMA issuer
    // The whole warp runs the loop, so descriptors, addresses and wait results
    // stay warp-uniform; one lane, elected once, issues every MMA and commit
    // (a commit tracks the MMAs of the thread that issues it).
    const bool leader = tc::elect_one();
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t iq = tc::idesc_f16(128, kH, 0, 0);
    const uint32_t ip = tc::idesc_f16(128, kH, 1, 1);
    // descriptors at the operands' bases; a step adds its byte offset / 16
    const uint64_t vk_desc = tc::sw128_desc(sbase + kVOff, 16, 1024);     // V, K-major
    const uint64_t qk_desc = tc::sw128_desc(sbase + kQOff, 16, 1024);     // Q, K-major
    const uint64_t vm_desc = tc::sw128_desc(sbase + kVOff, 16384, 1024);  // V^T, MN-major
    const uint64_t p_desc = tc::sw128_desc(sbase + kPOff, 0, 1024);       // P^T, MN-major
    bool ok = true;
    int seg = 0;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const uint32_t par = i & 1;
      const uint32_t s_col = (uint32_t)(i & 1) * kH;
      bool first = i == 0;
      for (int c = 0; c < 4 && ok; ++c) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->v_full[c], par, abort_flag));
        if (!ok) break;
        if (c == 0) {
          // the converters read this tile's info word before arriving
          first = (info[i % kRing] & kInfoFirst) != 0;
          if (first) {
            // the segment's query image has landed in shared memory
            ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->q_ready, seg & 1, abort_flag));
            if (!ok) break;
            ++seg;
          }
        }
        tc::tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k8 = 0; k8 < 8; ++k8) {
            const int kk = 8 * c + k8;  // 16-dim step: atom kk/4, 32-byte column kk%4
            tc::mma_f16(tm + s_col, vk_desc + (uint64_t)((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                        qk_desc + (uint64_t)((((kk >> 2) * 8192) + (kk & 3) * 32) >> 4), iq,
                        kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) tc::mma_commit(&bars->s_full[i & 1]);
      __syncwarp();
      ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->p_full, par, abort_flag));
      if (!ok) break;
      tc::tc_fence_after();
      if (leader) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16(tm + kOCol + kH * mt, vm_desc + (uint64_t)((2 * mt * 16384 + kk * 2048) >> 4),
                        p_desc + (uint64_t)((kk * 2048) >> 4), ip, (!first || kk > 0) ? 1u : 0u);
          tc::mma_commit(&bars->v_empty[mt]);
        }
        tc::mma_commit(&bars->pv_done);
      }
      __syncwarp();
    }
    if (!ok && leader) {
      *abort_flag = 1;
      flag(a.dev_status, V4KV_DEV_TIMEOUT);
    }
    // every MMA issued has completed once this barrier flips; this wait
    // ignores the abort flag (tensor memory is freed after it)
    if (leader) tc::mma_commit(&bars->drain);
    __syncwarp();
    volatile int never = 0;
    if (!tc::mbar_wait(&bars->drain, 0, &never) && leader) flag(a.dev_status, V4KV_DEV_TIMEOUT);
    __syncwarp();
  } else {
    // ======================= workers (warps 0-7): softmax and gather + convert
    // Softmax: thread (warp w, lane l) owns tile row j = 32 (w % 4) + l (its
    // TMEM lane) and heads 32 hh .. 32 hh + 31 (hh = w / 4); its partial
    // normalisers live in tensor memory (columns kLCol + 32 hh ..). Conversion: warp w writes rows 16w ..
    // 16w + 15 of every V chunk. Per tile: softmax(i), then the conversion of
    // tile i + 1 as the second product of tile i frees each V chunk; the codes
    // of tile i + 1 are loaded before softmax(i).
    const int hh = warp >> 2;
    const int row = 32 * (warp & 3) + lane;   // tile row = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    uint4 rawv[4][4];
    const uint32_t l_addr = lane_base + kLCol + 32 * hh;
    {
      uint32_t z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0u;
      tc::tmem_st32(l_addr, z);
      tc::tmem_wait_st();
    }
    float k0 = a.qk0[b0];
    int q_issued = 1;  // query copies started by this thread (tid 0 only)
    bool wide = false; // a bf16 value outside the f16 range was clamped
    bool ok = true;

    // fp8 rows: lane covers rows 16w + 4r + lane/8 (r = 0..3), 16 bytes at
    // 16*(lane%8) of each 128-byte dim chunk
    auto load_fp8 = [&](int t) {
      const uint8_t** rp = rowptr + (t % kRing) * kT;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint8_t* p = rp[16 * warp + 4 * r + (lane >> 3)];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          rawv[c][r] = p ? ldg_stream(p + 128 * c + 16 * (lane & 7)) : make_uint4(0, 0, 0, 0);
      }
    };
    // convert tile t into the V buffer; chunk c waits for the second product of
    // tile t - 1 to release it (v_empty)
    auto convert = [&](int t, bool fp8) -> bool {
      if (fp8) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (t > 0 && !tc::mbar_wait(&bars->v_empty[c], (t - 1) & 1, abort_flag)) return false;
          const int part = lane & 7;                 // 16-dim piece within the chunk
          const uint32_t atom = 2 * c + (part >> 2);
          const uint32_t q = 2 * (part & 3);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t vr = 16 * warp + 4 * r + (lane >> 3);
            uint4 lo, hi;
            fp8x16_to_f16(rawv[c][r], lo, hi);
            uint8_t* base = sm + kVOff + atom * 16384;
            if (part & 4) {
              *reinterpret_cast<uint4*>(base + tc::sw128_off(vr, q + 1)) = hi;
              *reinterpret_cast<uint4*>(base + tc::sw128_off(vr, q)) = lo;
            } else {
              *reinterpret_cast<uint4*>(base + tc::sw128_off(vr, q)) = lo;
              *reinterpret_cast<uint4*>(base + tc::sw128_off(vr, q + 1)) = hi;
            }
          }
          tc::fence_proxy_async_smem();
          tc::mbar_arrive(&bars->v_full[c]);
        }
      } else {
        // bf16 rows: lane covers rows 16w + 2r + lane/16 (r = 0..7), 16 bytes at
        // 16*(lane%16) of each 256-byte dim chunk; chunk c + 1 is loaded while
        // chunk c is converted (the two buffers reuse the code registers)
        const uint8_t** rp = rowptr + (t % kRing) * kT;
#define V4KV_RB(k, r) rawv[2 * (k) + ((r) >> 2)][(r) & 3]
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const uint8_t* p = rp[16 * warp + 2 * r + (lane >> 4)];
          V4KV_RB(0, r) = p ? ldg_stream(p + 16 * (lane & 15)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) {
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              const uint8_t* p = rp[16 * warp + 2 * r + (lane >> 4)];
              V4KV_RB((c + 1) & 1, r) = p ? ldg_stream(p + 256 * (c + 1) + 16 * (lane & 15)) : make_uint4(0, 0, 0, 0);
            }
          }
          if (t > 0 && !tc::mbar_wait(&bars->v_empty[c], (t - 1) & 1, abort_flag)) return false;
          const int part = lane & 15;                // 8-dim piece within the chunk
          const uint32_t atom = 2 * c + (part >> 3);
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint32_t vr = 16 * warp + 2 * r + (lane >> 4);
            *reinterpret_cast<uint4*>(sm + kVOff + atom * 16384 + tc::sw128_off(vr, part & 7)) =
                bf16x8_to_f16(V4KV_RB(c & 1, r), wide);
          }
          tc::fence_proxy_async_smem();
          tc::mbar_arrive(&bars->v_full[c]);
        }
#undef V4KV_RB
      }
      return true;
    };

    // tile 0
    {
      ok = tc::mbar_wait(&bars->addr_ready[0], 0, abort_flag);
      const bool fp8 = ok && (info[0] & kInfoFp8) != 0;
      if (ok && fp8) load_fp8(0);
      if (ok) ok = convert(0, fp8);
    }
    Cursor cu;
    cursor_set(cu, a, b0, lt0, L0);
    bool seg_first = true;  // the current tile opens a segment
    for (int i = 0; i < n_tiles && ok; ++i) {
      const bool seg_last = i == n_tiles - 1 || cu.lt == cu.nt - 1;
      // S(i) complete implies PV(i-1) complete (the MMAs run in issue order),
      // so waiting for pv_done(i-1) here costs nothing and frees P and O^T
      ok = ok && tc::mbar_wait_spin(&bars->s_full[i & 1], (i >> 1) & 1, abort_flag, 32) &&
           (i == 0 || tc::mbar_wait(&bars->pv_done, (i - 1) & 1, abort_flag));
      // the eight worker warps leave together (they meet at named barriers)
      ok = named_and(1, 256, ok);
      if (!ok) break;
      tc::tc_fence_after();
      // a row is an item when its address was resolved; its scale may be any
      // value (value = code * scale): |scale| enters the exponent, its sign the
      // weight P', and a zero scale gives a zero-valued item that still counts
      // in the normaliser with score 0
      const bool valid = rowptr[(i % kRing) * kT + row] != nullptr;
      const float ks = meta[(i % kRing) * kT + row];
      const float aks = fabsf(ks);
      const float cj = valid ? k0 * ks : 0.f;
      const float lk = !valid ? -INFINITY : (aks > 0.f ? __log2f(aks) : 0.f);
      const float inv_k = !valid ? 0.f : (aks > 0.f ? __frcp_rn(aks) : 1.f);
      const float sgn = (valid && ks != 0.f) ? copysignf(1.f, ks) : 0.f;
      // u = score in log2 units including log2 ks; d = u - m_ref (in place)
      float d[32];
      const uint32_t s_addr = lane_base + (uint32_t)(i & 1) * kH + 32 * hh;
      {
        uint32_t r32[32];
        tc::tmem_ld32(s_addr, r32);
        tc::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) d[h] = fmaf(__uint_as_float(r32[h]), cj, lk);
      }
      if (seg_last && i + 1 < n_tiles && tid == 0) {
        // QK(i) is complete (S(i) was read), so Q is free: copy the next
        // segment's query image while the rest of this tile runs
        Cursor nx = cu;
        cursor_next(nx, a);
        issue_q(a, nx.b, sbase + kQOff, &bars->q_ready);
        ++q_issued;
      }
      float dmax = -INFINITY;
      if (!seg_first) {
        const float4* mr4 = reinterpret_cast<const float4*>(mref + 32 * hh);
#pragma unroll
        for (int h4 = 0; h4 < 8; ++h4) {
          const float4 m4 = mr4[h4];
          d[4 * h4] -= m4.x;
          d[4 * h4 + 1] -= m4.y;
          d[4 * h4 + 2] -= m4.z;
          d[4 * h4 + 3] -= m4.w;
          dmax = fmaxf(dmax, fmaxf(fmaxf(d[4 * h4], d[4 * h4 + 1]), fmaxf(d[4 * h4 + 2], d[4 * h4 + 3])));
        }
      }
      // A segment's first tile sets the references to its per-head maxima
      // (d still holds u, the normalisers are zero and O^T is written afresh);
      // a later tile raises them, rarely, when a score exceeds its reference
      // by 2^kTau.
      if (seg_first || named_or(1, 256, dmax > kTau)) {
        if (!seg_first) {
          // u is recomputed from S (still in tensor memory) to keep it exact
          uint32_t r32[32];
          tc::tmem_ld32(s_addr, r32);
          tc::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 32; ++h) d[h] = fmaf(__uint_as_float(r32[h]), cj, lk);
        }
        {
          // per-head maximum over the warp's 32 rows: a transposing
          // shuffle reduction leaves head hb's maximum in this lane
          float t32[32], one[1];
#pragma unroll
          for (int h = 0; h < 32; ++h) t32[h] = d[h];
          const int hb = warp_reduce_scatter32<true>(t32, lane, one);
          red[warp * 32 + hb] = one[0];
        }
        named_sync(1, 256);
        if (tid < kH) {
          const int half = tid >> 5, hx = tid & 31;
          const float old = mref[tid];
          float nm = old;
#pragma unroll
          for (int w = 0; w < 4; ++w) nm = fmaxf(nm, red[(4 * half + w) * 32 + hx]);
          alpha[tid] = exp2f(old - nm);
          mref[tid] = nm;
        }
        named_sync(1, 256);
#pragma unroll
        for (int h = 0; h < 32; ++h) d[h] -= mref[32 * hh + h];
        if (!seg_first) {
          {
            uint32_t lv[32];
            tc::tmem_ld32(l_addr, lv);
            tc::tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 32; ++h)
              lv[h] = __float_as_uint(__uint_as_float(lv[h]) * alpha[32 * hh + h]);
            tc::tmem_st32(l_addr, lv);
            tc::tmem_wait_st();
          }
          // O^T rows of this lane (dims 128 mt + row, mt = 2hh, 2hh + 1) times
          // alpha per head column
#pragma unroll 1
          for (int m2 = 0; m2 < 2; ++m2) {
            const int mt = 2 * hh + m2;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              uint32_t r32[32];
              const uint32_t ta = lane_base + kOCol + kH * mt + 32 * half;
              tc::tmem_ld32(ta, r32);
              tc::tmem_wait_ld();
#pragma unroll
              for (int h = 0; h < 32; ++h)
                r32[h] = __float_as_uint(__uint_as_float(r32[h]) * alpha[32 * half + h]);
              tc::tmem_st32(ta, r32);
            }
          }
          tc::tmem_wait_st();
        }
      }
      // P' row of this item: heads 32 hh .. 32 hh + 31 in f16, 8 heads per
      // 16-byte chunk (chunks 4 hh .. 4 hh + 3 of the MN-major swizzled row);
      // d keeps the fp32 weights for the normaliser update after the arrive
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = 8 * c + 2 * e;
          d[h] = fast_exp2(d[h]);
          d[h + 1] = fast_exp2(d[h + 1]);
          pk[e] = h2u(__floats2half2_rn(sgn * d[h], sgn * d[h + 1]));
        }
        *reinterpret_cast<uint4*>(sm + kPOff + tc::sw128_off(row, 4 * hh + c)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bars->p_full);
      tc::mbar_arrive(&bars->addr_free[i % kRing]);
      // the next tile's codes (fp8) fly while PV(i) runs. They are requested
      // only now: a barrier or a release arrival waits for every load this
      // thread has in flight, so loads issued before the softmax would hold
      // it back by a memory latency.
      bool nxt_fp8 = false;
      if (i + 1 < n_tiles) {
        ok = tc::mbar_wait(&bars->addr_ready[(i + 1) % kRing], ((i + 1) / kRing) & 1, abort_flag);
        ok = named_and(1, 256, ok);  // the workers leave together
        if (!ok) break;
        nxt_fp8 = (info[(i + 1) % kRing] & kInfoFp8) != 0;
        if (nxt_fp8) load_fp8(i + 1);
      }
      {
        uint32_t lv[32];
        tc::tmem_ld32(l_addr, lv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) lv[h] = __float_as_uint(fmaf(d[h], inv_k, __uint_as_float(lv[h])));
        tc::tmem_st32(l_addr, lv);
        tc::tmem_wait_st();
      }
      // convert tile i + 1 as PV(i) frees the V chunks (before the epilogue,
      // so that QK(i + 1) overlaps it; PV(i + 1) cannot start before the
      // epilogue has read O^T, since it needs this tile loop's next P')
      if (i + 1 < n_tiles && !(ok = convert(i + 1, nxt_fp8))) break;

      if (seg_last) {
        // a segment that covers its whole sequence writes the output itself
        // (bf16; the merge skips such sequences), any other one a partial result
        // (every segment but the block's first opens at the sequence's first
        // tile; the first one does when the block's range starts there)
        const bool whole = (cu.b != range[2] || range[3] == 0) && cu.lt == cu.nt - 1 && direct_output(a);
        const int b_done = cu.b, L_done = cu.s.L;
        cursor_next(cu, a);
        if (i + 1 < n_tiles) k0 = a.qk0[cu.b];
        ok = tc::mbar_wait(&bars->pv_done, i & 1, abort_flag);
        ok = named_and(1, 256, ok);
        if (!ok) break;
        tc::tc_fence_after();
        const size_t prow = ((size_t)b_done + cta) * kH;
        // normaliser: sum the 128 rows' partial sums per head
        {
          float lsum[32];
          {
            uint32_t lv[32];
            tc::tmem_ld32(l_addr, lv);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) lsum[e] = __uint_as_float(lv[e]);
          }
          float two[1];
          const int hb = warp_reduce_scatter32<false>(lsum, lane, two);
          named_sync(1, 256);  // red is free (no slow path in flight)
          red[warp * 32 + hb] = two[0];
          named_sync(1, 256);
          if (tid < kH) {
            const int half = tid >> 5, hx = tid & 31;
            const float l = red[(4 * half) * 32 + hx] + red[(4 * half + 1) * 32 + hx] +
                            red[(4 * half + 2) * 32 + hx] + red[(4 * half + 3) * 32 + hx];
            if (whole) {
              alpha[tid] = l > 0.f ? 1.f / l : 0.f;  // the merge's weight for a single slot is 1
            } else {
              a.part_ml[(prow + tid) * 2] = mref[tid];
              a.part_ml[(prow + tid) * 2 + 1] = l;
            }
            mref[tid] = kNone;
          }
          {
            uint32_t z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0u;
            tc::tmem_st32(l_addr, z);
            tc::tmem_wait_st();
          }
          named_sync(1, 256);
        }
        if (whole) {
          const int Lb = min(L_done, a.max_len);
          const bool rope = a.rope.rope_dim > 0 && Lb > 0;
          write_whole_output(reinterpret_cast<uint16_t*>(a.out) + (size_t)b_done * kH * kD,
                             rope ? a.rope_tab + (size_t)b_done * kRopeTable : nullptr, a.rope.rope_dim,
                             a.rope.rope_offset, lane_base, hh, row, alpha);
        } else {
          // partial result of (sequence b_done, block cta) in slot b_done + cta:
          // O^T un-normalised, relative to the reference maximum
#pragma unroll 1
          for (int m2 = 0; m2 < 2; ++m2) {
            const int mt = 2 * hh + m2;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              uint32_t r32[32];
              tc::tmem_ld32(lane_base + kOCol + kH * mt + 32 * half, r32);
              tc::tmem_wait_ld();
#pragma unroll
              for (int h = 0; h < 32; ++h)
                a.part_o[(prow + 32 * half + h) * kD + 128 * mt + row] = __uint_as_float(r32[h]);
            }
          }
        }
        seg_first = true;
      } else {
        cursor_next(cu, a);
        seg_first = false;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      flag(a.dev_status, V4KV_DEV_TIMEOUT);
    }
    if (__any_sync(0xffffffffu, wide) && lane == 0) flag(a.dev_status, V4KV_DEV_RANGE);
    if (tid == 0) {
      // the last query copy has landed before shared memory is released
      // (normally long since; after an abort it may still be in flight)
      volatile int never = 0;
      if (!tc::mbar_wait(&bars->q_ready, (q_issued - 1) & 1, &never)) flag(a.dev_status, V4KV_DEV_TIMEOUT);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc::tc_fence_after();
    tc::tmem_free(tmem, kTmemCols);
  }
}

// grid (heads / kMergeWarps, batch), a warp per head: warp w merges head
// kMergeWarps * blockIdx.x + w of sequence b over the blocks whose tile ranges
// met it (lane l: dims 16l .. 16l + 15), normalises, applies the inverse RoPE
// at position L - 1 (cos/sin from the prep kernel's table) and stores bf16
// (or e4m3 with a scale per head).
template <int kMergeFirst>
__global__ void __launch_bounds__(kMergeWarps * 32) decode_tc_merge_kernel(DecodeArgs a) {
  __shared__ float w_sh[kMergeWarps][kMaxSplits];  // per warp: the blocks' weights
  __shared__ float2 cs_sh[kRopeTable];             // the sequence's inverse-RoPE cos / sin
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = kMergeWarps * blockIdx.x + warp, b = blockIdx.y;
  const int d0 = 16 * lane;
  // What the prep kernel wrote is read before the wait: the sweep launched
  // this grid only after its own wait for the prep kernel, so those writes
  // are complete, and these loads overlap the sweep's last blocks. The
  // sequence's blocks and length, which of them have tiles, and the
  // inverse-RoPE table (read at the end).
  const int2 sl = a.seq_slots[b];
  const int Lb = min(a.seq_lens[b], a.max_len);
  if (threadIdx.x < kRopeTable) cs_sh[threadIdx.x] = a.rope_tab[(size_t)b * kRopeTable + threadIdx.x];
  const int lo = sl.x, hi = sl.y;
  bool has_keep[(kMaxSplits + 31) / 32];
#pragma unroll
  for (int k = 0; k < (kMaxSplits + 31) / 32; ++k) {
    const int c = lo + lane + 32 * k;
    has_keep[k] = c <= hi && a.cta_x0[c + 1] > a.cta_x0[c];
  }
  tc::pdl_wait();  // the sweep's partial results are complete from here on
  if (lo == hi && direct_output(a)) return;  // one block ran the whole sequence and wrote its output
  // per block: (m, l); the first blocks' rows are requested at the same time
  // (they do not depend on the weights, which only select them)
  float2 ml_keep[(kMaxSplits + 31) / 32];
#pragma unroll
  for (int k = 0; k < (kMaxSplits + 31) / 32; ++k) {
    const int c = lo + lane + 32 * k;
    ml_keep[k] = make_float2(-INFINITY, 0.f);
    if (c <= hi) ml_keep[k] = reinterpret_cast<const float2*>(a.part_ml)[((size_t)b + c) * kH + h];
  }
  float4 v0[kMergeFirst][4];
#pragma unroll
  for (int j = 0; j < kMergeFirst; ++j) {
    if (lo + j <= hi) {
      const float4* o4 = reinterpret_cast<const float4*>(a.part_o + (((size_t)b + lo + j) * kH + h) * kD + d0);
#pragma unroll
      for (int q = 0; q < 4; ++q) v0[j][q] = o4[q];
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < (kMaxSplits + 31) / 32; ++k) {
    if (!has_keep[k]) ml_keep[k] = make_float2(-INFINITY, 0.f);
    M = fmaxf(M, ml_keep[k].x);
  }
  M = warp_max(M);
  float L = 0.f;
#pragma unroll
  for (int k = 0; k < (kMaxSplits + 31) / 32; ++k) {
    const int c = lo + lane + 32 * k;
    if (c <= hi) {
      const float w = ml_keep[k].x == -INFINITY ? 0.f : exp2f(ml_keep[k].x - M);
      w_sh[warp][c - lo] = w;
      L = fmaf(w, ml_keep[k].y, L);
    }
  }
  L = warp_sum(L);
  __syncwarp();
  // weighted sum of the blocks' rows in block order (a block with weight 0
  // adds 0 * 0, as every block's row would)
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  auto add_rows = [&](int c, int nj, float4 (*v)[4]) {
#pragma unroll 4
    for (int j = 0; j < nj; ++j) {
      const float w = c + j <= hi ? w_sh[warp][c + j - lo] : 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 x = w != 0.f ? v[j][q] : make_float4(0.f, 0.f, 0.f, 0.f);
        acc[4 * q] = fmaf(w, x.x, acc[4 * q]);
        acc[4 * q + 1] = fmaf(w, x.y, acc[4 * q + 1]);
        acc[4 * q + 2] = fmaf(w, x.z, acc[4 * q + 2]);
        acc[4 * q + 3] = fmaf(w, x.w, acc[4 * q + 3]);
      }
    }
  };
  add_rows(lo, kMergeFirst, v0);
  for (int c = lo + kMergeFirst; c <= hi; c += kMergeFirst) {
    float4 v[kMergeFirst][4];
#pragma unroll
    for (int j = 0; j < kMergeFirst; ++j) {
      if (c + j <= hi) {
        const float4* o4 = reinterpret_cast<const float4*>(a.part_o + (((size_t)b + c + j) * kH + h) * kD + d0);
#pragma unroll
        for (int q = 0; q < 4; ++q) v[j][q] = o4[q];
      }
    }
    add_rows(c, kMergeFirst, v);
  }
  __syncthreads();  // the RoPE table is in shared memory
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] *= inv;
  if (a.rope.rope_dim > 0 && Lb > 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int d = d0 + 2 * k;
      if (d >= a.rope.rope_offset && d + 1 < a.rope.rope_offset + a.rope.rope_dim) {
        const int i = (d - a.rope.rope_offset) >> 1;
        float c, s;
        if (i < kRopeTable) {
          c = cs_sh[i].x;
          s = cs_sh[i].y;
        } else {
          rope_cs(a.rope, i, (long long)Lb - 1, &c, &s);
        }
        rope_apply(acc[2 * k], acc[2 * k + 1], c, -s);
      }
    }
  }
  float amax = 0.f;
  if (a.out_fp8) {
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(acc[e]));
    amax = warp_max(amax);
  }
  store_output<16>(a, (size_t)b * kH + h, d0, acc, amax, lane == 0);
}

// grid (batch + 1), 256 threads. Block b < batch writes sequence b's query as
// the shared-memory image of the first product's B operand: f16, scaled by
// 2^e so that max|q| * 2^e < 2^15, eight 64-dim atoms of 64 head rows x 128 B
// in the 128-byte swizzle, so that one linear copy puts it in place; and
// qk0[b] = sm_scale * log2(e) * 2^-e. Block `batch` writes the tile prefix
// sums cum[0..batch].
__global__ void __launch_bounds__(256) decode_tc_prep_kernel(DecodeArgs a) {
  tc::pdl_wait();  // q and the lengths (written by earlier work in the stream) are complete
  tc::pdl_launch_dependents();
  const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  __shared__ float red[8];
  __shared__ int wsum[8];
  if (b == a.batch) {
    // tiles and estimated cost per sequence, their prefix sums, then each
    // block's range: block c starts at the tile where the cost prefix reaches
    // c/G of the total
    __shared__ long long csum[8];
    __shared__ int x0_sh[kMaxSplits + 1];
    __shared__ int b0_sh[kMaxSplits];
    // the prefix sums also go to shared memory (when they fit) for the
    // binary searches below, which would otherwise chain global loads
    __shared__ int cum_sh[kPrepCache + 1];
    __shared__ long long ccum_sh[kPrepCache + 1];
    __shared__ int len_sh[kPrepCache];  // clamped lengths
    const bool cached = a.batch <= kPrepCache;
    int carry = 0;
    long long ccarry = 0;
    long long cmax = 0;  // the largest sequence cost (this thread's share)
    for (int base = 0; base < a.batch; base += 256) {
      const int bb = base + t;
      int n = 0;
      long long cost = 0;
      if (bb < a.batch) {
        if (a.seq_lens[bb] > a.max_len) flag(a.dev_status, V4KV_DEV_OVERFLOW);
        const Seq sq = seq_of(a, bb, nullptr);
        n = tiles_of(sq);
        cost = seq_cost(a, sq);
        cmax = max(cmax, cost);
        if (cached) len_sh[bb] = sq.L;
      }
      int incl = n;
      long long cincl = cost;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        const long long cy = __shfl_up_sync(0xffffffffu, cincl, o);
        if (lane >= o) { incl += y; cincl += cy; }
      }
      if (lane == 31) { wsum[warp] = incl; csum[warp] = cincl; }
      __syncthreads();
      int before = carry;
      long long cbefore = ccarry;
      for (int w = 0; w < warp; ++w) { before += wsum[w]; cbefore += csum[w]; }
      if (bb < a.batch) {
        a.cum[bb] = before + incl - n;
        a.costcum[bb] = cbefore + cincl - cost;
        if (cached) {
          cum_sh[bb] = before + incl - n;
          ccum_sh[bb] = cbefore + cincl - cost;
        }
      }
      for (int w = 0; w < 8; ++w) { carry += wsum[w]; ccarry += csum[w]; }
      __syncthreads();
    }
    if (t == 0) {
      a.cum[a.batch] = carry;
      a.costcum[a.batch] = ccarry;
      if (cached) {
        cum_sh[a.batch] = carry;
        ccum_sh[a.batch] = ccarry;
      }
    }
    // the largest sequence cost, over the block
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    if (lane == 0) csum[warp] = cmax;
    __syncthreads();  // the prefix sums are visible to the whole block
    for (int w = 0; w < 8; ++w) cmax = max(cmax, csum[w]);
    const int* cum = cached ? cum_sh : a.cum;
    const long long* costcum = cached ? ccum_sh : a.costcum;
    const int G = a.n_splits;
    // One sequence per block when every sequence fits one block at a cost
    // no greater than an even split plus the split's own cost (partial
    // results and their merge): each block then writes its sequence's output
    // itself. Otherwise block c starts where the cost prefix reaches c/G of
    // the total.
    const bool whole = a.batch <= G && cmax * G <= ccarry + (long long)kCostMerge * G;
    for (int c = t; c <= G; c += 256) {
      int x0 = carry, b0 = a.batch;
      if (whole) {
        if (c < a.batch) {
          x0 = cum[c];
          b0 = c;
        }
      } else if (c < G && ccarry > 0) {
        const long long target = (long long)c * ccarry / G;
        int l = 0, r = a.batch - 1;  // last sequence whose cost prefix is <= target
        while (l < r) {
          const int m = (l + r + 1) >> 1;
          if (costcum[m] <= target) l = m; else r = m - 1;
        }
        b0 = l;
        const Seq sq = cached ? seq_from_len(a, len_sh[b0]) : seq_of(a, b0, nullptr);
        x0 = cum[b0] + tile_at_cost(a, sq, target - costcum[b0]);
      }
      a.cta_x0[c] = x0;
      x0_sh[c] = x0;
      if (c < G) b0_sh[c] = b0;
    }
    __syncthreads();
    for (int c = t; c < G; c += 256) {
      const int x0 = x0_sh[c], x1 = x0_sh[c + 1], b0 = b0_sh[c];
      const bool live = x0 < x1 && b0 < a.batch;
      a.cta_rec[c] = live ? make_int4(x0, x1, b0, x0 - cum[b0]) : make_int4(x0, x0, a.batch, 0);
      a.cta_L0[c] = live ? (cached ? len_sh[b0] : seq_of(a, b0, nullptr).L) : 0;
    }
    // blocks whose ranges [x0[c], x0[c+1]) meet each sequence's tiles [c0, c1)
    for (int bb = t; bb < a.batch; bb += 256) {
      const int c0 = cum[bb], c1 = cum[bb + 1];
      int lo = 0, hi = -1;
      if (c1 > c0) {
        int l = 0, r = G;  // first c with x0[c+1] > c0
        while (l < r) {
          const int m = (l + r) >> 1;
          if (x0_sh[m + 1] > c0) r = m; else l = m + 1;
        }
        lo = l;
        l = lo; r = G;     // first c with x0[c] >= c1
        while (l < r) {
          const int m = (l + r) >> 1;
          if (x0_sh[m] >= c1) r = m; else l = m + 1;
        }
        hi = l - 1;
      }
      a.seq_slots[bb] = make_int2(lo, hi);
    }
    return;
  }
  // thread t holds 8-dim chunks u = t + 256 k (k < 16) of the 64 x 64 chunks
  float x[16][8];
  const size_t qoff = (size_t)b * kH * kD;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const size_t o = qoff + (size_t)(t + 256 * k) * 8;
    if (a.q_dtype == V4KV_FP32) {
      const float4 x0 = reinterpret_cast<const float4*>(a.q)[o / 4];
      const float4 x1 = reinterpret_cast<const float4*>(a.q)[o / 4 + 1];
      x[k][0] = x0.x; x[k][1] = x0.y; x[k][2] = x0.z; x[k][3] = x0.w;
      x[k][4] = x1.x; x[k][5] = x1.y; x[k][6] = x1.z; x[k][7] = x1.w;
    } else {
      const uint4 r = reinterpret_cast<const uint4*>(a.q)[o / 8];
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[k][2 * i] = __uint_as_float(w[i] << 16);
        x[k][2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  }
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[k][i]));
  m = warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax = 0.f;
  for (int w = 0; w < 8; ++w) amax = fmaxf(amax, red[w]);
  int e = 0;
  if (amax > 0.f) {
    int k;
    frexpf(amax, &k);  // amax < 2^k
    e = 15 - k;
  }
  const float qs = ldexpf(1.f, e);
  uint8_t* img = a.qh + (size_t)b * kQBytes;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int u = t + 256 * k;
    const int h = u / (kD / 8), c8 = u % (kD / 8);  // 8-dim chunk c8 of head h
    uint32_t hv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) hv[i] = h2u(__floats2half2_rn(x[k][2 * i] * qs, x[k][2 * i + 1] * qs));
    *reinterpret_cast<uint4*>(img + (c8 >> 3) * 8192 + tc::sw128_off(h, c8 & 7)) =
        make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
  if (t == 0) a.qk0[b] = a.sm_scale * 1.4426950408889634f * ldexpf(1.f, -e);
  // cos/sin of the inverse RoPE at the query position, for the merge
  if (t < kRopeTable && 2 * t < a.rope.rope_dim) {
    const int Lb = min(a.seq_lens[b], a.max_len);
    float c = 1.f, s = 0.f;
    if (Lb > 0) rope_cs(a.rope, t, (long long)Lb - 1, &c, &s);
    a.rope_tab[(size_t)b * kRopeTable + t] = make_float2(c, s);
  }
}

// workspace of the tensor-core path: query images, their multipliers, partial
// results (o, m, l) per slot, tile prefix sums
size_t decode_tc_workspace_bytes(int batch, int num_sms) {
  const size_t slots = (size_t)batch + num_sms;
  const size_t qk0 = ((size_t)batch * sizeof(float) + 255) / 256 * 256;
  return (size_t)batch * kQBytes + qk0 + slots * kH * (size_t)(kD + 2) * sizeof(float) +
         ((size_t)batch + 1) * sizeof(int32_t) + 256 + ((size_t)batch + 1) * sizeof(long long) +
         ((size_t)num_sms + 1) * sizeof(int32_t) + 16 + (size_t)num_sms * (sizeof(int4) + sizeof(int32_t)) +
         256 + (size_t)batch * sizeof(int2) + 256 +
         (size_t)batch * kRopeTable * sizeof(float2) + 256;
}

void decode_tc_layout(DecodeArgs& a, void* workspace) {
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const size_t slots = (size_t)a.batch + a.n_splits;
  a.qh = w;
  w += (size_t)a.batch * kQBytes;
  a.qk0 = reinterpret_cast<float*>(w);
  w += ((size_t)a.batch * sizeof(float) + 255) / 256 * 256;
  a.part_o = reinterpret_cast<float*>(w);
  a.part_ml = a.part_o + slots * kH * kD;
  a.cum = reinterpret_cast<int32_t*>(a.part_ml + slots * kH * 2);
  uint8_t* c = reinterpret_cast<uint8_t*>(a.cum + a.batch + 1);
  c = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(c) + 255) & ~uintptr_t(255));
  a.costcum = reinterpret_cast<long long*>(c);
  a.cta_x0 = reinterpret_cast<int32_t*>(a.costcum + a.batch + 1);
  uint8_t* rc = reinterpret_cast<uint8_t*>(a.cta_x0 + a.n_splits + 1);
  rc = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rc) + 15) & ~uintptr_t(15));
  a.cta_rec = reinterpret_cast<int4*>(rc);
  a.cta_L0 = reinterpret_cast<int32_t*>(a.cta_rec + a.n_splits);
  uint8_t* q = reinterpret_cast<uint8_t*>(a.cta_L0 + a.n_splits);
  q = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(q) + 255) & ~uintptr_t(255));
  a.seq_slots = reinterpret_cast<int2*>(q);
  uint8_t* r = reinterpret_cast<uint8_t*>(a.seq_slots + a.batch);
  r = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(r) + 255) & ~uintptr_t(255));
  a.rope_tab = reinterpret_cast<float2*>(r);
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_tc_prep_kernel, dim3(a.batch + 1), dim3(256), 0, stream, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_tc_kernel, dim3(a.n_splits), dim3(kThreads), kSmemBytes, stream, a);
  if (e != cudaSuccess) return e;
  // a merge warp holds the rows of kMergeFirst blocks in flight (the first
  // ones requested with the blocks' (m, l)): four when the grid of the wider
  // kernel (about four blocks per SM) fits one wave, else two (seven per SM)
  const dim3 mgrid(kH / kMergeWarps, a.batch);
  if ((long long)a.batch * (kH / kMergeWarps) <= 4LL * a.n_splits)
    return launch_pdl(decode_tc_merge_kernel<4>, mgrid, dim3(kMergeWarps * 32), 0, stream, a);
  return launch_pdl(decode_tc_merge_kernel<2>, mgrid, dim3(kMergeWarps * 32), 0, stream, a);
}

}  // namespace v4kv
