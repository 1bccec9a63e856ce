// Decode attention on the tcgen05 tensor cores for 64 query heads sharing one
// K = V vector per item (P1 §2.1: shared K/V; §2.3: raw-token window).
//
// Per tile of 128 items (entries or window tokens) of one sequence:
//   S^T[128 x 64] = V[128 x 512] . Q^T          (M = items, N = heads, K = dims)
//   P' = 2^(S^T * c_j + log2|ks_j| - m_h)       (CUDA cores, one thread per item)
//   O^T[512 x 64] += V^T[512 x 128] . P'^T      (M = dims in 4 tiles of 128)
//
// fp8 tiles (the compressed entries; an fp8 window) run a software pipeline:
//   * The fp8 codes of the tile go from global memory through registers into
//     tensor memory unchanged (items as lanes, four codes per column). The
//     first product reads them from there as the A operand (kind::f8f6f4), so
//     V costs no shared-memory bandwidth in it. The query enters as three
//     exact e4m3 terms (q = hi + mid + lo after a power-of-two scaling, about
//     12 significant bits): three MMAs per 32-dim step share the A operand and
//     accumulate into the same scores.
//   * The second product needs V^T in f16 from shared memory. The converter
//     warps read the codes back from tensor memory chunk by chunk (128 dims),
//     convert them exactly to f16 and store them into a ring of three 32 KB
//     chunk slots that the second product drains M-tile by M-tile.
//   * Order on the tensor pipe: QK(t+1), PV(t), QK(t+2), PV(t+1), ... so the
//     softmax of tile t runs while PV(t-1) and QK(t+1) execute.
// bf16 tiles (a bf16 window or bf16 entries) run one at a time: the f16 query
// image and the tile's f16 values fill shared memory and both products read
// them there (kind::f16).
//
// The entry's fp32 scale ks_j enters the score multiplier c_j and, through
// log2|ks_j|, the exponent, so P' is the weight of the raw code vector; its
// sign enters P'. The normaliser is sum_j |P'_hj| / |ks_j| (a zero scale is
// a zero-valued item of score 0). m_h is a reference maximum per head, raised
// only when a score exceeds it by more than 2^8 (P' <= 256), at which point
// O^T and the partial sums are rescaled. The normalisers of each row (one per
// head) live in tensor memory.
//
// Warp roles (512 threads): warps 0-3 run the softmax (warp q owns tile rows
// 32q .. 32q + 31, its tensor-memory lane quarter, all 64 heads); warps 4-11
// convert (warp w: rows 32(w%4) + 16((w-4)/4) .. + 15); warp 12 allocates
// tensor memory and one of its lanes issues every MMA; warps 13 and 14
// resolve the rows of the even and odd tiles up to kRing - 1 ahead and
// prefetch them into L2; warp 15 copies the query images.
//
// Schedule: the kernel is persistent. The tiles of all sequences form one
// list (each sequence: its window tiles first, then its entries padded to
// whole tiles); block c processes the tile range [x0[c], x0[c+1]) that the
// prep kernel balanced by estimated cost. A block writes one partial result
// (O, m, l) per sequence it touches into slot b + c, which is unique because
// b + c increases strictly along the tile list; the merge kernel combines
// the slots of each sequence.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace v4kv {

namespace {

constexpr int kH = 64;          // heads (MMA N)
constexpr int kD = 512;         // dims
constexpr int kT = 128;         // items per tile (MMA M of the first product)
constexpr int kThreads = 512;
constexpr float kTau = 8.f;     // rescale when a score exceeds the reference by 2^8
constexpr float kNone = -1e30f; // reference maximum before any item

constexpr int kMmaWarp = 12;
constexpr int kAddrWarp = 13;   // 13 and 14
constexpr int kLoadWarp = 15;

// shared memory map (bytes from a 1024-aligned base)
//   fp8 tiles:  Q3 image [0, 96K), chunk ring slots [96K, 192K), P' [192K, 208K)
//   bf16 tiles: f16 query image [0, 64K), f16 tile [64K, 192K), P' [192K, 208K)
constexpr uint32_t kQ3Off = 0;         // 3 terms x 4 chunks x (64 rows x 128 B)
constexpr uint32_t kQ3Bytes = 98304;
constexpr uint32_t kRingOff = 98304;   // 3 slots x (2 dim atoms x 128 rows x 128 B)
constexpr uint32_t kSlotBytes = 32768;
constexpr uint32_t kQhOff = 0;         // f16 query: 8 dim atoms x 64 rows x 128 B
constexpr uint32_t kVhOff = 65536;     // f16 tile: 8 dim atoms x 128 rows x 128 B
constexpr uint32_t kPOff = 196608;     // 128 rows x 128 B (64 heads f16)
constexpr int kRing = 6;               // tiles of row addresses kept ready
constexpr uint32_t kMetaOff = 212992;                 // [kRing][128] fp32 item scales
constexpr uint32_t kPtrOff = kMetaOff + kRing * 512;  // [kRing][128] row addresses (null = skip)
constexpr uint32_t kMrefOff = kPtrOff + kRing * 1024; // [64] reference max per head
constexpr uint32_t kAlphaOff = kMrefOff + 256;        // [64] rescale factors
constexpr uint32_t kRedOff = kAlphaOff + 256;         // [4][64] per-warp reductions
constexpr uint32_t kBarOff = kRedOff + 1024;          // mbarriers
constexpr uint32_t kMiscOff = kBarOff + 512;          // tmem address, flags, range
constexpr uint32_t kSmemBytes = kMiscOff + 64 + 1024; // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per block");
static_assert(kRingOff + 3 * kSlotBytes == kPOff && kVhOff + 8 * 16384 == kPOff, "map");

// tensor memory columns: fp8 tile [0, 128), S [128, 192), O^T 4 x 64 at
// [192, 448), normalisers [448, 512)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kVCol = 0;
constexpr uint32_t kSCol = 128;
constexpr uint32_t kOCol = 192;
constexpr uint32_t kLCol = 448;

struct Bars {
  uint64_t addr_ready[kRing];  // 32 arrivals (an address warp)
  uint64_t addr_free[kRing];   // 384 arrivals (converters and softmax)
  uint64_t vt_full;            // 256: an fp8 tile is in tensor memory
  uint64_t qk8_done;           // commit: the fp8 tile's first product has read it
  uint64_t s_full;             // commit: scores of the next tile ready
  uint64_t s_free;             // 128: the softmax holds the scores in registers
  uint64_t p_full;             // 128: P' of the next tile stored
  uint64_t pv_done;            // commit: the tile's second product is complete
  uint64_t v_full[3];          // 256: a ring slot holds its f16 chunk
  uint64_t v_empty[3];         // commit: the M-tile that read the slot is complete
  uint64_t sv_full;            // 256: a bf16 tile is in shared memory as f16
  uint64_t ring_free;          // commit before a bf16 tile: every earlier MMA complete
  uint64_t ser_done;           // commit: a bf16 tile's products are complete
  uint64_t q3_ready;           // tx: a Q3 image landed
  uint64_t qh_ready;           // tx: an f16 query image landed
  uint64_t q_free;             // commit: the last first product of a run read its image
  uint64_t o_free;             // 128: the segment epilogue has read O^T
  uint64_t drain;              // commit: every MMA issued
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// 2^x on the special-function unit (ftz: results below 2^-126 become 0)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int ordered_key(float f) {
  int k = __float_as_int(f);
  return k >= 0 ? k : (k ^ 0x7fffffff);
}
__device__ __forceinline__ float from_ordered_key(int k) {
  return __int_as_float(k >= 0 ? k : (k ^ 0x7fffffff));
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
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

// One sequence's items: window tiles first (tokens [w0, L)), then its
// selected entries padded to whole tiles.
struct Seq {
  int L, n_sel, n_win, w0, nwt, nmt;
};

__device__ __forceinline__ Seq seq_of(const DecodeArgs& a, int b) {
  Seq s;
  const int L = min(max(0, a.seq_lens[b]), a.max_len);
  s.L = L;
  const int n_vis = max(0, L - a.window_len) / a.ratio;
  s.n_sel = a.topk ? a.k : n_vis;
  s.w0 = max(0, L - a.window_len);
  s.n_win = L - s.w0;
  s.nwt = (s.n_win + kT - 1) / kT;
  s.nmt = (s.n_sel + kT - 1) / kT;
  return s;
}

__device__ __forceinline__ int tiles_of(const Seq& s) { return s.nwt + s.nmt; }

// tile lt of a sequence holds fp8 codes (else bf16)
__device__ __forceinline__ bool tile_fp8(const DecodeArgs& a, const Seq& s, int lt) {
  return (lt < s.nwt ? a.window.dtype : a.main.dtype) == V4KV_FP8_E4M3;
}

// Estimated cost of a sequence's tiles in the sweep: fp8 tiles 4, bf16 tiles
// 12 (they run one at a time), and 4 for opening a segment (query copy,
// epilogue).
constexpr int kCostFp8 = 4, kCostBf16 = 12, kCostSeg = 4;

__device__ __forceinline__ long long seq_cost(const DecodeArgs& a, const Seq& s) {
  if (tiles_of(s) == 0) return 0;
  const int cw = a.window.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  const int cm = a.main.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  return kCostSeg + (long long)s.nwt * cw + (long long)s.nmt * cm;
}

// tile of sequence s at which `off` cost units (from the sequence's start)
// fall, clamped to the sequence's tiles
__device__ __forceinline__ int tile_at_cost(const DecodeArgs& a, const Seq& s, long long off) {
  const int cw = a.window.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  const int cm = a.main.dtype == V4KV_FP8_E4M3 ? kCostFp8 : kCostBf16;
  off -= kCostSeg;
  if (off <= 0) return 0;
  if (off < (long long)s.nwt * cw) return (int)(off / cw);
  const long long k = s.nwt + (off - (long long)s.nwt * cw) / cm;
  return (int)min(k, (long long)(tiles_of(s) - 1));
}

// Walks a block's tile range: sequence b, tile lt of nt in that sequence.
struct Cursor {
  int b, lt, nt;
  Seq s;
};

__device__ __forceinline__ void cursor_set(Cursor& c, const DecodeArgs& a, int b, int lt) {
  c.b = b;
  c.lt = lt;
  c.s = seq_of(a, b);
  c.nt = tiles_of(c.s);
}

__device__ __forceinline__ void cursor_next(Cursor& c, const DecodeArgs& a) {
  ++c.lt;
  while (c.lt >= c.nt && c.b + 1 < a.batch) {
    ++c.b;
    c.lt = 0;
    c.s = seq_of(a, c.b);
    c.nt = tiles_of(c.s);
  }
}

// Where tile i of a block's range stands: its kind and whether it opens or
// closes its segment (the block's part of one sequence) and its run (the
// segment's consecutive tiles of one kind, which share a query image).
struct TileFlags {
  bool fp8, seg_first, seg_last, run_first, run_last;
};

__device__ __forceinline__ TileFlags flags_of(const DecodeArgs& a, const Cursor& c, int i,
                                              int n_tiles) {
  TileFlags f;
  f.fp8 = tile_fp8(a, c.s, c.lt);
  f.seg_first = i == 0 || c.lt == 0;
  f.seg_last = i == n_tiles - 1 || c.lt == c.nt - 1;
  f.run_first = f.seg_first || tile_fp8(a, c.s, c.lt - 1) != f.fp8;
  f.run_last = f.seg_last || tile_fp8(a, c.s, c.lt + 1) != f.fp8;
  return f;
}

// mbar_wait for a whole warp: every lane waits and the warp agrees on the
// result, so that it stays converged for the .sync.aligned instructions after
__device__ __forceinline__ bool warp_wait(uint64_t* bar, int phase, volatile int* abort) {
  return __all_sync(0xffffffffu, tc::mbar_wait(bar, (uint32_t)(phase & 1), abort));
}

__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Address warp: lane l resolves rows l, l+32, l+64, l+96 of tile lt of
// sequence b into the row-address and scale tables (nullptr for a skipped
// item), then asks L2 for the rows' cache lines so that the converters'
// loads find them there. The loads go in phases (top-k indices, block-table
// entries, scales), each phase's four loads independent of one another, so a
// tile costs three memory latencies rather than twelve. Problems are flagged
// as V4KV_DEV_* bits.
__device__ __forceinline__ void resolve_tile(const DecodeArgs& a, int b, const Seq& s, int lt,
                                             int lane, const uint8_t** rp, float* ms) {
  const bool main_tile = lt >= s.nwt;  // a tile is all entries or all window
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
    j[r] = -1;
    if (main_tile) {
      const int it = (lt - s.nwt) * kT + lane + 32 * r;
      if (it < s.n_sel) j[r] = a.topk ? (long long)a.topk[(size_t)b * a.k + it] : (long long)it;
    } else {
      const int w = lt * kT + lane + 32 * r;
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
  const int lines = fp8 ? kD / 128 : 2 * kD / 128;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    if (p[r])
      for (int k = 0; k < lines; ++k) prefetch_l2_line(p[r] + 128 * k);
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

// 4 fp8 codes (one word, lowest byte first) -> 4 f16 values as two words
__device__ __forceinline__ void fp8x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = h2u(e4m3x2_to_half2((uint16_t)(w & 0xffffu)));
  hi = h2u(e4m3x2_to_half2((uint16_t)(w >> 16)));
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
    const float x = __uint_as_float(w[i] << 16), y = __uint_as_float(w[i] & 0xffff0000u);
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y), "f"(x));
    o[i] = r;
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

constexpr uint32_t kQhImg = kH * kD * 2;  // one f16 query image
constexpr uint32_t kQ3Img = kQ3Bytes;     // one three-term fp8 query image
constexpr int kMaxSplits = 160;           // sweep blocks at most (the plan caps the grid)
constexpr int kPrepCache = 2048;          // batches whose prefix sums the prep keeps in shared memory

// Sum 32 per-lane values over the 32 lanes of a warp (reduce-scatter): lane l
// ends with the sum of value `rev` where the lane bits pick halves (bit 4: 16
// values, bit 3: 8, ... bit 0: 1). Returns that value's index.
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
      v[k] = mine + __shfl_xor_sync(0xffffffffu, other, off);
    }
    if (upper) base += n;
  }
  out1[0] = v[0];
  return base;
}

// Column (0..31) of a 128-dim chunk of the fp8 tile in tensor memory that
// holds the four codes of dims d4 .. d4 + 3 (d4 a multiple of 4). A converter
// thread writes, for p = lane % 4, the words of its 16-byte loads at bytes
// 16p .. 16p + 15 and 64 + 16p .. 64 + 16p + 15 of the chunk into the
// columns its .16x256b registers map to (8k + 2p + e for its word 2k + e), so
// the columns hold the dims in this order; the Q3 image orders its K axis the
// same way.
__device__ __forceinline__ int chunk_dim_col(int d4) {
  const int hi = d4 >= 64;
  const int rel = d4 - 64 * hi;
  const int p = rel >> 4;
  const int j = 4 * hi + ((rel & 15) >> 2);
  return 8 * (j >> 1) + 2 * p + (j & 1);
}

// Converter: the codes of rows rA and rB of the tile whose row addresses are
// rp, each 128-dim chunk c as the 16 registers of a .16x256b store (bytes
// 16p .. 16p + 15 and 64 + 16p .. 64 + 16p + 15 of the chunk)
__device__ __forceinline__ void conv_load(const uint8_t* const* rp, int rA, int rB, int p,
                                          uint32_t (&raw)[4][16]) {
  const uint8_t* pa = rp[rA];
  const uint8_t* pb = rp[rB];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 a0 = make_uint4(0, 0, 0, 0), b0 = a0, a1 = a0, b1 = a0;
    if (pa) {
      a0 = ldg_stream(pa + 128 * c + 16 * p);
      b0 = ldg_stream(pa + 128 * c + 64 + 16 * p);
    }
    if (pb) {
      a1 = ldg_stream(pb + 128 * c + 16 * p);
      b1 = ldg_stream(pb + 128 * c + 64 + 16 * p);
    }
    uint32_t* r = raw[c];
    r[0] = a0.x; r[1] = a0.y; r[2] = a1.x; r[3] = a1.y;
    r[4] = a0.z; r[5] = a0.w; r[6] = a1.z; r[7] = a1.w;
    r[8] = b0.x; r[9] = b0.y; r[10] = b1.x; r[11] = b1.y;
    r[12] = b0.z; r[13] = b0.w; r[14] = b1.z; r[15] = b1.w;
  }
}

// Converter: one chunk (16 registers in .16x256b order) of rows rA, rB as f16
// into ring position gpos, once the second product has released the slot
__device__ __forceinline__ bool conv_store(uint8_t* sm, Bars* bars, volatile int* abort_flag,
                                           const uint32_t (&r)[16], int gpos, int rA, int rB, int p) {
  const int slot = gpos % 3, use = gpos / 3;
  if (use > 0 && !warp_wait(&bars->v_empty[slot], use - 1, abort_flag)) return false;
  uint8_t* base = sm + kRingOff + slot * kSlotBytes;
#pragma unroll
  for (int half = 0; half < 2; ++half) {     // bytes 16p.. (atom 0) and 64 + 16p.. (atom 1)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {         // rows rA, rB
      const int row = rr ? rB : rA;
      uint32_t h[8];
#pragma unroll
      for (int k = 0; k < 2; ++k)            // words 4(2 half + k) + 2 rr + 0/1
#pragma unroll
        for (int e = 0; e < 2; ++e)
          fp8x4_to_f16(r[4 * (2 * half + k) + 2 * rr + e], h[4 * k + 2 * e], h[4 * k + 2 * e + 1]);
      uint8_t* at = base + half * 16384;
      *reinterpret_cast<uint4*>(at + tc::sw128_off(row, 2 * p)) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(at + tc::sw128_off(row, 2 * p + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
    }
  }
  tc::fence_proxy_async_smem();
  tc::mbar_arrive(&bars->v_full[slot]);
  return true;
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
  float* mref = reinterpret_cast<float*>(sm + kMrefOff);
  float* alpha = reinterpret_cast<float*>(sm + kAlphaOff);
  float* red = reinterpret_cast<float*>(sm + kRedOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kMiscOff + 4);
  int* range = reinterpret_cast<int*>(sm + kMiscOff + 16);  // x0, x1, b0, lt0

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

  // barriers and tensor memory first: this overlaps the query-preparation
  // kernel still running ahead of this one
  if (tid == 0) {
    for (int k = 0; k < kRing; ++k) {
      tc::mbar_init(&bars->addr_ready[k], 32);
      tc::mbar_init(&bars->addr_free[k], 384);
    }
    tc::mbar_init(&bars->vt_full, 256);
    tc::mbar_init(&bars->qk8_done, 1);
    tc::mbar_init(&bars->s_full, 1);
    tc::mbar_init(&bars->s_free, 128);
    tc::mbar_init(&bars->p_full, 128);
    tc::mbar_init(&bars->pv_done, 1);
    for (int s = 0; s < 3; ++s) {
      tc::mbar_init(&bars->v_full[s], 256);
      tc::mbar_init(&bars->v_empty[s], 1);
    }
    tc::mbar_init(&bars->sv_full, 256);
    tc::mbar_init(&bars->ring_free, 1);
    tc::mbar_init(&bars->ser_done, 1);
    tc::mbar_init(&bars->q3_ready, 1);
    tc::mbar_init(&bars->qh_ready, 1);
    tc::mbar_init(&bars->q_free, 1);
    tc::mbar_init(&bars->o_free, 128);
    tc::mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(tmem_slot, kTmemCols);
  if (tid < kH) mref[tid] = kNone;
  tc::pdl_wait();  // the tile prefix sums and query images are complete from here on
  tc::pdl_launch_dependents();

  // ---- this block's tile range [x0, x1) and the sequence of its first tile
  if (tid == 0) {
    const int x0 = a.cta_x0[cta], x1 = a.cta_x0[cta + 1];
    const int b0 = x0 < x1 ? a.cta_b0[cta] : a.batch;
    range[0] = x0;
    range[1] = (b0 < a.batch) ? x1 : x0;
    range[2] = b0;
    range[3] = b0 < a.batch ? x0 - a.cum[b0] : 0;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const int x0 = range[0], x1 = range[1];
  const int n_tiles = x1 - x0;
  const int b0 = range[2], lt0 = range[3];
  const uint32_t tmem = *tmem_slot;
  if (x0 >= x1) {
    if (warp == kMmaWarp) tc::tmem_free(tmem, kTmemCols);
    return;
  }

  if (warp == kAddrWarp || warp == kAddrWarp + 1) {
    // ======================= address resolution + L2 prefetch, up to kRing - 1 tiles ahead
    // (warp 13 the even tiles, warp 14 the odd ones)
    const int aw = warp - kAddrWarp;
    Cursor cu;
    cursor_set(cu, a, b0, lt0);
    if (aw) cursor_next(cu, a);
    for (int t = aw; t < n_tiles; t += 2) {
      const int buf = t % kRing;
      if (t >= kRing && !warp_wait(&bars->addr_free[buf], (t - kRing) / kRing, abort_flag)) break;
      resolve_tile(a, cu.b, cu.s, cu.lt, lane, rowptr + buf * kT, meta + buf * kT);
      __syncwarp();
      tc::mbar_arrive(&bars->addr_ready[buf]);
      cursor_next(cu, a);
      cursor_next(cu, a);
    }
  } else if (warp == kLoadWarp) {
    // ======================= query images: one per run of same-kind tiles
    // (Q3 for fp8 runs, the f16 image for bf16 runs), each copied once the
    // run before it has finished reading the region
    Cursor cu;
    cursor_set(cu, a, b0, lt0);
    int runs = 0, n_ser = 0, last3 = -1, lasth = -1;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const TileFlags f = flags_of(a, cu, i, n_tiles);
      if (f.run_first) {
        if (runs > 0) ok = warp_wait(&bars->q_free, runs - 1, abort_flag);
        // the Q3 image also covers the first chunk of the f16 tile area
        if (ok && f.fp8 && n_ser > 0) ok = warp_wait(&bars->ser_done, n_ser - 1, abort_flag);
        if (!ok) break;
        if (lane == 0) {
          if (f.fp8) {
            tc::mbar_arrive_expect_tx(&bars->q3_ready, kQ3Img);
            const uint8_t* src = a.q3 + (size_t)cu.b * kQ3Img;
            for (int k = 0; k < 6; ++k)
              tc::bulk_load(sbase + kQ3Off + k * (kQ3Img / 6), src + k * (kQ3Img / 6), kQ3Img / 6,
                            &bars->q3_ready);
          } else {
            tc::mbar_arrive_expect_tx(&bars->qh_ready, kQhImg);
            const uint8_t* src = a.qh + (size_t)cu.b * kQhImg;
            for (int k = 0; k < 4; ++k)
              tc::bulk_load(sbase + kQhOff + k * (kQhImg / 4), src + k * (kQhImg / 4), kQhImg / 4,
                            &bars->qh_ready);
          }
        }
        if (f.fp8) ++last3; else ++lasth;
        ++runs;
      }
      if (!f.fp8) ++n_ser;
      cursor_next(cu, a);
    }
    // every copy has landed before shared memory is released (normally long
    // since; after an abort one may still be in flight)
    volatile int never = 0;
    if (last3 >= 0 && !tc::mbar_wait(&bars->q3_ready, last3 & 1, &never)) flag(a.dev_status, V4KV_DEV_TIMEOUT);
    if (lasth >= 0 && !tc::mbar_wait(&bars->qh_ready, lasth & 1, &never)) flag(a.dev_status, V4KV_DEV_TIMEOUT);
    if (!ok) {
      *abort_flag = 1;
      flag(a.dev_status, V4KV_DEV_TIMEOUT);
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer
    // The whole warp runs the loop, so descriptors, addresses and wait results
    // stay warp-uniform; one lane, elected once, issues every MMA and commit
    // (a commit tracks the MMAs of the thread that issues it).
    const bool leader = tc::elect_one();
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t id8 = tc::idesc_f16(128, kH, 0, 0);   // e4m3 x e4m3 -> f32 (format fields 0)
    const uint32_t iq = tc::idesc_f16(128, kH, 0, 0);
    const uint32_t ip = tc::idesc_f16(128, kH, 1, 1);
    const uint64_t q3_desc = tc::sw128_desc(sbase + kQ3Off, 16, 1024);     // Q3 terms, K-major
    const uint64_t qh_desc = tc::sw128_desc(sbase + kQhOff, 16, 1024);     // f16 Q, K-major
    const uint64_t vk_desc = tc::sw128_desc(sbase + kVhOff, 16, 1024);     // f16 tile, K-major
    const uint64_t vm_desc = tc::sw128_desc(sbase + kVhOff, 16384, 1024);  // f16 tile^T, MN-major
    const uint64_t rm_desc = tc::sw128_desc(sbase + kRingOff, 16384, 1024);  // ring slot^T, MN-major
    const uint64_t p_desc = tc::sw128_desc(sbase + kPOff, 0, 1024);        // P^T, MN-major
    Cursor cu;
    cursor_set(cu, a, b0, lt0);
    bool ok = true;
    int n8 = 0, nser = 0, nrun3 = 0, nrunh = 0, nseg = 0;
    int pend = -1, pend_chunk = 0, pend_seg = 0;
    bool pend_first = false;
    auto wait = [&](uint64_t* bar, int phase) -> bool {
      return __all_sync(0xffffffffu, tc::mbar_wait_spin(bar, phase & 1, abort_flag));
    };
    // second product of fp8 tile j (its chunks at ring positions g0 .. g0 + 3)
    auto pv8 = [&](int j, int g0, bool first, int seg) -> bool {
      if (!wait(&bars->p_full, j)) return false;
      if (first && seg > 0 && !wait(&bars->o_free, seg - 1)) return false;
      for (int mt = 0; mt < 4; ++mt) {
        const int g = g0 + mt, slot = g % 3;
        if (!wait(&bars->v_full[slot], g / 3)) return false;
        tc::tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16(tm + kOCol + kH * mt,
                        rm_desc + (uint64_t)((slot * kSlotBytes + kk * 2048) >> 4),
                        p_desc + (uint64_t)((kk * 2048) >> 4), ip, (!first || kk > 0) ? 1u : 0u);
          tc::mma_commit(&bars->v_empty[slot]);
        }
        __syncwarp();
      }
      if (leader) tc::mma_commit(&bars->pv_done);
      __syncwarp();
      return true;
    };
    for (int i = 0; i < n_tiles && ok; ++i) {
      const TileFlags f = flags_of(a, cu, i, n_tiles);
      if (f.seg_first && i > 0) ++nseg;
      if (f.fp8) {
        // ---- first product of fp8 tile i: A = codes in tensor memory, B = Q3 terms
        ok = wait(&bars->vt_full, n8);
        if (ok && f.run_first) ok = wait(&bars->q3_ready, nrun3);
        if (ok && i > 0) ok = wait(&bars->s_free, i - 1);
        if (!ok) break;
        tc::tc_fence_after();
        if (leader) {
#pragma unroll 1
          for (int ks = 0; ks < 16; ++ks) {
#pragma unroll
            for (int term = 0; term < 3; ++term)
              tc::mma_f8_ts(tm + kSCol, tm + kVCol + 8 * ks,
                            q3_desc + (uint64_t)(((term * 4 + (ks >> 2)) * 8192 + (ks & 3) * 32) >> 4),
                            id8, (ks > 0 || term > 0) ? 1u : 0u);
          }
          tc::mma_commit(&bars->s_full);
          tc::mma_commit(&bars->qk8_done);
          if (f.run_last) tc::mma_commit(&bars->q_free);
        }
        __syncwarp();
        if (f.run_first) ++nrun3;
        // ---- second product of the previous fp8 tile
        if (pend >= 0 && !(ok = pv8(pend, pend_chunk, pend_first, pend_seg))) break;
        pend = i;
        pend_chunk = 4 * n8;
        pend_first = f.seg_first;
        pend_seg = nseg;
        ++n8;
      } else {
        // ---- bf16 tile: drain, then both products from shared memory
        if (pend >= 0) {
          if (!(ok = pv8(pend, pend_chunk, pend_first, pend_seg))) break;
          pend = -1;
        }
        if (leader) tc::mma_commit(&bars->ring_free);
        __syncwarp();
        ok = wait(&bars->sv_full, nser);
        if (ok && f.run_first) ok = wait(&bars->qh_ready, nrunh);
        if (ok && i > 0) ok = wait(&bars->s_free, i - 1);
        if (!ok) break;
        tc::tc_fence_after();
        if (leader) {
#pragma unroll 4
          for (int kk = 0; kk < 32; ++kk)
            tc::mma_f16(tm + kSCol, vk_desc + (uint64_t)((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                        qh_desc + (uint64_t)((((kk >> 2) * 8192) + (kk & 3) * 32) >> 4), iq,
                        kk > 0 ? 1u : 0u);
          tc::mma_commit(&bars->s_full);
          if (f.run_last) tc::mma_commit(&bars->q_free);
        }
        __syncwarp();
        if (f.run_first) ++nrunh;
        ok = wait(&bars->p_full, i);
        if (ok && f.seg_first && nseg > 0) ok = wait(&bars->o_free, nseg - 1);
        if (!ok) break;
        tc::tc_fence_after();
        if (leader) {
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc::mma_f16(tm + kOCol + kH * mt, vm_desc + (uint64_t)((2 * mt * 16384 + kk * 2048) >> 4),
                          p_desc + (uint64_t)((kk * 2048) >> 4), ip, (!f.seg_first || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(&bars->pv_done);
          tc::mma_commit(&bars->ser_done);
        }
        __syncwarp();
        ++nser;
      }
      cursor_next(cu, a);
    }
    if (ok && pend >= 0) ok = pv8(pend, pend_chunk, pend_first, pend_seg);
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
  } else if (warp >= 4) {
    // ======================= converters (warps 4-11)
    // Warp (q, g) = (warp % 4, (warp - 4) / 4) owns tile rows R0 .. R0 + 15,
    // R0 = 32q + 16g. In the .16x256b shape, lane l holds rows R0 + l/4 and
    // R0 + l/4 + 8 and, of every 128-dim chunk, the bytes 16p .. 16p + 15 and
    // 64 + 16p .. 64 + 16p + 15 (p = l % 4): 64 contiguous bytes of a row per
    // warp load, the same 16 bytes per thread in registers, tensor memory and
    // the f16 ring.
    const int q = warp & 3, g = (warp - 4) >> 2;
    const int R0 = 32 * q + 16 * g;
    const int rA = R0 + (lane >> 2), rB = rA + 8, p = lane & 3;
    const uint32_t tl = tmem + ((uint32_t)R0 << 16);
    uint32_t raw[4][16];     // a tile's codes, per chunk in the .16x256b register order
    uint32_t held[16];       // chunk 3 of the last fp8 tile, read back from tensor memory
    int held_g = -1;         // its ring position (-1: none)
    bool have_raw = false;
    bool wide = false;       // a bf16 value outside the f16 range was clamped
    bool ok = true;
    int n8 = 0, nser = 0;
    bool ser_pending = false;  // a bf16 tile has used the ring area since the last ring write

    Cursor cu;
    cursor_set(cu, a, b0, lt0);
    for (int i = 0; i < n_tiles && ok; ++i) {
      const TileFlags f = flags_of(a, cu, i, n_tiles);
      if (f.fp8) {
        if (!have_raw) {
          if (!(ok = warp_wait(&bars->addr_ready[i % kRing], i / kRing, abort_flag))) break;
          conv_load(rowptr + (i % kRing) * kT, rA, rB, p, raw);
        }
        // the tensor-memory tile is free once the previous fp8 tile's first
        // product has read it (this warp read its own rows back already)
        if (n8 > 0 && !(ok = warp_wait(&bars->qk8_done, n8 - 1, abort_flag))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_st16x256_x4(tl + kVCol + 32 * c, raw[c]);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bars->vt_full);
        tc::mbar_arrive(&bars->addr_free[i % kRing]);
        have_raw = false;
        // the next fp8 tile's codes fly while this one is converted
        if (i + 1 < n_tiles) {
          Cursor nx = cu;
          cursor_next(nx, a);
          if (tile_fp8(a, nx.s, nx.lt)) {
            if (!(ok = warp_wait(&bars->addr_ready[(i + 1) % kRing], (i + 1) / kRing, abort_flag))) break;
            conv_load(rowptr + ((i + 1) % kRing) * kT, rA, rB, p, raw);
            have_raw = true;
          }
        }
        if (ser_pending) {
          if (!(ok = warp_wait(&bars->ser_done, nser - 1, abort_flag))) break;
          ser_pending = false;
        }
        // the previous fp8 tile's last chunk (its slot frees when the second
        // product of that tile has read its first chunk)
        if (held_g >= 0) {
          if (!(ok = conv_store(sm, bars, abort_flag, held, held_g, rA, rB, p))) break;
          held_g = -1;
        }
        // chunks 0-2 of this tile from tensor memory into the ring, chunk 3
        // into registers (so that the next tile may overwrite tensor memory)
        for (int c = 0; c < 3 && ok; ++c) {
          uint32_t r[16];
          tc::tmem_ld16x256_x4(tl + kVCol + 32 * c, r);
          tc::tmem_wait_ld();
          ok = conv_store(sm, bars, abort_flag, r, 4 * n8 + c, rA, rB, p);
        }
        if (!ok) break;
        tc::tmem_ld16x256_x4(tl + kVCol + 96, held);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        held_g = 4 * n8 + 3;
        ++n8;
      } else {
        // ---- bf16 tile into the f16 area, once every earlier MMA has completed
        if (held_g >= 0) {
          if (!(ok = conv_store(sm, bars, abort_flag, held, held_g, rA, rB, p))) break;
          held_g = -1;
        }
        if (!(ok = warp_wait(&bars->ring_free, nser, abort_flag))) break;
        if (!(ok = warp_wait(&bars->addr_ready[i % kRing], i / kRing, abort_flag))) break;
        const uint8_t* const* rp = rowptr + (i % kRing) * kT;
        // lane covers rows R0 + 2r + lane/16 (r = 0..7), 16 bytes at
        // 16 * (lane % 16) of each 256-byte (128-dim) chunk
        const int part = lane & 15;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint4 v[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint8_t* pr = rp[R0 + 2 * r + (lane >> 4)];
            v[r] = pr ? ldg_stream(pr + 256 * c + 16 * part) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint32_t vr = R0 + 2 * r + (lane >> 4);
            const uint32_t atom = 2 * c + (part >> 3);
            *reinterpret_cast<uint4*>(sm + kVhOff + atom * 16384 + tc::sw128_off(vr, part & 7)) =
                bf16x8_to_f16(v[r], wide);
          }
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bars->sv_full);
        tc::mbar_arrive(&bars->addr_free[i % kRing]);
        ++nser;
        ser_pending = true;
      }
      cursor_next(cu, a);
    }
    if (ok && held_g >= 0) ok = conv_store(sm, bars, abort_flag, held, held_g, rA, rB, p);
    if (!ok) {
      *abort_flag = 1;
      flag(a.dev_status, V4KV_DEV_TIMEOUT);
    }
    if (__any_sync(0xffffffffu, wide) && lane == 0) flag(a.dev_status, V4KV_DEV_RANGE);
  } else {
    // ======================= softmax (warps 0-3)
    // Thread (warp q, lane l) owns tile row 32q + l (its TMEM lane) for all 64
    // heads; its partial normalisers live in tensor memory (columns kLCol ..).
    // The four warps meet at named barrier 1 after every bounded wait, so they
    // leave together when one gives up.
    const int q = warp;
    const int row = 32 * q + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const uint32_t l_addr = lane_base + kLCol;
    {
      uint32_t z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0u;
      tc::tmem_st32(l_addr, z);
      tc::tmem_st32(l_addr + 32, z);
      tc::tmem_wait_st();
    }
    Cursor cu;
    cursor_set(cu, a, b0, lt0);
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const TileFlags f = flags_of(a, cu, i, n_tiles);
      const float k0 = f.fp8 ? a.qk08[cu.b] : a.qk0[cu.b];
      ok = tc::mbar_wait(&bars->addr_ready[i % kRing], (i / kRing) & 1, abort_flag) &&
           tc::mbar_wait_spin(&bars->s_full, i & 1, abort_flag, 32);
      ok = !named_or(1, 128, !ok);
      if (!ok) break;
      tc::tc_fence_after();
      float u[64];  // scores in log2 units including log2|ks|, then u - m_ref
      {
        uint32_t* r = reinterpret_cast<uint32_t*>(u);
        tc::tmem_ld32(lane_base + kSCol, r);
        tc::tmem_ld32(lane_base + kSCol + 32, r + 32);
        tc::tmem_wait_ld();
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&bars->s_free);
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
      float dmax = -INFINITY;
      {
        const float4* mr4 = reinterpret_cast<const float4*>(mref);
#pragma unroll
        for (int h4 = 0; h4 < 16; ++h4) {
          const float4 m4 = mr4[h4];
#pragma unroll
          for (int e = 0; e < 4; ++e) u[4 * h4 + e] = fmaf(u[4 * h4 + e], cj, lk);
          dmax = fmaxf(dmax, fmaxf(fmaxf(u[4 * h4] - m4.x, u[4 * h4 + 1] - m4.y),
                                   fmaxf(u[4 * h4 + 2] - m4.z, u[4 * h4 + 3] - m4.w)));
        }
      }
      bool waited = false;  // pv_done of tile i - 1 has been waited for
      if (named_or(1, 128, dmax > kTau)) {
        // rare: raise the reference of every head to its running maximum; the
        // earlier tiles' products must be complete before O^T is rescaled
        if (i > 0) {
          ok = tc::mbar_wait(&bars->pv_done, (i - 1) & 1, abort_flag);
          ok = !named_or(1, 128, !ok);
          if (!ok) break;
          waited = true;
          tc::tc_fence_after();
        }
#pragma unroll
        for (int h = 0; h < 64; ++h) {
          const int wm = __reduce_max_sync(0xffffffffu, ordered_key(u[h]));
          if (lane == 0) red[q * 64 + h] = from_ordered_key(wm);
        }
        named_sync(1, 128);
        if (tid < kH) {
          const float old = mref[tid];
          float nm = old;
#pragma unroll
          for (int w = 0; w < 4; ++w) nm = fmaxf(nm, red[64 * w + tid]);
          alpha[tid] = exp2f(old - nm);
          mref[tid] = nm;
        }
        named_sync(1, 128);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t lv[32];
          tc::tmem_ld32(l_addr + 32 * half, lv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 32; ++h)
            lv[h] = __float_as_uint(__uint_as_float(lv[h]) * alpha[32 * half + h]);
          tc::tmem_st32(l_addr + 32 * half, lv);
        }
        tc::tmem_wait_st();
        if (!f.seg_first) {
          // O^T rows of this lane (dims 128 mt + row) times alpha per head column
#pragma unroll 1
          for (int mt = 0; mt < 4; ++mt) {
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
        named_sync(1, 128);  // red and alpha are free again
      }
      // P' row of this item (64 heads f16, eight 16-byte chunks of the swizzled
      // MN-major row) once the previous tile's second product has read P'
      if (i > 0 && !waited) {
        ok = tc::mbar_wait(&bars->pv_done, (i - 1) & 1, abort_flag);
        ok = !named_or(1, 128, !ok);
        if (!ok) break;
      }
      {
        const float4* mr4 = reinterpret_cast<const float4*>(mref);
#pragma unroll
        for (int h4 = 0; h4 < 16; ++h4) {
          const float4 m4 = mr4[h4];
          u[4 * h4] = fast_exp2(u[4 * h4] - m4.x);
          u[4 * h4 + 1] = fast_exp2(u[4 * h4 + 1] - m4.y);
          u[4 * h4 + 2] = fast_exp2(u[4 * h4 + 2] - m4.z);
          u[4 * h4 + 3] = fast_exp2(u[4 * h4 + 3] - m4.w);
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = 8 * c + 2 * e;
          pk[e] = h2u(__floats2half2_rn(sgn * u[h], sgn * u[h + 1]));
        }
        *reinterpret_cast<uint4*>(sm + kPOff + tc::sw128_off(row, c)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bars->p_full);
      tc::mbar_arrive(&bars->addr_free[i % kRing]);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t lv[32];
        tc::tmem_ld32(l_addr + 32 * half, lv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h)
          lv[h] = __float_as_uint(fmaf(u[32 * half + h], inv_k, __uint_as_float(lv[h])));
        tc::tmem_st32(l_addr + 32 * half, lv);
      }
      tc::tmem_wait_st();

      if (f.seg_last) {
        // ---- segment epilogue: partial result of (sequence b, block cta) in
        // slot b + cta, O^T un-normalised, relative to the reference maximum
        ok = tc::mbar_wait(&bars->pv_done, i & 1, abort_flag);
        ok = !named_or(1, 128, !ok);
        if (!ok) break;
        tc::tc_fence_after();
        const size_t prow = ((size_t)cu.b + cta) * kH;
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
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
        // normaliser: sum the 128 rows' partial sums per head
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float lsum[32];
          {
            uint32_t lv[32];
            tc::tmem_ld32(l_addr + 32 * half, lv);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) lsum[e] = __uint_as_float(lv[e]);
          }
          float two[1];
          const int hb = warp_reduce_scatter32(lsum, lane, two);
          red[q * 64 + 32 * half + hb] = two[0];
        }
        named_sync(1, 128);
        if (tid < kH) {
          const float l = red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
          a.part_ml[(prow + tid) * 2] = mref[tid];
          a.part_ml[(prow + tid) * 2 + 1] = l;
          mref[tid] = kNone;
        }
        {
          uint32_t z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0u;
          tc::tmem_st32(l_addr, z);
          tc::tmem_st32(l_addr + 32, z);
          tc::tmem_wait_st();
        }
        named_sync(1, 128);
        tc::tc_fence_before();
        tc::mbar_arrive(&bars->o_free);
      }
      cursor_next(cu, a);
    }
    if (!ok) {
      *abort_flag = 1;
      flag(a.dev_status, V4KV_DEV_TIMEOUT);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_free(tmem, kTmemCols);
  }
}

// grid (heads / 8, batch), 256 threads: warp w merges head 8 * blockIdx.x + w
// of sequence b over the blocks whose tile ranges met it (lane l: dims 16l ..
// 16l + 15), normalises, applies the inverse RoPE at position L - 1 (cos/sin
// from the prep kernel's table) and stores bf16.
__global__ void __launch_bounds__(256) decode_tc_merge_kernel(DecodeArgs a) {
  __shared__ float w_sh[8][kMaxSplits];  // per warp: the blocks' weights
  tc::pdl_wait();  // the sweep's partial results are complete from here on
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = 8 * blockIdx.x + warp, b = blockIdx.y;
  const int2 sl = a.seq_slots[b];
  const int lo = sl.x, hi = sl.y;
  float M = -INFINITY;
  for (int c = lo + lane; c <= hi; c += 32) {
    const bool empty = a.cta_x0[c + 1] <= a.cta_x0[c];
    const float m = empty ? -INFINITY : a.part_ml[(((size_t)b + c) * kH + h) * 2];
    w_sh[warp][c - lo] = m;
    M = fmaxf(M, m);
  }
  M = warp_max(M);
  float L = 0.f;
  for (int c = lo + lane; c <= hi; c += 32) {
    const float m = w_sh[warp][c - lo];
    const float w = m == -INFINITY ? 0.f : exp2f(m - M);
    w_sh[warp][c - lo] = w;
    if (w > 0.f) L = fmaf(w, a.part_ml[(((size_t)b + c) * kH + h) * 2 + 1], L);
  }
  L = warp_sum(L);
  __syncwarp();
  const int d0 = 16 * lane;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int c = lo; c <= hi; ++c) {
    const float w = w_sh[warp][c - lo];
    if (w == 0.f) continue;
    const float4* o4 = reinterpret_cast<const float4*>(a.part_o + (((size_t)b + c) * kH + h) * kD + d0);
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = o4[q];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[4 * q] = fmaf(w, v[q].x, acc[4 * q]);
      acc[4 * q + 1] = fmaf(w, v[q].y, acc[4 * q + 1]);
      acc[4 * q + 2] = fmaf(w, v[q].z, acc[4 * q + 2]);
      acc[4 * q + 3] = fmaf(w, v[q].w, acc[4 * q + 3]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] *= inv;
  const int Lb = min(a.seq_lens[b], a.max_len);
  if (a.rope.rope_dim > 0 && Lb > 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int d = d0 + 2 * k;
      if (d >= a.rope.rope_offset && d + 1 < a.rope.rope_offset + a.rope.rope_dim) {
        const int i = (d - a.rope.rope_offset) >> 1;
        float c, s;
        if (i < kRopeTable) {
          const float2 cs = a.rope_tab[(size_t)b * kRopeTable + i];
          c = cs.x;
          s = cs.y;
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

// grid (batch + 1), 256 threads. Block b < batch writes sequence b's query
// images for the sweep's B operands:
//   * f16, scaled by 2^e so that max|q| * 2^e < 2^15, eight 64-dim atoms of
//     64 head rows x 128 B in the 128-byte swizzle (one linear copy puts it in
//     place), and qk0[b] = sm_scale * log2(e) * 2^-e;
//   * three e4m3 terms: x = q * 2^e8 with max|x| in [128, 256), hi = e4m3(x),
//     mid = e4m3(x - hi), lo = e4m3(x - hi - mid) (round to nearest even; the
//     residuals are exact in fp32), each as four 128-dim chunks of 64 head
//     rows x 128 B in the 128-byte swizzle, the K axis of a chunk in the order
//     the converters leave the codes in tensor memory (chunk_dim_col); and
//     qk08[b] = sm_scale * log2(e) * 2^-e8.
// Block `batch` writes the tile prefix sums, the cost prefix sums and every
// sweep block's range.
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
    // the prefix sums also go to shared memory (when they fit) for the
    // binary searches below, which would otherwise chain global loads
    __shared__ int cum_sh[kPrepCache + 1];
    __shared__ long long ccum_sh[kPrepCache + 1];
    const bool cached = a.batch <= kPrepCache;
    int carry = 0;
    long long ccarry = 0;
    for (int base = 0; base < a.batch; base += 256) {
      const int bb = base + t;
      int n = 0;
      long long cost = 0;
      if (bb < a.batch) {
        if (a.seq_lens[bb] > a.max_len) flag(a.dev_status, V4KV_DEV_OVERFLOW);
        const Seq sq = seq_of(a, bb);
        n = tiles_of(sq);
        cost = seq_cost(a, sq);
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
    __syncthreads();  // the prefix sums are visible to the whole block
    const int* cum = cached ? cum_sh : a.cum;
    const long long* costcum = cached ? ccum_sh : a.costcum;
    const int G = a.n_splits;
    for (int c = t; c <= G; c += 256) {
      int x0 = carry, b0 = a.batch;
      if (c < G && ccarry > 0) {
        const long long target = (long long)c * ccarry / G;
        int l = 0, r = a.batch - 1;  // last sequence whose cost prefix is <= target
        while (l < r) {
          const int m = (l + r + 1) >> 1;
          if (costcum[m] <= target) l = m; else r = m - 1;
        }
        b0 = l;
        const Seq sq = seq_of(a, b0);
        x0 = cum[b0] + tile_at_cost(a, sq, target - costcum[b0]);
      }
      a.cta_x0[c] = x0;
      if (c < G) a.cta_b0[c] = b0;
      x0_sh[c] = x0;
    }
    __syncthreads();
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
  int e = 0, e8 = 0;
  if (amax > 0.f) {
    int k;
    frexpf(amax, &k);  // 2^(k-1) <= amax < 2^k
    e = 15 - k;
    e8 = 8 - k;        // max|q| * 2^e8 in [128, 256)
  }
  const float qs = ldexpf(1.f, e);
  const float qs8 = ldexpf(1.f, e8);
  uint8_t* img = a.qh + (size_t)b * kQhImg;
  uint8_t* img3 = a.q3 + (size_t)b * kQ3Img;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int u = t + 256 * k;
    const int h = u / (kD / 8), c8 = u % (kD / 8);  // 8-dim chunk c8 of head h
    uint32_t hv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) hv[i] = h2u(__floats2half2_rn(x[k][2 * i] * qs, x[k][2 * i + 1] * qs));
    *reinterpret_cast<uint4*>(img + (c8 >> 3) * 8192 + tc::sw128_off(h, c8 & 7)) =
        make_uint4(hv[0], hv[1], hv[2], hv[3]);
    // the three fp8 terms of these 8 dims (dims 8 c8 .. 8 c8 + 7 lie in
    // 128-dim chunk c8 / 16, as two groups of four)
    const int c = c8 >> 4, dl = 8 * (c8 & 15);
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t w3[3] = {0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float xv = x[k][4 * g + i] * qs8;
        const uint8_t hi = (uint8_t)__nv_cvt_float_to_fp8(xv, __NV_SATFINITE, __NV_E4M3);
        const float r1 = xv - e4m3_to_float(hi);
        const uint8_t mid = (uint8_t)__nv_cvt_float_to_fp8(r1, __NV_SATFINITE, __NV_E4M3);
        const float r2 = r1 - e4m3_to_float(mid);
        const uint8_t lo = (uint8_t)__nv_cvt_float_to_fp8(r2, __NV_SATFINITE, __NV_E4M3);
        w3[0] |= (uint32_t)hi << (8 * i);
        w3[1] |= (uint32_t)mid << (8 * i);
        w3[2] |= (uint32_t)lo << (8 * i);
      }
      // byte position of the column in the chunk's 128-byte K row
      const int kb = 4 * chunk_dim_col(dl + 4 * g);
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        uint8_t* at = img3 + (term * 4 + c) * 8192 + tc::sw128_off(h, kb >> 4) + (kb & 15);
        *reinterpret_cast<uint32_t*>(at) = w3[term];
      }
    }
  }
  if (t == 0) {
    a.qk0[b] = a.sm_scale * 1.4426950408889634f * ldexpf(1.f, -e);
    a.qk08[b] = a.sm_scale * 1.4426950408889634f * ldexpf(1.f, -e8);
  }
  // cos/sin of the inverse RoPE at the query position, for the merge
  if (t < kRopeTable && 2 * t < a.rope.rope_dim) {
    const int Lb = min(a.seq_lens[b], a.max_len);
    float c = 1.f, s = 0.f;
    if (Lb > 0) rope_cs(a.rope, t, (long long)Lb - 1, &c, &s);
    a.rope_tab[(size_t)b * kRopeTable + t] = make_float2(c, s);
  }
}

// workspace of the tensor-core path: query images (f16 and three-term fp8),
// their multipliers, partial results (o, m, l) per slot, tile prefix sums
size_t decode_tc_workspace_bytes(int batch, int num_sms) {
  const size_t slots = (size_t)batch + num_sms;
  const size_t qk0 = ((size_t)batch * sizeof(float) + 255) / 256 * 256;
  return (size_t)batch * kQhImg + (size_t)batch * kQ3Img + 2 * qk0 +
         slots * kH * (size_t)(kD + 2) * sizeof(float) + ((size_t)batch + 1) * sizeof(int32_t) + 256 +
         ((size_t)batch + 1) * sizeof(long long) + (2 * (size_t)num_sms + 1) * sizeof(int32_t) + 256 +
         (size_t)batch * sizeof(int2) + 256 + (size_t)batch * kRopeTable * sizeof(float2) + 256;
}

void decode_tc_layout(DecodeArgs& a, void* workspace) {
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const size_t slots = (size_t)a.batch + a.n_splits;
  a.qh = w;
  w += (size_t)a.batch * kQhImg;
  a.q3 = w;
  w += (size_t)a.batch * kQ3Img;
  a.qk0 = reinterpret_cast<float*>(w);
  w += ((size_t)a.batch * sizeof(float) + 255) / 256 * 256;
  a.qk08 = reinterpret_cast<float*>(w);
  w += ((size_t)a.batch * sizeof(float) + 255) / 256 * 256;
  a.part_o = reinterpret_cast<float*>(w);
  a.part_ml = a.part_o + slots * kH * kD;
  a.cum = reinterpret_cast<int32_t*>(a.part_ml + slots * kH * 2);
  uint8_t* c = reinterpret_cast<uint8_t*>(a.cum + a.batch + 1);
  c = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(c) + 255) & ~uintptr_t(255));
  a.costcum = reinterpret_cast<long long*>(c);
  a.cta_x0 = reinterpret_cast<int32_t*>(a.costcum + a.batch + 1);
  a.cta_b0 = a.cta_x0 + a.n_splits + 1;
  uint8_t* q = reinterpret_cast<uint8_t*>(a.cta_b0 + a.n_splits);
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
  return launch_pdl(decode_tc_merge_kernel, dim3(kH / 8, a.batch), dim3(256), 0, stream, a);
}

}  // namespace v4kv
