// SubBlock block selection (xiaodao.ai "MiniMax-H3 的 6.24 倍，不能直接算成六倍
// 产能", section "6.24 倍里，真正有损的部分大约是三倍": query and key are cut into
// 64-token blocks, the key blocks that contribute little are estimated and
// only the high-scoring ones are kept; chat-gpts.plus "MiniMax-H3 在 8×H200 上
// 基准测试…", section "事件核心：发生了什么": blocks below a threshold are
// skipped).
//
// Scores on tensor cores.  A work item is 128 query blocks of one (batch,
// head), one per TMEM lane.  The block scores s_ij = q_bar_i . k_bar_j are
// fp32 dot products; the tensor core computes them from tf32 pieces: x = hi +
// lo with hi = x with its low 13 mantissa bits cleared (exactly a tf32 value)
// and lo = x - hi, and s = hi_q.hi_k + hi_q.lo_k + lo_q.hi_k (kind::tf32, fp32
// accumulation; the dropped lo.lo term and the tf32 reading of lo leave an
// error of a few 1e-6 of |q_bar_i| |k_bar_j|).  A pass over the row streams
// the key blocks in tiles of 128: M = 128 query blocks, N = 128 key blocks,
// K = 8 channels per MMA, 16 K-steps x 3 products per tile into one of two
// accumulators of 128 TMEM columns, so that the tensor core fills one while
// the other is read.  The same inputs and instruction sequence give the same
// scores in every pass.
//   * Q pieces: the selector threads load their query block's mean (each of
//     the two selector warpgroups half of the channels), split it and store
//     hi / lo into the block's TMEM lane (the A operand).
//   * K pieces: a TMA warp streams k_bar in stages of 128 key blocks x 32
//     channels (one 128-byte swizzle row of fp32 per key block), four stages
//     deep; four converter warps split each stage in place into hi (where TMA
//     wrote it) and lo (a second buffer with the same swizzled positions).
//   * The tiles of a pass alternate between the two selector warpgroups: the
//     first takes tiles 0, 1, 2, ... (accumulator 0), the second tiles T-1,
//     T-2, ... (accumulator 1).
// Exact top-K per row, in up to four passes over the scores (three when
// compaction and output merge):
//   1. sample: one tile of every ceil(nblk/128)-th key block, one product
//      (hi.hi); mean m and deviation sd of the row's sampled scores place a
//      window of 1.5 sd around m + z sd, z the normal quantile of the kept
//      fraction;
//   2. histogram: 128 bins, bin(s) = round(clamp(s * A + B, 0, 127)), a
//      non-decreasing function of s; bins 1 .. 126 cover the window, 0 and
//      127 everything below and above it; u32 counts per row in shared
//      memory (a warp's 32 rows hit 32 banks) by adds without a result and
//      without a branch; the bin holding the (K-1)-th largest off-diagonal
//      score follows from the counts;
//   3. compaction: the scores of that bin (a few dozen at most) go to
//      shared memory with their block index; the (K-1)-th largest under the
//      order (score descending, block index ascending) among them is the cut;
//      for nblk <= 2048 this pass also sets the output bitmask of every block
//      above the bin, and the candidates at or above the cut are added to it
//      afterwards, so that the output pass is not needed;
//   4. output: the diagonal and every block at or above the cut.  For nblk
//      <= 4096 each thread sets one bit per kept block in a shared-memory
//      bitmask; at the next item's start (while the tensor core begins that
//      item) the selector warps write the rows, word by word, a word's kept
//      blocks in one store of consecutive entries.  Beyond 4096 each
//      warpgroup writes its own tiles' blocks from its end of the row (the
//      first forward, the second backward from the last position).
// The histogram's counts decide each item's remaining passes: when some
// row's bin holds more than the merged pass's 20 slots per warpgroup, the
// item runs compaction (40 slots) and output as separate passes; when some
// bin holds more than 40 blocks (a sample that misplaced the window, or mass
// ties), it runs instead six radix levels restricted to that bin: the four
// bytes of an order-preserving key of the score, then the two bytes of
// (65535 - block index), which fixes the cut exactly.  Threshold mode (keep
// s >= tau) and the trivial budgets run the output pass alone.
//
// Roles (512 threads, one CTA per SM, persistent over work items):
//   warp 0: TMA producer           warp 1: TMEM allocator + MMA issuer
//   warps 4-7: converters          warps 8-15: two selector warpgroups
//                                  (TMEM lane quarter = warp % 4)
// The producer warpgroups give up registers (80 per thread) to the selector
// warpgroups (176), whose chunk code is unrolled over 32 scores.
// Every mbarrier wait is bounded; a failed wait is shared with the other
// selector warpgroup at the next named barrier, after which the kernel stores
// nothing more, lets its own copies and MMAs finish, frees TMEM and returns.
#include "internal.h"

namespace sbattn {

namespace {

constexpr int kThreads = 512;
constexpr int kRows = 128;                    // query blocks per work item (MMA M)
constexpr int kTileN = 128;                   // key blocks per tile (MMA N)
constexpr int kChunkD = 32;                   // channels per stage (128 bytes of fp32)
constexpr int kChunks = kHeadDim / kChunkD;   // 4
constexpr int kStages = 4;                    // a stage: one tile x one chunk of 32 channels
constexpr int kHalfBytes = kTileN * kChunkD * 4;      // 16 KB: hi (TMA target) or lo
constexpr int kStageBytes = 2 * kHalfBytes;
// One 64 KB region of shared memory, zero between uses, serves in turn as
//   * the window histogram: u32 counts [bin][row], 128 bins (a warp's 32
//     rows hit 32 banks whatever their bins);
//   * the candidates of the boundary bin: f32 scores [wg][slot][row], then
//     u16 block indices [wg][slot][row] (from 32 KB on, 20 slots, when the
//     bitmask of a merged compaction-and-output pass holds the first 32 KB);
//   * the kept-block bitmask: u32 words [word][row ^ (word % 32)], 32 blocks
//     per word (nblk <= 4096); the xor spreads both a warp's 32 rows of one
//     word and one row's 32 words over the 32 banks;
//   * the fallback's byte histograms: u16 counts [digit][row], 256 digits.
constexpr int kWinBins = 128;
constexpr int kBins = 256;
constexpr int kHistBytes = kBins * kRows * 2;         // 64 KB
constexpr int kOffHist = kStages * kStageBytes;       // 128 KB
// Candidates per row and selector warpgroup: 40 when they have the region to
// themselves (scores at 0, indices after them), 20 when the merged pass keeps
// the bitmask in the region's first 32 KB (scores at 32 KB, then indices).
constexpr int kCap = 40, kCapMerged = 20;
constexpr int kMergedMaxTiles = 16;                   // bitmask of 64 words per row = 32 KB
constexpr int kOffCandMerged = 32 * 1024;
static_assert(2 * kCap * kRows * 6 <= kHistBytes, "candidates fit the shared region");
static_assert(kOffCandMerged + 2 * kCapMerged * kRows * 6 <= kHistBytes, "merged candidates fit behind the bitmask");
static_assert(kMergedMaxTiles * 4 * kRows * 4 <= kOffCandMerged, "merged bitmask fits before the candidates");
static_assert(kWinBins * kRows * 4 <= kHistBytes, "window histogram fits the shared region");
constexpr int kMaskWords = kHistBytes / (kRows * 4);  // 128 words: 4096 blocks per row
constexpr int kOffMisc = kOffHist + kHistBytes;       // 192 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQhi = 0, kColQlo = 128, kColD = 256;  // accumulator b at kColD + 128 b
constexpr int kLevels = 6;                    // fallback: 4 key bytes + 2 index bytes
constexpr float kWindowSd = 0.75f;            // half-width of the histogram window, in sd
// registers: the selectors' unrolled chunk code takes the producers' share
constexpr uint32_t kRegsProducers = 80, kRegsSelectors = 176;
static_assert(256 * kRegsProducers + 256 * kRegsSelectors == kThreads * 128, "register split = 512 x 128");

enum PassKind { kSample = 0, kHist = 1, kCompact = 2, kLevel = 3, kOutput = 4, kMerged = 5 };
enum Verdict { kFast = 0, kSplit = 1, kSlow = 2 };

struct Misc {
  uint64_t raw_full[kStages], conv_full[kStages], stage_empty[kStages];
  uint64_t d_full[2], d_empty[2];  // accumulator b belongs to selector warpgroup b
  uint64_t q_ready, q_empty;       // the item's Q pieces in TMEM
  uint64_t plan;                   // one phase per item: its verdict is in plan_verdict
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int plan_verdict;
  // per query block of the item, written by the first selector warpgroup
  float bin_a[kRows], bin_b[kRows], cut_s[kRows];
  int cut_j[kRows], tb[kRows];
  uint32_t kpre[kRows], kmask[kRows], vpre[kRows], vmask[kRows];
  int n0[kRows], n1[kRows], need[kRows], w0[kRows], w1[kRows];
};
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc);

// kind::tf32 instruction descriptor: fp32 D, tf32 A and B (format code 2),
// both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTileN >> 3) << 17) |
                            ((uint32_t)(kRows >> 4) << 24);

SB_DEV void umma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

SB_DEV void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Named barriers of the 256 selector threads: a plain one, and reductions of
// a predicate over all of them.
SB_DEV void sel_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
SB_DEV bool sel_and(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\tbar.red.and.pred b, 2, 256, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}
SB_DEV bool sel_or(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\tbar.red.or.pred b, 3, 256, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}

// Monotone map from float to uint32 (larger float -> larger key); adding
// +0 first turns -0 into +0, so that the two zeros are equal keys.
SB_DEV uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}
SB_DEV float key_value(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k); }

// Window bin of a score: round(clamp(s * A + B, 0, 127)).  The window maps
// to bins 1 .. 126; bin 0 holds everything below it and bin 127 everything
// above.  Each step is non-decreasing in s (fma, max, min, and rounding to an
// integer by adding 1.5 * 2^23), so a higher bin means a strictly higher
// score.
SB_DEV uint32_t bin_of(float s, float A, float B) {
  const float x = fminf(fmaxf(fmaf(s, A, B), 0.0f), 127.0f);
  return __float_as_uint(x + 12582912.0f) & 0x7Fu;
}

SB_DEV uint32_t tf32_hi(uint32_t u) { return u & 0xFFFFE000u; }


// The schedule every role walks: work items (128 query blocks of one
// batch-head) strided over the grid, passes, the tiles of a pass (in the
// order tile_of gives) and the four channel chunks of a tile.
struct Plan {
  int items, row_blocks, tiles, stride, ns;
  bool general;  // budget form with 1 < keep < nblk
  bool bitmask;  // kept blocks gathered in shared memory, written row by row
  bool merged;   // compaction and output in one pass (bitmask and candidates share the region)
  SB_DEV void init(const SelectArgs& a) {
    row_blocks = (a.nblk + kRows - 1) / kRows;
    items = a.B * a.H * row_blocks;
    tiles = (a.nblk + kTileN - 1) / kTileN;
    stride = (a.nblk + kTileN - 1) / kTileN;  // sampled blocks: j = m * stride, m < ns <= 128
    ns = (a.nblk + stride - 1) / stride;
    general = !a.threshold_mode && a.keep > 1 && a.keep < a.nblk;
    bitmask = a.nblk <= kMaskWords * 32;
    merged = general && tiles <= kMergedMaxTiles;
  }
  // The histogram's verdict on an item: kFast (every boundary bin fits the
  // candidate slots), kSplit (some bin needs the larger slots of a separate
  // compaction pass), kSlow (some bin is too large: radix levels).  Passes of
  // an item; the producers assume four until they read the verdict, before
  // the fourth.
  SB_DEV bool merged_for(int v) const { return merged && v == kFast; }
  SB_DEV int total(int v) const { return general ? (v == kSlow ? 3 + kLevels : (merged_for(v) ? 3 : 4)) : 1; }
  SB_DEV int total_before_verdict() const { return general ? 4 : 1; }
  SB_DEV int kind(int p, int v) const {
    if (!general) return kOutput;
    if (p == 0) return kSample;
    if (p == 1) return kHist;
    if (v != kSlow) return p == 2 ? (merged_for(v) ? kMerged : kCompact) : kOutput;
    return p < 2 + kLevels ? kLevel : kOutput;
  }
  SB_DEV int ntiles(int kind) const { return kind == kSample ? 1 : tiles; }
};
// Position pos of a pass -> tile: even positions ascend from tile 0, odd ones
// descend from the last tile.
SB_DEV int tile_of(int pos, int tiles) { return (pos & 1) ? tiles - 1 - (pos >> 1) : (pos >> 1); }

// Shared-memory stores and adds on 32-bit shared addresses (no address-space
// conversion per element); the add returns nothing, so nothing waits for it.
SB_DEV void sts_u32(uint32_t a, uint32_t v) { asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory"); }
SB_DEV void red_add(uint32_t a, uint32_t v) { asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory"); }
// Stores under a predicate, with no branch around them (a divergent branch
// per element costs more than the work it skips).
SB_DEV void stg_s32_if(bool p, int32_t* a, int32_t v) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.global.s32 [%0], %1;\n\t}\n" ::"l"(a), "r"(v),
               "r"((uint32_t)p)
               : "memory");
}
SB_DEV void sts_u32_if(bool p, uint32_t a, uint32_t v) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.shared.u32 [%0], %1;\n\t}\n" ::"r"(a), "r"(v),
               "r"((uint32_t)p)
               : "memory");
}
SB_DEV void sts_u16_if(bool p, uint32_t a, uint32_t v) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.shared.u16 [%0], %1;\n\t}\n" ::"r"(a),
               "h"((unsigned short)v), "r"((uint32_t)p)
               : "memory");
}

// What one selector thread carries through a tile.
struct Row {
  int i, nblk, r;           // my query block, key blocks, my row within the item
  bool row;                 // i < nblk
  float A, B;               // window bin map
  uint32_t tb;              // the bin being resolved
  float cs;                 // cut: keep s > cs, or s == cs and j <= cj
  int cj;
  uint32_t kpre, kmask, vpre, vmask, sh;  // fallback radix state
  bool vlevel;              // fallback level on the block index bytes
  uint32_t h32;             // shared address of my window-histogram column: + bin * 512
  uint32_t hw;              // shared address of my u16 byte-histogram word: + digit * 256
  uint32_t inc;             // my half of that word
  bool bitmask;             // output into the shared bitmask
  uint32_t mask;            // its shared address
  uint32_t cs_addr;         // shared address of my candidate scores: + slot * 512
  uint32_t cj_addr;         // ... and of their block indices: + slot * 256
  int n, cap_slots;         // candidates found, room for them
  int32_t* out;             // my output row
  int w, top;               // kept blocks written; first position of the second warpgroup
  bool desc;                // second warpgroup: writes backwards from top
  int cap;
  float* srow;              // scores dump row or null
  float sum, sq;            // sampled scores
  int ns_seen;
  int stride, ns;
};

// Output decision for block j with score bits u: the diagonal and every block
// at or above the cut are written, in my direction.
template <bool Checks>
SB_DEV void output_one(uint32_t u, int j, Row& R) {
  if (Checks && j >= R.nblk) return;
  const float s = __uint_as_float(u);
  if (R.srow != nullptr) R.srow[j] = s;
  const bool kept = (Checks && j == R.i) || s > R.cs || (s == R.cs && j <= R.cj);
  if (kept) {
    const int pos = R.desc ? R.top - R.w : R.w;
    if (pos >= 0 && pos < R.cap) R.out[pos] = j;  // bounded by the row's capacity
    ++R.w;
  }
}

// One chunk of 32 scores of my row, block indices j0 .. j0+31 (sample pass:
// sample indices j0 .. j0+31).  Checks: the tile holds the diagonal or runs
// past nblk (or is the sample), so each element is tested; elsewhere the
// loops have no branch but the rare candidate store.
template <int Kind, bool Checks>
SB_DEV void scan_chunk(const uint32_t (&v)[32], int j0, Row& R) {
  if (Kind == kSample) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int m = j0 + e, j = m * R.stride;
      const float s = __uint_as_float(v[e]);
      const bool use = ((uint32_t)(m < R.ns) & (uint32_t)(j != R.i)) != 0u;
      R.sum += use ? s : 0.0f;
      R.sq = fmaf(use ? s : 0.0f, s, R.sq);
      R.ns_seen += use ? 1 : 0;
    }
  } else if (Kind == kHist) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = j0 + e;
      const uint32_t b = bin_of(__uint_as_float(v[e]), R.A, R.B);
      const uint32_t valid = Checks ? ((uint32_t)(j < R.nblk) & (uint32_t)(j != R.i)) : 1u;
      red_add(R.h32 + b * 512u, valid);
    }
  } else if (Kind == kCompact) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = j0 + e;
      const float s = __uint_as_float(v[e]);
      uint32_t take = (uint32_t)(bin_of(s, R.A, R.B) == R.tb);
      if (Checks) take &= (uint32_t)(j < R.nblk) & (uint32_t)(j != R.i);
      const bool room = (take & (uint32_t)(R.n < R.cap_slots)) != 0u;
      sts_u32_if(room, R.cs_addr + (uint32_t)R.n * 512u, v[e]);
      sts_u16_if(room, R.cj_addr + (uint32_t)R.n * 256u, (uint32_t)j);
      R.n += (int)take;
    }
  } else if (Kind == kMerged) {
    // compaction of the boundary bin and the bitmask of the blocks above it
    // (and the diagonal) in one sweep
    uint32_t m = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = j0 + e;
      const float s = __uint_as_float(v[e]);
      const uint32_t b = bin_of(s, R.A, R.B);
      const uint32_t valid = Checks ? ((uint32_t)(j < R.nblk) & (uint32_t)(j != R.i)) : 1u;
      const uint32_t take = (uint32_t)(b == R.tb) & valid;
      const bool room = (take & (uint32_t)(R.n < R.cap_slots)) != 0u;
      sts_u32_if(room, R.cs_addr + (uint32_t)R.n * 512u, v[e]);
      sts_u16_if(room, R.cj_addr + (uint32_t)R.n * 256u, (uint32_t)j);
      R.n += (int)take;
      uint32_t kept = (uint32_t)(b > R.tb) & valid;
      if (Checks) kept |= (uint32_t)(j == R.i);
      m |= kept << e;
    }
    if (R.srow != nullptr) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (!Checks || j0 + e < R.nblk) R.srow[j0 + e] = __uint_as_float(v[e]);
    }
    const uint32_t w = (uint32_t)j0 >> 5;
    sts_u32(R.mask + (w * kRows + ((uint32_t)R.r ^ (w & 31u))) * 4u, m);
  } else if (Kind == kLevel) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = j0 + e;
      const float s = __uint_as_float(v[e]);
      const uint32_t key = order_key(s), vj = 0xFFFFu - (uint32_t)j;
      uint32_t member = (uint32_t)(bin_of(s, R.A, R.B) == R.tb) & (uint32_t)((key & R.kmask) == R.kpre) &
                        (uint32_t)((vj & R.vmask) == R.vpre);
      if (Checks) member &= (uint32_t)(j < R.nblk) & (uint32_t)(j != R.i);
      const uint32_t digit = ((R.vlevel ? vj : key) >> R.sh) & 0xFFu;
      red_add(R.hw + digit * 256u, member * R.inc);
    }
  } else if (R.bitmask) {  // kOutput into the bitmask: one word per chunk
    uint32_t m = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = j0 + e;
      const float s = __uint_as_float(v[e]);
      // (bitwise, not short-circuit, so that no lane branches)
      uint32_t kept = (uint32_t)(s > R.cs) | ((uint32_t)(s == R.cs) & (uint32_t)(j <= R.cj));
      if (Checks) kept = (kept | (uint32_t)(j == R.i)) & (uint32_t)(j < R.nblk);
      m |= kept << e;
    }
    if (R.srow != nullptr) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (!Checks || j0 + e < R.nblk) R.srow[j0 + e] = __uint_as_float(v[e]);
    }
    const uint32_t w = (uint32_t)j0 >> 5;
    sts_u32(R.mask + (w * kRows + ((uint32_t)R.r ^ (w & 31u))) * 4u, m);
  } else {  // kOutput written directly, in my direction (constant register indices either way)
    if (R.desc) {
#pragma unroll
      for (int e = 31; e >= 0; --e) output_one<Checks>(v[e], j0 + e, R);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) output_one<Checks>(v[e], j0 + e, R);
    }
  }
}

// My 128 columns of accumulator `d` (lane quarter address), in four chunks of
// 32 with the next chunk's load in flight; descending chunk order for the
// backward writer.
template <int Kind, bool Checks>
SB_DEV void scan_tile(uint32_t d, int jbase, Row& R) {
  uint32_t va[32], vb[32];
  const bool back = Kind == kOutput && R.desc;
  tmem_ld_32cols(d + (back ? 96u : 0u), va);
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int ca = back ? 3 - 2 * h : 2 * h, cb = back ? 2 - 2 * h : 2 * h + 1;
    tmem_wait_ld_regs(va);
    tmem_ld_32cols(d + (uint32_t)cb * 32u, vb);
    if (R.row) scan_chunk<Kind, Checks>(va, jbase + ca * 32, R);
    tmem_wait_ld_regs(vb);
    if (h == 0) tmem_ld_32cols(d + (back ? 32u : 64u), va);
    if (R.row) scan_chunk<Kind, Checks>(vb, jbase + cb * 32, R);
  }
}

template <int Kind>
SB_DEV void scan_tile(uint32_t d, int jbase, bool checks, Row& R) {
  if (checks)
    scan_tile<Kind, true>(d, jbase, R);
  else
    scan_tile<Kind, false>(d, jbase, R);
}

// Scan my row's 256 bins from the top (clearing them) for the bin where the
// running count reaches `need`; returns it (or -1) with the count above it
// and its own count.
SB_DEV int find_bin(const uint16_t* hist_row, int need, int& above, int& cnt) {
  uint16_t* h = const_cast<uint16_t*>(hist_row);
  int cum = 0, bin = -1;
  above = 0;
  cnt = 0;
#pragma unroll 4
  for (int b = kBins - 1; b >= 0; --b) {  // (selects, no branch)
    const int c = h[b * kRows];
    h[b * kRows] = 0;
    const bool open = bin < 0;
    const bool hit = open && cum + c >= need;
    bin = hit ? b : bin;
    above = hit ? cum : above;
    cnt = hit ? c : cnt;
    cum += (open && !hit) ? c : 0;
  }
  return bin;
}

// Kept lists of item (bh, rb) from the shared bitmask.  Each of the eight
// selector warps takes every eighth row, four rows at a time (independent
// chains: a warp issues only about one instruction every few cycles, so the
// work per word is kept short and interleaved).  Word by word: lane l keeps
// block 32 w + l if bit l is set and writes it at the row's running count
// plus the set bits below l, so a word's kept blocks go out in one store of
// consecutive entries; then the rows' words are cleared.
SB_DEV void write_rows(uint8_t* smem, const SelectArgs& a, int bh, int rb, int sel_warp, int lane) {
  const int W = (a.nblk + 31) >> 5;
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + kOffHist);
  const uint32_t below = (1u << lane) - 1u;
  for (int r0 = sel_warp; r0 < kRows; r0 += 32) {
    int32_t* orow[4];
    int base[4];
    bool live[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int ii = rb * kRows + r0 + 8 * k;
      live[k] = ii < a.nblk;
      orow[k] = a.kept_idx + ((size_t)bh * a.nblk + (live[k] ? ii : 0)) * a.K_capacity;
      base[k] = 0;
    }
#pragma unroll 2
    for (int w = 0; w < W; ++w) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rr = r0 + 8 * k;
        const uint32_t m = live[k] ? bm[w * kRows + (rr ^ (w & 31))] : 0u;  // (every lane reads the same word)
        const int pos = base[k] + __popc(m & below);
        stg_s32_if(((m >> lane) & 1u) != 0u && pos < a.K_capacity, orow[k] + pos, w * 32 + lane);
        base[k] += __popc(m);
      }
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!live[k]) continue;
      const int rr = r0 + 8 * k;
      for (int w = lane; w < W; w += 32) bm[w * kRows + (rr ^ (w & 31))] = 0u;  // zero for the next histogram
      for (int q = base[k] + lane; q < a.K_capacity; q += 32) orow[k][q] = -1;
      if (lane == 0) a.kept_cnt[(size_t)bh * a.nblk + rb * kRows + rr] = min(base[k], a.K_capacity);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    select_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_s, SelectArgs a,
                  uint64_t wait_limit_ns) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc* ms = reinterpret_cast<Misc*>(smem + kOffMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((smem_addr(smem) & 1023u) != 0u) return;  // swizzle atoms need 1024-byte alignment
  Plan pl;
  pl.init(a);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ms->raw_full[s], 1);
      mbar_init(&ms->conv_full[s], 128);
      mbar_init(&ms->stage_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ms->d_full[b], 1);
      mbar_init(&ms->d_empty[b], 128);
    }
    mbar_init(&ms->q_ready, 256);
    mbar_init(&ms->q_empty, 1);
    mbar_init(&ms->plan, 1);
    mbar_init(&ms->drain, 1);
    ms->abort = 0;
    ms->plan_verdict = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_s);
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // histograms start at zero; every level clears the bins it read and the
  // compaction clears the candidate slots it used
  for (int e = threadIdx.x; e < kHistBytes / 16; e += kThreads)
    reinterpret_cast<uint4*>(smem + kOffHist)[e] = make_uint4(0u, 0u, 0u, 0u);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  volatile int* abort_flag = &ms->abort;
  volatile int* plan_verdict = &ms->plan_verdict;
  const WaitCtl wc{abort_flag, wait_limit_ns};

  if (warp < 8) {
    warpgroup_regs_dec<kRegsProducers>();
    if (warp == 0) {
      // ------------------------------------------------------------- TMA
      bool ok = true;
      uint32_t sc = 0, ic = 0;
      if (lane == 0) {
        for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x, ++ic) {
          const int bh = item / pl.row_blocks;
          int verdict = kFast;
          int total = pl.total_before_verdict();
          for (int p = 0; p < total && ok; ++p) {
            if (pl.general && p == 3) {
              if (!(ok = mbar_wait(&ms->plan, ic & 1, wc))) break;
              verdict = *plan_verdict;
              total = pl.total(verdict);
              if (p >= total) break;
            }
            const int kind = pl.kind(p, verdict), nt = pl.ntiles(kind);
            for (int pos = 0; pos < nt && ok; ++pos) {
              const int tile = tile_of(pos, nt);
              for (int c = 0; c < kChunks && ok; ++c) {
                const int s = sc % kStages;
                if (!(ok = mbar_wait(&ms->stage_empty[s], ((sc / kStages) & 1) ^ 1, wc))) break;
                mbar_arrive_expect_tx(&ms->raw_full[s], kHalfBytes);
                if (kind == kSample)
                  tma_load_3d(smem + s * kStageBytes, &tm_s, &ms->raw_full[s], c * kChunkD, 0, bh);
                else
                  tma_load_3d(smem + s * kStageBytes, &tm_k, &ms->raw_full[s], c * kChunkD, tile * kTileN, bh);
                ++sc;
              }
            }
          }
        }
        if (!ok) {
          *abort_flag = 1;
          // copies already issued land before the CTA exits
          const uint64_t t0 = global_timer_ns();
          for (int s = 0; s < kStages; ++s) {
            const uint32_t n_s = (sc + kStages - 1 - s) / kStages;
            if (n_s > 0)
              while (!mbar_try_wait(&ms->raw_full[s], (n_s - 1) & 1) && global_timer_ns() - t0 < 100000000ull) {
              }
          }
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------- MMA
      bool ok = true;
      if (lane == 0) {
        uint32_t sc = 0, ic = 0, dc0 = 0, dc1 = 0;  // accumulators used so far
        for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x, ++ic) {
          if (!(ok = mbar_wait(&ms->q_ready, ic & 1, wc))) break;
          int verdict = kFast;
          int total = pl.total_before_verdict();
          for (int p = 0; p < total && ok; ++p) {
            if (pl.general && p == 3) {
              if (!(ok = mbar_wait(&ms->plan, ic & 1, wc))) break;
              verdict = *plan_verdict;
              total = pl.total(verdict);
              if (p >= total) break;
            }
            const int kind = pl.kind(p, verdict), nt = pl.ntiles(kind);
            const bool three = kind != kSample;  // the sample needs hi.hi only
            for (int pos = 0; pos < nt && ok; ++pos) {
              const int b = pos & 1;
              if (!(ok = mbar_wait(&ms->d_empty[b], ((b ? dc1 : dc0) & 1) ^ 1, wc))) break;
              tc_fence_after();
              const uint32_t d = tmem + kColD + (uint32_t)b * kTileN;
              for (int c = 0; c < kChunks && ok; ++c, ++sc) {
                const int s = sc % kStages;
                if (!(ok = mbar_wait(&ms->conv_full[s], (sc / kStages) & 1, wc))) break;
                tc_fence_after();
                const uint32_t st = smem_addr(smem + s * kStageBytes);
                const uint64_t bhi0 = smem_desc(st, 16, 1024, kSwizzle128B);
                const uint64_t blo0 = smem_desc(st + kHalfBytes, 16, 1024, kSwizzle128B);
  #pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint32_t ks = (uint32_t)(c * 4 + kk);  // K-step of 8 channels
                  const uint32_t ahi = tmem + kColQhi + ks * 8, alo = tmem + kColQlo + ks * 8;
                  // +32 bytes per K-step inside the 128-byte row = +2 in the address field
                  const uint64_t bhi = bhi0 + (uint64_t)(kk * 2), blo = blo0 + (uint64_t)(kk * 2);
                  umma_tf32_ts(d, ahi, bhi, (c == 0 && kk == 0) ? 0u : 1u);
                  if (three) {
                    umma_tf32_ts(d, ahi, blo, 1u);
                    umma_tf32_ts(d, alo, bhi, 1u);
                  }
                }
                umma_commit(&ms->stage_empty[s]);
              }
              if (ok) {
                umma_commit(&ms->d_full[b]);
                (b ? dc1 : dc0) += 1;
              }
            }
          }
          if (ok) umma_commit(&ms->q_empty);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (lane == 0) {
        if (!ok) *abort_flag = 1;
        umma_commit(&ms->drain);  // every MMA of this thread is done before TMEM is freed
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&ms->drain, 0) && global_timer_ns() - t0 < 100000000ull) {
        }
      }
      __syncwarp();
    } else if (warp >= 4) {
      // ------------------------------------------------------------- converters
      const int tid = threadIdx.x - 128;
      uint32_t sc = 0, ic = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x, ++ic) {
        int verdict = kFast;
        int total = pl.total_before_verdict();
        for (int p = 0; p < total && ok; ++p) {
          if (pl.general && p == 3) {
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ms->plan, ic & 1, wc)))) break;
            verdict = *plan_verdict;
            total = pl.total(verdict);
            if (p >= total) break;
          }
          const int n_stages = pl.ntiles(pl.kind(p, verdict)) * kChunks;
          for (int q = 0; q < n_stages && ok; ++q, ++sc) {
            const int s = sc % kStages;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ms->raw_full[s], (sc / kStages) & 1, wc)))) break;
            uint4* hi = reinterpret_cast<uint4*>(smem + s * kStageBytes);
            uint4* lo = reinterpret_cast<uint4*>(smem + s * kStageBytes + kHalfBytes);
  #pragma unroll 4
            for (int e = tid; e < kHalfBytes / 16; e += 128) {
              const uint4 v = hi[e];
              const uint4 h = make_uint4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
              hi[e] = h;
              lo[e] = make_uint4(__float_as_uint(__uint_as_float(v.x) - __uint_as_float(h.x)),
                                 __float_as_uint(__uint_as_float(v.y) - __uint_as_float(h.y)),
                                 __float_as_uint(__uint_as_float(v.z) - __uint_as_float(h.z)),
                                 __float_as_uint(__uint_as_float(v.w) - __uint_as_float(h.w)));
            }
            fence_proxy_async_smem();  // the pieces are read by the tensor core
            mbar_arrive(&ms->conv_full[s]);
          }
        }
      }
      if (!ok && threadIdx.x == 128) *abort_flag = 1;
    }
  } else {
    warpgroup_regs_inc<kRegsSelectors>();
    // ------------------------------------------------------------- selectors
    const int wg = (warp - 8) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = query block of the item
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    uint16_t* hist_row = reinterpret_cast<uint16_t*>(smem + kOffHist) + r;  // + bin * kRows
    Row R;
    R.nblk = a.nblk;
    const uint32_t region = smem_addr(smem + kOffHist);
    uint32_t* h32 = reinterpret_cast<uint32_t*>(smem + kOffHist) + r;  // my window-histogram column
    // candidate slots: their layout follows each item's verdict
    int cap = kCap;
    float* cand_s = nullptr;
    uint16_t* cand_j = nullptr;
    auto place_candidates = [&](bool merged_item) {
      cap = merged_item ? kCapMerged : kCap;
      float* base = reinterpret_cast<float*>(smem + kOffHist + (merged_item ? kOffCandMerged : 0));
      cand_s = base + wg * cap * kRows + r;
      cand_j = reinterpret_cast<uint16_t*>(base + 2 * cap * kRows) + wg * cap * kRows + r;
      R.cs_addr = smem_addr(cand_s);
      R.cj_addr = smem_addr(cand_j);
      R.cap_slots = cap;
    };
    R.h32 = region + (uint32_t)r * 4u;
    R.hw = region + (uint32_t)(r >> 1) * 4u;
    R.inc = 1u << ((r & 1) * 16);
    R.bitmask = pl.bitmask;
    R.mask = region;
    R.r = r;
    place_candidates(pl.merged);
    R.desc = wg == 1;
    R.cap = a.K_capacity;
    R.stride = pl.stride;
    R.ns = pl.ns;
    // normal quantile of the kept fraction of the off-diagonal blocks
    const float zq = pl.general ? normcdfinvf(1.0f - (float)(a.keep - 1) / (float)(a.nblk - 1)) : 0.0f;
    uint32_t tc = 0, ic = 0;
    int pend_bh = -1, pend_rb = 0;  // an item whose kept lists wait in the bitmask
    bool ok = true;
    for (int item = blockIdx.x; item < pl.items; item += gridDim.x, ++ic) {
      const int bh = item / pl.row_blocks;
      const int rb = item - bh * pl.row_blocks;
      R.i = rb * kRows + r;
      R.row = R.i < a.nblk;
      // ---- my query block's mean (my warpgroup's 64 channels), split into
      // tf32 pieces, into my TMEM lane
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&ms->q_empty, (ic & 1) ^ 1, wc));
      if (ok) {
        tc_fence_after();
        const float4* qrow =
            reinterpret_cast<const float4*>(a.q_bar + ((size_t)bh * a.nblk + (R.row ? R.i : 0)) * kHeadDim) + wg * 16;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          uint32_t hv[32], lv[32];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 v = R.row ? __ldg(qrow + part * 8 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t h = tf32_hi(__float_as_uint(f[k]));
              hv[4 * e + k] = h;
              lv[4 * e + k] = __float_as_uint(f[k] - __uint_as_float(h));
            }
          }
          const uint32_t col = (uint32_t)(wg * 64 + part * 32);
          tmem_st_32cols(lane_addr + kColQhi + col, hv);
          tmem_st_32cols(lane_addr + kColQlo + col, lv);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ms->q_ready);
      }
      if (!(ok = sel_and(ok))) break;
      // ---- the previous item's kept lists, while the tensor core starts on
      // this item's first tiles
      if (pend_bh >= 0) {
        write_rows(smem, a, pend_bh, pend_rb, warp - 8, lane);
        pend_bh = -1;
        sel_sync();  // the bitmask is clear before this item writes into it
      }
      // ---- selection state of my row
      int need = a.keep - 1;  // off-diagonal blocks still to place (budget form)
      if (a.threshold_mode) {
        R.cs = a.tau;
        R.cj = 0xFFFF;
      } else if (a.keep <= 1) {
        R.cs = __int_as_float(0x7f800000);  // +inf: nothing but the diagonal
        R.cj = -1;
      } else {
        R.cs = __int_as_float(0xff800000);  // -inf: everything (general rows set their cut later)
        R.cj = 0xFFFF;
      }
      R.A = 0.0f;
      R.B = 0.0f;
      R.tb = 0;
      R.kpre = R.kmask = R.vpre = R.vmask = 0;
      R.sh = 24;
      R.vlevel = false;
      R.n = 0;
      R.w = 0;
      R.top = a.threshold_mode ? a.K_capacity - 1 : a.keep - 1;
      R.out = a.kept_idx + ((size_t)bh * a.nblk + (R.row ? R.i : 0)) * a.K_capacity;
      R.srow = a.scores != nullptr && R.row ? a.scores + ((size_t)bh * a.nblk + R.i) * a.nblk : nullptr;
      R.sum = R.sq = 0.0f;
      R.ns_seen = 0;
      int verdict = kFast;
      int total = pl.total(kFast);
      for (int p = 0; p < total; ++p) {
        const int kind = pl.kind(p, verdict), nt = pl.ntiles(kind);
        const int mine = wg == 0 ? (nt + 1) / 2 : nt / 2;
        if (kind == kLevel) {
          const int lvl = p - 2;
          R.vlevel = lvl >= 4;
          R.sh = R.vlevel ? (uint32_t)(8 - 8 * (lvl - 4)) : (uint32_t)(24 - 8 * lvl);
        }
        for (int k = 0; k < mine && ok; ++k) {
          const int tile = wg == 0 ? k : nt - 1 - k;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ms->d_full[wg], tc & 1, wc)))) break;
          tc_fence_after();
          const uint32_t d = lane_addr + kColD + (uint32_t)wg * kTileN;
          const int jbase = tile * kTileN;
          const bool checks = kind == kSample || tile == rb || jbase + kTileN > a.nblk;
          switch (kind) {
            case kSample: scan_tile<kSample, true>(d, 0, R); break;
            case kHist: scan_tile<kHist>(d, jbase, checks, R); break;
            case kCompact: scan_tile<kCompact>(d, jbase, checks, R); break;
            case kMerged: scan_tile<kMerged>(d, jbase, checks, R); break;
            case kLevel: scan_tile<kLevel>(d, jbase, checks, R); break;
            default: scan_tile<kOutput>(d, jbase, checks, R); break;
          }
          tc_fence_before();
          mbar_arrive(&ms->d_empty[wg]);
          ++tc;
        }
        if (!(ok = sel_and(ok))) break;  // also: every atomic and slot of the pass is done
        // ---- end of pass
        if (kind == kSample) {
          if (wg == 0) {
            if (R.row) {
              const float cnt = (float)(R.ns_seen > 0 ? R.ns_seen : 1);
              const float mean = R.sum / cnt;
              const float sd = sqrtf(fmaxf(R.sq / cnt - mean * mean, 0.0f));
              const float lo = mean + (zq - kWindowSd) * sd;
              float A = (kWinBins - 2) / (2.0f * kWindowSd * sd);  // bins 1 .. 126 across the window
              float B = 1.0f - lo * A;
              if (!(sd > 0.0f) || !isfinite(A) || !isfinite(B)) A = B = 0.0f;  // one bin: the fallback decides
              ms->bin_a[r] = A;
              ms->bin_b[r] = B;
            }
          }
          sel_sync();
          R.A = ms->bin_a[r];
          R.B = ms->bin_b[r];
        } else if (kind == kHist) {
          bool bad = false, big = false;
          if (wg == 0 && R.row) {
            int cum = 0, tb = -1, above = 0, cnt = 0;
#pragma unroll 4
            for (int b = kWinBins - 1; b >= 0; --b) {  // from the top; clears every bin (selects, no branch)
              const int c = (int)h32[b * kRows];
              h32[b * kRows] = 0u;
              const bool open = tb < 0;
              const bool hit = open && cum + c >= need;
              tb = hit ? b : tb;
              above = hit ? cum : above;
              cnt = hit ? c : cnt;
              cum += (open && !hit) ? c : 0;
            }
            R.tb = tb < 0 ? 0u : (uint32_t)tb;
            need -= above;
            bad = tb < 0 || cnt > kCap;  // (bins 0 and 127, outside the window, are large)
            big = cnt > kCapMerged;
            ms->tb[r] = (int)R.tb;
            ms->need[r] = need;
          }
          const bool slow_item = sel_or(bad);
          const bool split_item = sel_or(big);
          verdict = slow_item ? kSlow : (split_item ? kSplit : kFast);
          if (wg == 0 && r == 0) {
            *plan_verdict = verdict;
            mbar_arrive(&ms->plan);
          }
          total = pl.total(verdict);
          place_candidates(pl.merged_for(verdict));
          R.tb = (uint32_t)ms->tb[r];
        } else if (kind == kCompact || kind == kMerged) {
          // the cut: the candidate with need - 1 candidates before it in
          // (score descending, index ascending) order; each warpgroup ranks
          // its own candidates against all of them
          (wg == 0 ? ms->n0 : ms->n1)[r] = R.n;
          if (wg == 0) {
            ms->cut_s[r] = __int_as_float(0x7f800000);  // (none found: nothing but the diagonal)
            ms->cut_j[r] = -1;
          }
          sel_sync();
          const int n0 = min(ms->n0[r], cap), n1 = min(ms->n1[r], cap);
          float* s0 = cand_s - wg * cap * kRows;  // the first warpgroup's slots, then the second's
          uint16_t* j0 = cand_j - wg * cap * kRows;
          float* s1 = s0 + cap * kRows;
          uint16_t* j1 = j0 + cap * kRows;
          if (R.row && n0 + n1 <= 32) {
            // up to 32 candidates, as 48-bit keys (order key of the score,
            // then 65535 - index) in registers; each warpgroup ranks 16 slots
            const int target = ms->need[r] - 1;
            uint64_t key[32];
#pragma unroll
            for (int y = 0; y < 32; ++y) {
              const bool first = y < n0, second = !first && y - n0 < n1;
              const int slot = first ? y : y - n0;
              const float sv = first ? s0[slot * kRows] : (second ? s1[slot * kRows] : 0.0f);
              const uint32_t jv = first ? j0[slot * kRows] : (second ? j1[slot * kRows] : 0u);
              key[y] = (first || second) ? (((uint64_t)order_key(sv) << 16) | (uint64_t)(0xFFFFu - jv)) : 0ull;
            }
            uint64_t mine[16];  // (selects keep every register index constant)
            int rank[16];       // independent counts (no chain through one sum)
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              mine[x] = wg == 0 ? key[x] : key[16 + x];
              rank[x] = 0;
            }
#pragma unroll
            for (int y = 0; y < 32; ++y)
#pragma unroll
              for (int x = 0; x < 16; ++x) rank[x] += key[y] > mine[x] ? 1 : 0;
#pragma unroll
            for (int x = 0; x < 16; ++x)
              if (wg * 16 + x < n0 + n1 && rank[x] == target) {
                ms->cut_s[r] = key_value((uint32_t)(mine[x] >> 16));
                ms->cut_j[r] = (int)(0xFFFFu - (uint32_t)(mine[x] & 0xFFFFu));
              }
          } else if (R.row) {
            // more: each warpgroup ranks its own candidates against all of them
            const int target = ms->need[r] - 1;
            const int mine = wg == 0 ? n0 : n1;
            for (int x = 0; x < mine; ++x) {
              const float sx = cand_s[x * kRows];
              const int jx = cand_j[x * kRows];
              int rank = 0;
#pragma unroll 4
              for (int y = 0; y < n0; ++y) {
                const float sy = s0[y * kRows];
                rank += (int)((uint32_t)(sy > sx) | ((uint32_t)(sy == sx) & (uint32_t)((int)j0[y * kRows] < jx)));
              }
#pragma unroll 4
              for (int y = 0; y < n1; ++y) {
                const float sy = s1[y * kRows];
                rank += (int)((uint32_t)(sy > sx) | ((uint32_t)(sy == sx) & (uint32_t)((int)j1[y * kRows] < jx)));
              }
              if (rank == target) {
                ms->cut_s[r] = sx;
                ms->cut_j[r] = jx;
              }
            }
          }
          sel_sync();
          R.cs = ms->cut_s[r];
          R.cj = ms->cut_j[r];
          if (kind == kMerged && R.row) {
            // the candidates at or above the cut join the bitmask
            uint32_t* bm = reinterpret_cast<uint32_t*>(smem + kOffHist);
            for (int x = 0; x < min(R.n, cap); ++x) {
              const float sx = cand_s[x * kRows];
              const uint32_t jx = cand_j[x * kRows];
              if (sx > R.cs || (sx == R.cs && (int)jx <= R.cj)) {
                const uint32_t w = jx >> 5;
                atomicOr(bm + w * kRows + ((uint32_t)r ^ (w & 31u)), 1u << (jx & 31u));
              }
            }
          }
          for (int x = 0; x < min(R.n, cap); ++x) {  // my slots back to zero
            cand_s[x * kRows] = 0.0f;
            cand_j[x * kRows] = 0;
          }
          sel_sync();  // cleared before the output pass writes the bitmask
          if (kind == kMerged) {  // the rows are written from the bitmask at the next item's start
            pend_bh = bh;
            pend_rb = rb;
          }
        } else if (kind == kLevel) {
          if (wg == 0 && R.row) {
            int above, cnt;
            int b = find_bin(hist_row, need, above, cnt);
            if (b < 0) b = 0;
            need -= above;
            if (R.vlevel) {
              R.vpre |= (uint32_t)b << R.sh;
              R.vmask |= 0xFFu << R.sh;
            } else {
              R.kpre |= (uint32_t)b << R.sh;
              R.kmask |= 0xFFu << R.sh;
            }
            ms->kpre[r] = R.kpre;
            ms->kmask[r] = R.kmask;
            ms->vpre[r] = R.vpre;
            ms->vmask[r] = R.vmask;
            if (p == 1 + kLevels) {  // the last level: key and index of the cut are fixed
              ms->cut_s[r] = key_value(R.kpre);
              ms->cut_j[r] = (int)(0xFFFFu - R.vpre);
            }
          }
          sel_sync();
          R.kpre = ms->kpre[r];
          R.kmask = ms->kmask[r];
          R.vpre = ms->vpre[r];
          R.vmask = ms->vmask[r];
          if (p == 1 + kLevels) {
            R.cs = ms->cut_s[r];
            R.cj = ms->cut_j[r];
          }
        } else if (pl.bitmask) {  // kOutput: the rows are written from the bitmask at the next item's start
          pend_bh = bh;
          pend_rb = rb;
        } else {  // kOutput written directly
          (wg == 0 ? ms->w0 : ms->w1)[r] = R.w;
          sel_sync();
          if (R.row) {
            const int w0 = ms->w0[r], w1 = ms->w1[r];
            const int written = min(w0 + w1, a.K_capacity);
            if (wg == 0) {
              a.kept_cnt[(size_t)bh * a.nblk + R.i] = written;
            } else {
              if (a.threshold_mode && w1 > 0 && w0 + w1 <= a.K_capacity) {
                // my blocks sit at the end of the row: move them behind the first warpgroup's
                const int src = a.K_capacity - w1;
                for (int e = 0; e < w1 && src != w0; ++e) R.out[w0 + e] = R.out[src + e];
              }
              for (int e = a.threshold_mode ? written : a.keep; e < a.K_capacity; ++e) R.out[e] = -1;
            }
          }
        }
      }
      if (!ok) break;
    }
    if (ok && pend_bh >= 0) write_rows(smem, a, pend_bh, pend_rb, warp - 8, lane);
    if (!ok) {
      tmem_wait_ld();
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [B*H, nblk, 128] fp32 seen as 3-D (d, key block, batch-head), every
// `stride`-th key block from block 0 (rows = ceil(nblk / stride)); a box is
// 32 channels x 128 rows, 128-byte swizzle; rows past the end read 0.
int make_pooled_map(CUtensorMap* map, const float* base, int nblk, int BH, int stride) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess || p == nullptr)
    return SBATTN_ERR_CUDA;
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(p);
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)((nblk + stride - 1) / stride), (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)stride * kHeadDim * 4, (cuuint64_t)nblk * kHeadDim * 4};
  const cuuint32_t box[3] = {(cuuint32_t)kChunkD, (cuuint32_t)kTileN, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace

int select_max_nblk() { return 65535; }  // u16 histogram counts

int launch_select(const SelectArgs& a, cudaStream_t stream) {
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  if (a.nblk > select_max_nblk()) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap map, sample_map;
  int rc = make_pooled_map(&map, a.k_bar, a.nblk, a.B * a.H, 1);
  if (rc != SBATTN_OK) return rc;
  // the sample pass: every ceil(nblk/128)-th key block, at most 128 of them
  if ((rc = make_pooled_map(&sample_map, a.k_bar, a.nblk, a.B * a.H, (a.nblk + kTileN - 1) / kTileN)) != SBATTN_OK)
    return rc;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return SBATTN_ERR_CUDA;
  // the register split (kRegsProducers / kRegsSelectors) adds up to exactly
  // the launch allocation of 128 per thread; anything else would wait forever
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, select_kernel) != cudaSuccess || fa.numRegs != 128) return SBATTN_ERR_CUDA;
  const long items = (long)a.B * a.H * ((a.nblk + kRows - 1) / kRows);
  const int grid = (int)(items < sms ? items : sms);
  select_kernel<<<grid, kThreads, kSmemBytes, stream>>>(map, sample_map, a, kWaitLimitNs);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace sbattn
