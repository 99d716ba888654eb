// Block-sparse attention over the kept key blocks (xiaodao.ai "MiniMax-H3 的
// 6.24 倍，不能直接算成六倍产能", section "6.24 倍里，真正有损的部分大约是三倍":
// only the high-scoring key blocks enter the block-sparse attention kernel).
//
// Work item = one 64-query block of one (batch, head) with its own kept list.
// Because every query block has its own keys, 128 query rows can never share
// a B operand; the kernel therefore works in the transposed orientation so
// that every tcgen05.mma has M = 128:
//
//   S^T[128 keys x 64 q]  = K_tile[128 keys x 128 d] . Q_i^T         (A = K, K-major; B = Q, K-major)
//   O^T[128 d    x 64 q] += V_tile^T[128 d x 128 keys] . P^T          (A = V, MN-major; B = P, MN-major)
//
// A key tile is two kept 64-token blocks, each fetched by TMA (two 64-channel
// boxes per block, 128-byte swizzle) straight into the canonical operand
// layout.  TMEM holds a ring of four S^T tiles (64 columns each) and four
// partial O^T accumulators; TMEM lane = key row for S, = channel for O.
//
// Tensor-core issue, measured on B200: with N = 64 an MMA has only 32 cycles
// of math, and the bound is how fast one thread can issue tcgen05.mma (about
// 54 cycles apart in a tight loop, 120 with address arithmetic in between)
// and the ~146-cycle latency of an MMA that accumulates into the tile the
// previous one wrote.  Two warps therefore issue MMAs, each from a tight,
// unrolled loop: one the QK^T chain of each tile into a ring of four S^T
// tiles in TMEM, the other PV, spread over four partial O^T accumulators
// (K-step kk into partial kk mod 4; the epilogue sums them), so that the two
// streams interleave in the tensor pipe.  TMA streaming and MMAs on the same
// SM do not slow each other down.
//
// Shared memory (208 KB): Q (one stage), K (three stages), V (two) and two
// P^T buffers, each released in two key halves: the softmax threads of key
// rows 0-63 may refill a buffer as soon as the first four PV K-steps that
// read it are done, and the PV issuer waits for the second half only before
// the last four.  The PV issuer, after acquiring a half through its
// mbarrier, executes the async-proxy fence that makes the softmax threads'
// generic stores visible to the tensor core (the fence may sit anywhere on
// the release/acquire path from the stores to the MMA that reads them).
//
// Two softmax work-groups of 128 threads split the 64 query columns of every
// tile (32 each); a thread owns one TMEM lane, i.e. one KEY row across its 32
// queries, and takes two tiles per step.  The per-query running maximum m is
// seeded from the first step of the item (one cross-lane reduction per item).
// Each later step's S^T is loaded, scaled (s * scale * log2 e - m) and checked
// one step ahead, while the previous step's P^T is stored: a thread publishes
// per query the largest excess of its logits over m, and a work-group barrier
// (bounded like every wait) orders all publications before the step starts.
// When some excess passes 2^8, the group raises m by exactly that excess and
// rescales O and the row sums before any p of the step is formed, so no p
// exceeds 2^8 whatever the logit range.  The raise is rare in practice.  Each
// thread keeps 32 partial row sums (packed in pairs), reduced once per item.
//
// Roles (384 threads, one CTA per SM, persistent over items; warps 0-3 run
// with 56 registers and the softmax warps with 224 after setmaxnreg):
//   warp 0: TMA producer for Q and K tiles; also writes each tile's count of
//           valid key rows into a small shared ring, so that the softmax
//           warps never read the kept lists
//   warp 1: TMA producer for V tiles
//   warp 2: TMEM allocator + QK^T issuer       warp 3: PV issuer
//   warps 4-7 and 8-11: softmax + epilogue work-groups for query columns
//   0-31 and 32-63 (TMEM lane quarter = warp % 4)
// Every mbarrier wait is bounded (2 s by default; the failure-detection entry
// point takes another limit and can withhold one V copy); on expiry the kernel records
// SBATTN_ERR_TIMEOUT, waits for its own copies and MMAs, frees TMEM and exits.
#include "internal.h"

namespace sbattn {

namespace {

constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;  // two work-groups of 128
constexpr int kQCols = 32;            // query columns per work-group
constexpr uint32_t kTmemCols = 512;
constexpr int kSBufs = 4;             // S^T ring in TMEM, 64 columns each
constexpr uint32_t kColO = 256;       // four partial O^T accumulators, 64 columns each
constexpr int kOParts = 4;
constexpr int kInfoSlots = 16;        // per-tile valid-row counts, ring
// registers per thread after setmaxnreg: warps 0-3 (copies, MMA issue) give
// theirs to the softmax warps; the split must equal the launch allocation
constexpr uint32_t kRegsIssue = 56, kRegsSoftmax = 224;
static_assert(128 * kRegsIssue + 256 * kRegsSoftmax == kThreads * 168, "register split = 384 x 168");

constexpr int kQBytes = 64 * 128 * 2;    // [2 channel halves][64 rows][128 B]
constexpr int kKVBytes = 128 * 128 * 2;  // [2 channel halves][128 rows][128 B]
constexpr int kPBytes = 128 * 64 * 2;    // [128 keys][64 queries] bf16
constexpr int kQStages = 1, kKStages = 3, kVStages = 2, kPStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQStages * kQBytes;
constexpr int kOffV = kOffK + kKStages * kKVBytes;
constexpr int kOffP = kOffV + kVStages * kKVBytes;
constexpr int kOffMisc = kOffP + kPStages * kPBytes;

constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Lookahead slots: the excesses of step s are published in slot s % 4 during
// step s - 1, read at the start of step s and cleared at the start of step
// s + 2 (when every thread of the group has passed step s + 1's barrier).
constexpr int kLookSlots = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kSBufs], s_empty[kSBufs];
  uint64_t p_full[kPStages][2], p_empty[kPStages][2];  // per P^T buffer and key half (rows 0-63, 64-127)
  uint64_t o_full, o_empty;
  uint64_t info_full[kInfoSlots];
  uint64_t wg_bar[2];  // barrier of each softmax work-group (bounded wait)
  uint64_t drain[2];  // per MMA issuer, for the error path
  uint32_t info[kInfoSlots];  // valid key rows of a tile: low half | high half << 8
  uint32_t tmem_base;
  int abort;
  uint64_t lk_bar[2];  // per work-group: the next step's excesses are published (lookahead)
  int look_flag[2][kLookSlots];        // per work-group and step slot: some logit exceeds m by 2^8
  uint32_t look_req[2][kLookSlots][32];  // per work-group, slot and query: largest excess (float bits)
  alignas(16) float negm2[64];  // minus the running max per query, in log2 units (read as float4)
  float alpha[64];      // rescale factors / final 1/l
  float red[2][4][32];  // cross-warp reduction scratch per work-group
};

static_assert(offsetof(Misc, negm2) % 16 == 0, "negm2 is read with 16-byte loads");
constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc);  // base is 1024-byte aligned (checked)

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 64, 1, 1);

SB_DEV void record_error(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Kept-list reader for one warp: lane l holds entries [base + l] of the
// current and the next 32-entry chunk; get(p) must be called with the same,
// non-decreasing p by all lanes.
struct KeptCursor {
  const int32_t* list;
  int cnt, base, cur, nxt, lane;
  SB_DEV void init(const int32_t* l, int c, int ln) {
    list = l; cnt = c; base = 0; lane = ln;
    cur = lane < cnt ? __ldg(list + lane) : -1;
    nxt = 32 + lane < cnt ? __ldg(list + 32 + lane) : -1;
  }
  SB_DEV int get(int p) {
    while (p >= base + 32) {
      base += 32;
      cur = nxt;
      const int q = base + 32 + lane;
      nxt = q < cnt ? __ldg(list + q) : -1;
    }
    return __shfl_sync(0xffffffffu, cur, p - base);
  }
};

struct Item {
  int b, h, i, cnt, ntiles;
  bool bad_cnt;
};

SB_DEV Item decode_item(const AttentionArgs& a, int item) {
  Item it;
  it.i = item % a.nblk;
  const int bh = item / a.nblk;
  it.h = bh % a.H;
  it.b = bh / a.H;
  int c = __ldg(a.kept_cnt + item);
  it.bad_cnt = c < 1 || c > a.K_capacity;
  if (c < 0 || c > a.K_capacity) c = 0;
  it.cnt = c;
  it.ntiles = (c + 1) / 2;
  return it;
}

// Transpose-reduce 32 per-lane values across the warp: afterwards v[0] holds
// the reduction over all 32 lanes of column `lane`.
template <bool kMax>
SB_DEV void warp_reduce_cols(float (&v)[32], int lane) {
#define SB_RED_ROUND(OFF, HALF)                                     \
  {                                                                 \
    const bool up = (lane & (OFF)) != 0;                            \
    _Pragma("unroll") for (int j = 0; j < (HALF); ++j) {            \
      const float send = up ? v[j] : v[j + (HALF)];                 \
      const float keep = up ? v[j + (HALF)] : v[j];                 \
      const float recv = __shfl_xor_sync(0xffffffffu, send, (OFF)); \
      v[j] = kMax ? fmaxf(keep, recv) : keep + recv;                \
    }                                                               \
  }
  SB_RED_ROUND(16, 16)
  SB_RED_ROUND(8, 8)
  SB_RED_ROUND(4, 4)
  SB_RED_ROUND(2, 2)
  SB_RED_ROUND(1, 1)
#undef SB_RED_ROUND
}

// Barrier of the 128 threads of a softmax work-group on an mbarrier, so that
// it is bounded like every other wait: a thread that gave up elsewhere cannot
// leave the others stuck.  Returns false on timeout / abort.
struct WgSync {
  uint64_t* bar;
  WaitCtl wc;
  uint32_t phase;
  SB_DEV bool operator()() {
    mbar_arrive(bar);
    const bool r = mbar_wait(bar, phase & 1, wc);
    ++phase;
    return __all_sync(0xffffffffu, r);
  }
};

// Work-group reduction of v over all 128 key lanes, per query column of the
// work-group; the result for column r (< 32) is returned to thread r.
template <bool kMax>
SB_DEV float wg_reduce_cols(float (&v)[32], float (*red)[32], int quarter, int lane, int r, WgSync& wg, bool& ok) {
  warp_reduce_cols<kMax>(v, lane);
  red[quarter][lane] = v[0];
  ok = wg();
  float res = 0.f;
  if (r < 32) {
    const float a = red[0][r], b = red[1][r], c = red[2][r], d = red[3][r];
    res = kMax ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
  }
  return res;
}

// A barrier of a work-group whose arrival and wait are separate points of
// the program (bounded like every wait).
struct SplitSync {
  uint64_t* bar;
  WaitCtl wc;
  uint32_t phase;
  SB_DEV void arrive() { mbar_arrive(bar); }
  SB_DEV bool wait() {
    const bool r = mbar_wait(bar, phase & 1, wc);
    ++phase;
    return __all_sync(0xffffffffu, r);
  }
};

// Is key row r of a tile a real key: the tile's info word holds the valid
// rows of its two kept blocks (low byte: rows 0-63, next byte: rows 64-127).
SB_DEV bool key_row_valid(uint32_t info, int r, int half) {
  return (uint32_t)(r & 63) < ((info >> (8 * half)) & 0xFFu);
}

// x <- s * c - m in the log2 domain (two lanes per instruction) for the two
// tiles of a step; rows outside the kept set -> -inf
SB_DEV void scale_logits(float (&x)[64], const float* negm2, float c, bool validA, bool validB) {
  const uint64_t c2 = f2_pack(c, c);
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
    const float4 m4 = reinterpret_cast<const float4*>(negm2)[q4];
    const uint64_t mlo = f2_pack(m4.x, m4.y), mhi = f2_pack(m4.z, m4.w);
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
      const int q = tile * 32 + 4 * q4;
      const uint64_t a0 = f2_fma(f2_pack(x[q], x[q + 1]), c2, mlo);
      const uint64_t a1 = f2_fma(f2_pack(x[q + 2], x[q + 3]), c2, mhi);
      f2_unpack(a0, x[q], x[q + 1]);
      f2_unpack(a1, x[q + 2], x[q + 3]);
    }
  }
  if (!validA) {
#pragma unroll
    for (int q = 0; q < 32; ++q) x[q] = -INFINITY;
  }
  if (!validB) {
#pragma unroll
    for (int q = 0; q < 32; ++q) x[32 + q] = -INFINITY;
  }
}

SB_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

SB_DEV bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& wc) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
}

// Walks the CTA's non-empty items and their tiles in order.
struct TileStream {
  int item, t, n;  // item index, tile within the item, ordinal among non-empty items
  Item it;
  SB_DEV void skip_empty(const AttentionArgs& a, int total) {
    while (item < total) {
      it = decode_item(a, item);
      if (it.ntiles > 0) return;
      item += gridDim.x;
    }
  }
  SB_DEV void init(const AttentionArgs& a, int total) {
    item = blockIdx.x;
    t = 0;
    n = 0;
    skip_empty(a, total);
  }
  SB_DEV void advance(const AttentionArgs& a, int total) {
    if (++t == it.ntiles) {
      t = 0;
      ++n;
      item += gridDim.x;
      skip_empty(a, total);
    }
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, AttentionArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc* ms = reinterpret_cast<Misc*>(smem + kOffMisc);
  const uint32_t sbase = smem_addr(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.B * a.H * a.nblk;
  if ((sbase & 1023u) != 0u) {  // the 128-byte swizzle atoms need 1024-byte alignment
    if (threadIdx.x == 0) record_error(a.status, SBATTN_ERR_DEVICE);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&ms->q_full[s], 1);
      mbar_init(&ms->q_empty[s], 1);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&ms->k_full[s], 1);
      mbar_init(&ms->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&ms->v_full[s], 1);
      mbar_init(&ms->v_empty[s], 1);
    }
    for (int s = 0; s < kPStages; ++s)
      for (int h = 0; h < 2; ++h) {
        mbar_init(&ms->p_full[s][h], kSoftmaxThreads / 2);
        mbar_init(&ms->p_empty[s][h], 1);
      }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&ms->s_full[s], 1);
      mbar_init(&ms->s_empty[s], kSoftmaxThreads);
    }
    for (int s = 0; s < kInfoSlots; ++s) mbar_init(&ms->info_full[s], 1);
    mbar_init(&ms->wg_bar[0], 128);
    mbar_init(&ms->wg_bar[1], 128);
    mbar_init(&ms->drain[0], 1);
    mbar_init(&ms->drain[1], 1);
    mbar_init(&ms->o_full, 1);
    mbar_init(&ms->o_empty, kSoftmaxThreads);
    ms->abort = 0;
    mbar_init(&ms->lk_bar[0], 128);
    mbar_init(&ms->lk_bar[1], 128);
    for (int e = 0; e < 2 * kLookSlots; ++e) (&ms->look_flag[0][0])[e] = 0;
    for (int e = 0; e < 2 * kLookSlots * 32; ++e) (&ms->look_req[0][0][0])[e] = 0u;
    fence_barrier_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 2) {
    tmem_alloc(&ms->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  volatile int* abort_flag = &ms->abort;
  const WaitCtl wc{abort_flag, a.wait_limit_ns};

  if (warp < 4) {
  warpgroup_regs_dec<kRegsIssue>();
  if (warp == 0 || warp == 1) {
    // ------------------------------------------------------------ producers
    const bool is_k = warp == 0;
    const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
    uint64_t* full = is_k ? ms->k_full : ms->v_full;
    uint64_t* empty = is_k ? ms->k_empty : ms->v_empty;
    const int nstages = is_k ? kKStages : kVStages;
    uint32_t tcount = 0, qcount = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const Item it = decode_item(a, item);
      if (it.ntiles == 0) continue;
      if (is_k && lane == 0) {
        const int qs = qcount % kQStages;
        ok = mbar_wait(&ms->q_empty[qs], ((qcount / kQStages) & 1) ^ 1, wc);
        if (ok) {
          mbar_arrive_expect_tx(&ms->q_full[qs], kQBytes);
          uint8_t* dst = smem + kOffQ + qs * kQBytes;
          tma_load_4d(dst, &tm_q, &ms->q_full[qs], 0, it.h, it.i * kBlock, it.b);
          tma_load_4d(dst + kQBytes / 2, &tm_q, &ms->q_full[qs], 64, it.h, it.i * kBlock, it.b);
          ++qcount;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      KeptCursor cur;
      cur.init(a.kept_idx + (size_t)item * a.K_capacity, it.cnt, lane);
      for (int t = 0; t < it.ntiles && ok; ++t) {
        const int j1 = cur.get(2 * t);
        const bool has2 = 2 * t + 1 < it.cnt;
        const int j2 = has2 ? cur.get(2 * t + 1) : j1;
        const bool ok1 = j1 >= 0 && j1 < a.nblk;
        const bool ok2 = has2 && j2 >= 0 && j2 < a.nblk;
        // invalid blocks are replaced by a valid one and masked via the row counts
        const int l1 = ok1 ? j1 : it.i;
        const int l2 = ok2 ? j2 : l1;
        if (lane == 0) {
          if (is_k) {
            if (!ok1 || (has2 && !ok2)) record_error(a.status, SBATTN_ERR_DEVICE);
            const uint32_t lo = ok1 ? (uint32_t)min(kBlock, a.N - j1 * kBlock) : 0u;
            const uint32_t hi = ok2 ? (uint32_t)min(kBlock, a.N - j2 * kBlock) : 0u;
            const int slot = tcount % kInfoSlots;
            ms->info[slot] = lo | (hi << 8);
            mbar_arrive(&ms->info_full[slot]);
          }
          const int st = tcount % nstages;
          if (!is_k && (int)tcount == a.withhold_v_tile) {
            // diagnostic: this V copy is never issued (the stage is skipped),
            // so the PV issuer's bounded wait for it must run out
            ++tcount;
          } else if ((ok = mbar_wait(&empty[st], ((tcount / nstages) & 1) ^ 1, wc))) {
            mbar_arrive_expect_tx(&full[st], kKVBytes);
            uint8_t* dst = smem + (is_k ? kOffK : kOffV) + st * kKVBytes;
            tma_load_4d(dst, tm, &full[st], 0, it.h, l1 * kBlock, it.b);
            tma_load_4d(dst + 8192, tm, &full[st], 0, it.h, l2 * kBlock, it.b);
            tma_load_4d(dst + 16384, tm, &full[st], 64, it.h, l1 * kBlock, it.b);
            tma_load_4d(dst + 24576, tm, &full[st], 64, it.h, l2 * kBlock, it.b);
            ++tcount;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        record_error(a.status, SBATTN_ERR_TIMEOUT);
        // let copies already issued land before the CTA exits
        const uint64_t t0 = global_timer_ns();
        for (int s = 0; s < nstages; ++s) {
          // the most recent phase armed on slot s has parity ((n_s - 1) & 1)
          const uint32_t n_s = (tcount + nstages - 1 - s) / nstages;
          if (n_s > 0)
            while (!mbar_try_wait(&full[s], (n_s - 1) & 1) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        for (int s = 0; is_k && s < kQStages; ++s) {
          const uint32_t nq = (qcount + kQStages - 1 - s) / kQStages;
          if (nq > 0)
            while (!mbar_try_wait(&ms->q_full[s], (nq - 1) & 1) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
      }
      __syncwarp();
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 2 issues QK^T (bounded by the S ring and the K ring), warp 3 PV
    // (bounded by P, V and the O accumulators).  With N = 64 every MMA has
    // only 32 cycles of math, so the issuing thread's own instruction latency
    // matters: the loops are unrolled over the K-steps and step precomputed
    // descriptors by constants (+32 B inside the 128-byte atom = +2 in the
    // descriptor's address field, which cannot carry for shared addresses).
    const bool is_qk = warp == 2;
    bool ok = true;
    if (lane == 0) {
      TileStream ts;
      ts.init(a, total);
      uint32_t gt = 0;  // global tile count of this front
      while (ts.item < total) {
        if (is_qk) {
          const int sb = gt % kSBufs, ks = gt % kKStages, qb = ts.n % kQStages;
          const bool last = ts.t == ts.it.ntiles - 1;
          ok = mbar_wait(&ms->s_empty[sb], ((gt / kSBufs) & 1) ^ 1, wc) &&
               mbar_wait(&ms->k_full[ks], (gt / kKStages) & 1, wc) &&
               (ts.t > 0 || mbar_wait(&ms->q_full[qb], (ts.n / kQStages) & 1, wc));
          if (!ok) break;
          tc_fence_after();
          const uint64_t kd = smem_desc(sbase + kOffK + ks * kKVBytes, 16, 1024, kSwizzle128B);
          const uint64_t qd = smem_desc(sbase + kOffQ + qb * kQBytes, 16, 1024, kSwizzle128B);
          const uint32_t d = tmem + sb * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(d, kd + (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2), qd + (uint64_t)((kk >> 2) * 512 + (kk & 3) * 2),
                      kIdescQK, kk > 0);
          umma_commit(&ms->s_full[sb]);
          umma_commit(&ms->k_empty[ks]);
          if (last) umma_commit(&ms->q_empty[qb]);
        } else {
          const int vs = gt % kVStages, pb = gt % kPStages;
          const uint32_t pph = (gt / kPStages) & 1;
          const bool first = ts.t == 0, last = ts.t == ts.it.ntiles - 1;
          ok = mbar_wait(&ms->v_full[vs], (gt / kVStages) & 1, wc) &&
               mbar_wait(&ms->p_full[pb][0], pph, wc) &&
               (!first || mbar_wait(&ms->o_empty, (ts.n & 1) ^ 1, wc));
          if (!ok) break;
          tc_fence_after();
          // the softmax threads' P^T stores (generic proxy), acquired through
          // p_full, become visible to the tensor core (async proxy)
          fence_proxy_async_smem();
          const uint64_t vd = smem_desc(sbase + kOffV + vs * kKVBytes, 16384, 1024, kSwizzle128B);
          const uint64_t pd = smem_desc(sbase + kOffP + pb * kPBytes, 8192, 1024, kSwizzle128B);
          // K-step kk accumulates into partial kk mod 4; the first tile of an
          // item starts each partial
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + kColO + kk * 64, vd + (uint64_t)(kk * 128), pd + (uint64_t)(kk * 128), kIdescPV, !first);
          umma_commit(&ms->p_empty[pb][0]);  // key rows 0-63 of this P^T buffer are free again
          if (!(ok = mbar_wait(&ms->p_full[pb][1], pph, wc))) break;
          tc_fence_after();
          fence_proxy_async_smem();
#pragma unroll
          for (int kk = 4; kk < 8; ++kk)
            umma_bf16(tmem + kColO + (kk & 3) * 64, vd + (uint64_t)(kk * 128), pd + (uint64_t)(kk * 128), kIdescPV, 1u);
          umma_commit(&ms->p_empty[pb][1]);
          umma_commit(&ms->v_empty[vs]);
          if (last) umma_commit(&ms->o_full);
        }
        ++gt;
        ts.advance(a, total);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (lane == 0) {
      if (!ok) {
        *abort_flag = 1;
        record_error(a.status, SBATTN_ERR_TIMEOUT);
      }
      // every MMA this thread issued is done before the CTA frees TMEM, also
      // when another role gave up first (in a normal run this wait is over at
      // once: the softmax consumed every result)
      uint64_t* drain = &ms->drain[is_qk ? 0 : 1];
      umma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  }
  } else {
    warpgroup_regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------ softmax + epilogue
    const int g = (warp - 4) >> 2;  // work-group: query columns [32g, 32g + 32)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: key row of S, channel of O
    const int half = r >> 6;            // which kept block of a tile this key row belongs to
    const int col0 = kQCols * g;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c = a.scale * kLog2e;
    float* negm2 = ms->negm2 + col0;
    float* alpha = ms->alpha + col0;
    float(*red)[32] = ms->red[g];
    int* look_flag = ms->look_flag[g];
    uint32_t(*look_req)[32] = ms->look_req[g];
    uint32_t gt = 0, on = 0;  // global tile index, item ordinal
    WgSync wg{&ms->wg_bar[g], wc, 0};
    SplitSync lk{&ms->lk_bar[g], wc, 0};
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const Item it = decode_item(a, item);
      if (it.bad_cnt && g == 0 && r == 0) record_error(a.status, SBATTN_ERR_DEVICE);
      uint16_t* obase = a.out + (((size_t)it.b * a.N + (size_t)it.i * kBlock) * a.H + it.h) * kHeadDim + r;
      const size_t row_stride = (size_t)a.H * kHeadDim;
      const int qrows = min(kBlock, a.N - it.i * kBlock);
      if (it.ntiles == 0) {
        for (int q = col0; q < col0 + kQCols; ++q)
          if (q < qrows) obase[(size_t)q * row_stride] = 0;
        continue;
      }
      uint64_t l2[kQCols / 2];  // partial row sums, packed pairs of queries
#pragma unroll
      for (int q = 0; q < kQCols / 2; ++q) l2[q] = 0ull;

      // The softmax takes the item's tiles two at a time (a step), so that its
      // fixed costs per wait are shared by 64 logits per thread.  S^T of a
      // step's tiles is loaded into x during the previous step (the item's
      // first step here), hiding the TMEM load latency behind the P^T stores,
      // and is scaled and checked there too (lookahead): every thread
      // publishes per query how far its logits of the next step exceed the
      // running maximum, and the work-group barrier `lk` orders those
      // publications before the next step starts.  A step whose logits run
      // more than 2^8 above m therefore raises m first, by exactly the largest
      // excess, before any of its p is computed: no p exceeds 2^8, whatever the
      // scale.  Barriers signalled in tile order by one thread (S^T full, info,
      // P^T empty) are waited on for the later tile of a step only.
      const int nsteps = (it.ntiles + 1) >> 1;
      float x[2 * kQCols];  // [0, 32): tile A, [32, 64): tile B
      bool validA = false, validB = false;
      {
        const bool hasB = it.ntiles > 1;
        const uint32_t gl = hasB ? gt + 1 : gt;
        ok = warp_wait(&ms->s_full[gl % kSBufs], (gl / kSBufs) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        tmem_ld_32cols(lane_addr + (gt % kSBufs) * 64 + col0, *reinterpret_cast<uint32_t(*)[32]>(x));
        if (hasB)
          tmem_ld_32cols(lane_addr + ((gt + 1) % kSBufs) * 64 + col0, *reinterpret_cast<uint32_t(*)[32]>(x + kQCols));
      }

      for (int step = 0; step < nsteps; ++step) {
        const int tA = 2 * step;
        const bool hasB = tA + 1 < it.ntiles;
        const uint32_t gA = gt + tA, gB = gA + 1;
        if (step == 0) {
          // ---- S^T of the first step is in x: release it, seed m from it
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&ms->s_empty[gA % kSBufs]);
          if (hasB) mbar_arrive(&ms->s_empty[gB % kSBufs]);
          const uint32_t gl = hasB ? gB : gA;
          ok = warp_wait(&ms->info_full[gl % kInfoSlots], (gl / kInfoSlots) & 1, wc);
          if (!ok) break;
          validA = key_row_valid(ms->info[gA % kInfoSlots], r, half);
          validB = hasB && key_row_valid(ms->info[gB % kInfoSlots], r, half);
          float v[kQCols];
#pragma unroll
          for (int q = 0; q < kQCols; ++q)
            v[q] = fmaxf(validA ? x[q] * c : -INFINITY, validB ? x[q + kQCols] * c : -INFINITY);
          const float mx = wg_reduce_cols<true>(v, red, quarter, lane, r, wg, ok);
          if (!ok) break;
          if (r < kQCols) negm2[r] = (mx == -INFINITY) ? 0.f : -mx;
          if (!(ok = wg())) break;
          scale_logits(x, negm2, c, validA, validB);
        } else {
          // ---- every thread of the group has published this step's excess
          if (!(ok = lk.wait())) break;
          const int sl = step & (kLookSlots - 1);
          if (look_flag[sl]) {
            // ---- rare path: some logit of this step exceeds m by more than
            // 2^8: raise m by the largest excess of each query, now
            if (r < kQCols) {
              const float up = __uint_as_float(look_req[sl][r]);
              alpha[r] = fast_exp2(-up);
              negm2[r] -= up;
            }
            if (!(ok = wg())) break;  // the new m is visible to the group
#pragma unroll
            for (int q = 0; q < kQCols; ++q) {
              const float up = __uint_as_float(look_req[sl][q]);
              x[q] -= up;
              x[kQCols + q] -= up;
            }
            // every PV issued so far must be complete before O is touched
            const uint32_t gp = gA - 1;
            ok = warp_wait(&ms->p_empty[gp % 2][0], (gp / 2) & 1, wc) &&
                 warp_wait(&ms->p_empty[gp % 2][1], (gp / 2) & 1, wc);
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int part = 0; part < kOParts; ++part) {
              uint32_t o[32];
              const uint32_t oaddr = lane_addr + kColO + part * 64 + col0;
              tmem_ld_32cols(oaddr, o);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < kQCols; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
              tmem_st_32cols(oaddr, o);
            }
            tmem_wait_st();
            tc_fence_before();
#pragma unroll
            for (int q = 0; q < kQCols; q += 2) l2[q >> 1] = f2_mul(l2[q >> 1], f2_pack(alpha[q], alpha[q + 1]));
          }
          // the slot of two steps ago is read by every thread of the group
          // (they all passed this step's lk) and is next written two steps on
          if (step >= 2) {
            const int old = (step - 2) & (kLookSlots - 1);
            if (r < kQCols) look_req[old][r] = 0u;
            if (r == 0) look_flag[old] = 0;
          }
        }
        // ---- p = 2^x and partial row sums (a row outside the kept set has
        // x = -inf and p = 0); the row sums take the bf16 weights PV actually
        // uses, so that O / l stays a convex combination of V rows even where
        // no p is 1
        uint32_t pk[2][kQCols / 2];
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
#pragma unroll
          for (int q = 0; q < kQCols; q += 2) {
            const int i = tile * kQCols + q;
            pk[tile][q >> 1] = pack_bf16x2(fast_exp2(x[i]), fast_exp2(x[i + 1]));
            l2[q >> 1] = f2_add(l2[q >> 1], f2_pack(__uint_as_float(pk[tile][q >> 1] << 16),
                                                    __uint_as_float(pk[tile][q >> 1] & 0xFFFF0000u)));
          }
        }
        // ---- start loading the next step's S^T
        const bool more = step + 1 < nsteps;
        const bool nB = tA + 3 < it.ntiles;
        const uint32_t gn = gA + 2;
        if (more) {
          const uint32_t gnl = nB ? gn + 1 : gn;
          ok = warp_wait(&ms->s_full[gnl % kSBufs], (gnl / kSBufs) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          tmem_ld_32cols(lane_addr + (gn % kSBufs) * 64 + col0, *reinterpret_cast<uint32_t(*)[32]>(x));
          if (nB)
            tmem_ld_32cols(lane_addr + ((gn + 1) % kSBufs) * 64 + col0, *reinterpret_cast<uint32_t(*)[32]>(x + kQCols));
        }
        // ---- bf16 P^T rows into shared memory once PV has released my half
        // of each buffer: row r holds 64 queries (128 B, 128-byte swizzle);
        // this work-group owns its 16-byte chunks 4g .. 4g + 3
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
          if (tile == 1 && !hasB) break;
          const uint32_t gx = gA + tile;
          const int pb = gx % 2;
          ok = warp_wait(&ms->p_empty[pb][half], ((gx / 2) & 1) ^ 1, wc);
          if (!ok) break;
          uint8_t* prow = smem + kOffP + pb * kPBytes + r * 128;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(prow + (((4 * g + c4) ^ (r & 7)) * 16)) =
                make_uint4(pk[tile][4 * c4], pk[tile][4 * c4 + 1], pk[tile][4 * c4 + 2], pk[tile][4 * c4 + 3]);
        }
        if (!ok) break;
        // the PV issuer makes these stores visible to the tensor core after
        // acquiring them through p_full (one proxy fence per half tile there
        // instead of one per softmax thread and step here)
        mbar_arrive(&ms->p_full[gA % 2][half]);
        if (hasB) mbar_arrive(&ms->p_full[gB % 2][half]);
        // ---- lookahead: scale the next step's logits and publish how far
        // they exceed the running maximum
        if (more) {
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&ms->s_empty[gn % kSBufs]);
          if (nB) mbar_arrive(&ms->s_empty[(gn + 1) % kSBufs]);
          const uint32_t gnl = nB ? gn + 1 : gn;
          ok = warp_wait(&ms->info_full[gnl % kInfoSlots], (gnl / kInfoSlots) & 1, wc);
          if (!ok) break;
          validA = key_row_valid(ms->info[gn % kInfoSlots], r, half);
          validB = nB && key_row_valid(ms->info[(gn + 1) % kInfoSlots], r, half);
          scale_logits(x, negm2, c, validA, validB);
          float lmax = -INFINITY;
#pragma unroll
          for (int q = 0; q < 2 * kQCols; q += 2) lmax = fmax3(lmax, x[q], x[q + 1]);
          if (lmax > kRescaleThreshold) {
            const int sl = (step + 1) & (kLookSlots - 1);
#pragma unroll
            for (int q = 0; q < kQCols; ++q) {
              const float ex = fmaxf(x[q], x[kQCols + q]);
              if (ex > kRescaleThreshold) atomicMax(&look_req[sl][q], __float_as_uint(ex));
            }
            look_flag[sl] = 1;
          }
          lk.arrive();
        }
      }
      if (!ok) break;
      gt += it.ntiles;

      // ---- epilogue: (sum of the partial O^T) / l -> out ----
      ok = warp_wait(&ms->o_full, on & 1, wc);
      if (!ok) break;
      tc_fence_after();
      {
        // flags raised by the item's last tiles are moot: O is complete; clear
        // them once every thread has finished the item (the o_full wait above)
        float v[kQCols];
#pragma unroll
        for (int q = 0; q < kQCols; q += 2) f2_unpack(l2[q >> 1], v[q], v[q + 1]);
        const float lsum = wg_reduce_cols<false>(v, red, quarter, lane, r, wg, ok);
        if (!ok) break;
        if (r < kQCols) {
          alpha[r] = lsum > 0.f ? 1.0f / lsum : 0.f;
#pragma unroll
          for (int sl = 0; sl < kLookSlots; ++sl) look_req[sl][r] = 0u;
        }
        if (r < kLookSlots) look_flag[r] = 0;
        if (!(ok = wg())) break;
      }
      float acc[kQCols];
      {
        uint32_t o0[32], o1[32];
        tmem_ld_32cols(lane_addr + kColO + 0 * 64 + col0, o0);
        tmem_ld_32cols(lane_addr + kColO + 1 * 64 + col0, o1);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < kQCols; ++q) acc[q] = __uint_as_float(o0[q]) + __uint_as_float(o1[q]);
        tmem_ld_32cols(lane_addr + kColO + 2 * 64 + col0, o0);
        tmem_ld_32cols(lane_addr + kColO + 3 * 64 + col0, o1);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < kQCols; ++q) acc[q] += __uint_as_float(o0[q]) + __uint_as_float(o1[q]);
      }
      tc_fence_before();
      mbar_arrive(&ms->o_empty);
      ++on;
#pragma unroll
      for (int q = 0; q < kQCols; ++q) {
        const float ov = acc[q] * alpha[q];
        if (col0 + q < qrows) obase[(size_t)(col0 + q) * row_stride] = __bfloat16_as_ushort(__float2bfloat16_rn(ov));
      }
    }
    if (!ok) {
      tmem_wait_ld();  // no TMEM load may be outstanding when the CTA frees TMEM
      if (r == 0) {
        *abort_flag = 1;
        record_error(a.status, SBATTN_ERR_TIMEOUT);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int launch_attention(const AttentionArgs& a, cudaStream_t stream) {
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  CUtensorMap maps[3];
  const uint16_t* ptrs[3] = {a.q, a.k, a.v};
  for (int m = 0; m < 3; ++m) {
    const int rc = make_bf16_row_map(&maps[m], ptrs[m], a.B, a.N, a.H);
    if (rc != SBATTN_OK) return rc;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return SBATTN_ERR_CUDA;
  // setmaxnreg moves registers between warpgroups within the CTA's launch
  // allocation; the split (kRegsIssue / kRegsSoftmax) adds up to exactly
  // 384 x 168, so the kernel must be built with 168 registers per thread
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, attention_kernel) != cudaSuccess || fa.numRegs != 168) return SBATTN_ERR_CUDA;
  const long total = (long)a.B * a.H * a.nblk;
  const int grid = (int)(total < sms ? total : sms);
  attention_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], a);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace sbattn
