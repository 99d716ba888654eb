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
// layout.  TMEM holds two S^T buffers (64 columns each) and the O^T
// accumulator (64 columns); TMEM lane = key row for S, = channel for O.
//
// Tensor-core issue, measured on B200: a tcgen05.mma costs the issuing
// thread about 146 cycles when it accumulates into the same TMEM tile as the
// MMA before it, whatever its N, and about 73 cycles when the issue stream
// rotates over eight accumulators.  An M=128, N=64, K=16 MMA has 32 cycles of
// math; PV of a tile is therefore spread over four partial O^T accumulators
// (K-step kk into partial kk mod 4; the epilogue sums them), and QK^T runs
// into a ring of four S^T tiles.
//
// Two softmax work-groups of 128 threads split the 64 query columns of every
// tile (32 each); a thread owns one TMEM lane, i.e. one KEY row across its 32
// queries, and handles two tiles per step.  The per-query running maximum m
// is seeded from the first step of the item (one cross-lane reduction per
// item).  Later steps need no barrier: a thread that meets a logit more than
// 2^8 above m raises a flag and records the excess per query (atomicMax); the
// work-group reads the flag at the start of the next step, once every thread
// has finished the previous one, and only then -- rarely -- raises m and
// rescales O and the partial row sums.  The flagged step's p values stay
// exact meanwhile: exp2 is only clamped beyond 2^100, which is reported as a
// device error.  Each thread keeps 32 partial row sums, reduced once per item.
//
// Roles (384 threads, one CTA per SM, persistent over items):
//   warp 0: TMA producer for Q and K tiles; also writes each tile's count of
//           valid key rows into a small shared ring, so that the softmax
//           warps never read the kept lists
//   warp 1: TMA producer for V tiles           warp 2: TMEM allocator + MMA issuer
//   warp 3: idle
//   warps 4-7 and 8-11: softmax + epilogue work-groups for query columns
//   0-31 and 32-63 (TMEM lane quarter = warp % 4)
// Every mbarrier wait is bounded (2 s); on expiry the kernel records
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

constexpr int kQBytes = 64 * 128 * 2;    // [2 channel halves][64 rows][128 B]
constexpr int kKVBytes = 128 * 128 * 2;  // [2 channel halves][128 rows][128 B]
constexpr int kPBytes = 128 * 64 * 2;    // [128 keys][64 queries] bf16
// Shared-memory rings.  A V stage waits for the softmax's P before PV frees
// it, so V gets the third stage; Q is reloaded once per item, covered by the
// QK^T front running ahead.
constexpr int kQStages = 1, kKStages = 2, kVStages = 3, kPStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQStages * kQBytes;
constexpr int kOffV = kOffK + kKStages * kKVBytes;
constexpr int kOffP = kOffV + kVStages * kKVBytes;
constexpr int kOffMisc = kOffP + kPStages * kPBytes;

constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kExpClamp = 100.0f;         // p <= 2^100: sums stay finite
constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kSBufs], s_empty[kSBufs];
  uint64_t p_full[kPStages], p_empty[kPStages];
  uint64_t o_full, o_empty;
  uint64_t info_full[kInfoSlots];
  uint64_t wg_bar[2];  // barrier of each softmax work-group (bounded wait)
  uint64_t drain;
  uint32_t info[kInfoSlots];  // valid key rows of a tile: low half | high half << 8
  uint32_t tmem_base;
  int abort;
  int flag[2][2];                 // per work-group, per step parity: a logit exceeded m by 2^8
  uint32_t raise_req[2][2][32];   // per work-group, per step parity: max excess per query (float bits)
  float m2[64];         // running max per query, scaled to log2 units
  float alpha[64];      // rescale factors / final 1/l
  float raise[64];      // increase of m in the current rescale
  float red[2][4][32];  // cross-warp reduction scratch per work-group
};

constexpr int kSmemBytes = kOffMisc + (int)sizeof(Misc) + 1024;  // + alignment slack

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
  volatile int* abort;
  uint32_t phase;
  SB_DEV bool operator()() {
    mbar_arrive(bar);
    const bool r = mbar_wait(bar, phase & 1, abort);
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

SB_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

SB_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
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
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc* ms = reinterpret_cast<Misc*>(smem + kOffMisc);
  const uint32_t sbase = smem_addr(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = a.B * a.H * a.nblk;

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
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&ms->p_full[s], kSoftmaxThreads);
      mbar_init(&ms->p_empty[s], 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&ms->s_full[s], 1);
      mbar_init(&ms->s_empty[s], kSoftmaxThreads);
    }
    for (int s = 0; s < kInfoSlots; ++s) mbar_init(&ms->info_full[s], 1);
    mbar_init(&ms->wg_bar[0], 128);
    mbar_init(&ms->wg_bar[1], 128);
    mbar_init(&ms->drain, 1);
    mbar_init(&ms->o_full, 1);
    mbar_init(&ms->o_empty, kSoftmaxThreads);
    ms->abort = 0;
    ms->flag[0][0] = ms->flag[0][1] = ms->flag[1][0] = ms->flag[1][1] = 0;
    for (int e = 0; e < 2 * 2 * 32; ++e) (&ms->raise_req[0][0][0])[e] = 0u;
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
        ok = mbar_wait(&ms->q_empty[qs], ((qcount / kQStages) & 1) ^ 1, abort_flag);
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
          ok = mbar_wait(&empty[st], ((tcount / nstages) & 1) ^ 1, abort_flag);
          if (ok) {
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
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    // One thread walks the tile stream twice: the QK^T front (bounded by the
    // S ring and the K ring) and the PV front (bounded by P and V); it issues
    // a whole tile of whichever front is ready, polling both.
    bool ok = true;
    if (lane == 0) {
      TileStream qk, pv;
      qk.init(a, total);
      pv.init(a, total);
      uint32_t gq = 0, gp = 0;  // global tile counts of the two fronts
      uint32_t inited = 0u;     // partial O accumulators started in the current item
      int qsb[2], qks[2], qqb[2];
      bool qlast[2];
      // Wait for the inputs of the next QK^T tile and take it from the front.
      auto qk_take = [&](int j) -> bool {
        qsb[j] = gq % kSBufs;
        qks[j] = gq % kKStages;
        qqb[j] = qk.n % kQStages;
        qlast[j] = qk.t == qk.it.ntiles - 1;
        if (!mbar_wait(&ms->s_empty[qsb[j]], ((gq / kSBufs) & 1) ^ 1, abort_flag)) return false;
        if (!mbar_wait(&ms->k_full[qks[j]], (gq / kKStages) & 1, abort_flag)) return false;
        if (qk.t == 0 && !mbar_wait(&ms->q_full[qqb[j]], (qk.n / kQStages) & 1, abort_flag)) return false;
        ++gq;
        qk.advance(a, total);
        return true;
      };
      auto qk_step = [&](int j, int kk) {
        const uint32_t k_addr = sbase + kOffK + qks[j] * kKVBytes + (kk >> 2) * 16384 + (kk & 3) * 32;
        const uint32_t q_addr = sbase + kOffQ + qqb[j] * kQBytes + (kk >> 2) * 8192 + (kk & 3) * 32;
        umma_bf16(tmem + qsb[j] * 64, smem_desc(k_addr, 16, 1024, kSwizzle128B),
                  smem_desc(q_addr, 16, 1024, kSwizzle128B), kIdescQK, kk > 0);
      };
      auto qk_commit = [&](int j) {
        umma_commit(&ms->s_full[qsb[j]]);
        umma_commit(&ms->k_empty[qks[j]]);
        if (qlast[j]) umma_commit(&ms->q_empty[qqb[j]]);
      };
      uint64_t last = global_timer_ns();
      while (pv.item < total) {
        bool progressed = false;
        // ---- QK^T front: a whole tile whenever its S slot and K are ready
        // (the S ring bounds it to four tiles ahead of the softmax)
        if (qk.item < total && mbar_test_wait(&ms->s_empty[gq % kSBufs], ((gq / kSBufs) & 1) ^ 1) &&
            mbar_test_wait(&ms->k_full[gq % kKStages], (gq / kKStages) & 1) &&
            (qk.t > 0 || mbar_test_wait(&ms->q_full[qk.n % kQStages], (qk.n / kQStages) & 1))) {
          ok = qk_take(0);  // (its waits are already satisfied)
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < 8; ++kk) qk_step(0, kk);
          qk_commit(0);
          progressed = true;
        }
        // ---- PV front: a whole tile once its P and V are ready, its K-steps
        // spread over the four partial O accumulators
        const int ps = gp % kPStages, vs = gp % kVStages;
        if (mbar_test_wait(&ms->p_full[ps], (gp / kPStages) & 1) &&
            mbar_test_wait(&ms->v_full[vs], (gp / kVStages) & 1) &&
            (pv.t > 0 || mbar_test_wait(&ms->o_empty, (pv.n & 1) ^ 1))) {
          const bool pfirst = pv.t == 0, plast = pv.t == pv.it.ntiles - 1;
          tc_fence_after();
          if (pfirst) inited = 0u;  // the first MMA of an item into each partial starts it
          const uint32_t v_addr = sbase + kOffV + vs * kKVBytes;
          const uint32_t p_addr = sbase + kOffP + ps * kPBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int part = kk & (kOParts - 1);
            umma_bf16(tmem + kColO + part * 64, smem_desc(v_addr + kk * 2048, 16384, 1024, kSwizzle128B),
                      smem_desc(p_addr + kk * 2048, 8192, 1024, kSwizzle128B), kIdescPV, (inited >> part) & 1u);
            inited |= 1u << part;
          }
          umma_commit(&ms->p_empty[ps]);
          umma_commit(&ms->v_empty[vs]);
          if (plast) umma_commit(&ms->o_full);
          ++gp;
          pv.advance(a, total);
          progressed = true;
        }
        if (progressed) {
          last = global_timer_ns();
        } else {
          if (*abort_flag || global_timer_ns() - last > kWaitLimitNs) {
            ok = false;
            break;
          }
          __nanosleep(20);
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        record_error(a.status, SBATTN_ERR_TIMEOUT);
        umma_commit(&ms->drain);  // completes once every issued MMA is done
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&ms->drain, 0) && global_timer_ns() - t0 < 100000000ull) {
        }
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------ softmax + epilogue
    const int g = (warp - 4) >> 2;  // work-group: query columns [32g, 32g + 32)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: key row of S, channel of O
    const int half = r >> 6;            // which kept block of a tile this key row belongs to
    const int col0 = kQCols * g;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c = a.scale * kLog2e;
    float* m2 = ms->m2 + col0;
    float* alpha = ms->alpha + col0;
    float(*red)[32] = ms->red[g];
    int* flag = ms->flag[g];
    uint32_t(*raise_req)[32] = ms->raise_req[g];
    uint32_t gt = 0, on = 0;  // global tile index, item ordinal
    WgSync wg{&ms->wg_bar[g], abort_flag, 0};
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
      float l[kQCols];
#pragma unroll
      for (int q = 0; q < kQCols; ++q) l[q] = 0.f;

      for (int tA = 0; tA < it.ntiles; tA += 2) {
        const bool hasB = tA + 1 < it.ntiles;
        const uint32_t gA = gt + tA, gB = gA + 1;
        const int par = (tA >> 1) & 1;  // step parity within the item
        if (tA > 0) {
          // ---- the previous step's flag: read once every thread of the
          // work-group has arrived on the P_full of that step's last tile
          const uint32_t gp_prev = gA - 1;
          ok = warp_wait(&ms->p_full[gp_prev % kPStages], (gp_prev / kPStages) & 1, abort_flag);
          if (!ok) break;
          if (flag[par ^ 1]) {
            // ---- rare path: raise m, rescale O and the partial sums ----
            if (r < kQCols) {
              const float up = __uint_as_float(raise_req[par ^ 1][r]);
              alpha[r] = fast_exp2(-up);
              m2[r] += up;
            }
            if (!(ok = wg())) break;
            // every PV issued so far must be complete before O is touched
            ok = warp_wait(&ms->p_empty[gp_prev % kPStages], (gp_prev / kPStages) & 1, abort_flag);
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
            for (int q = 0; q < kQCols; ++q) l[q] *= alpha[q];
            if (!(ok = wg())) break;  // everyone has read the request before it is cleared
            if (r < kQCols) raise_req[par ^ 1][r] = 0u;
            if (r == 0) flag[par ^ 1] = 0;
          }
        }
        // ---- S^T of the step's tiles: this work-group's 32 query columns
        ok = warp_wait(&ms->s_full[gA % kSBufs], (gA / kSBufs) & 1, abort_flag);
        if (ok && hasB) ok = warp_wait(&ms->s_full[gB % kSBufs], (gB / kSBufs) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        float x[2 * kQCols];  // [0, 32): tile A, [32, 64): tile B
        tmem_ld_32cols(lane_addr + (gA % kSBufs) * 64 + col0, *reinterpret_cast<uint32_t(*)[32]>(x));
        if (hasB) tmem_ld_32cols(lane_addr + (gB % kSBufs) * 64 + col0, *reinterpret_cast<uint32_t(*)[32]>(x + kQCols));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&ms->s_empty[gA % kSBufs]);
        if (hasB) mbar_arrive(&ms->s_empty[gB % kSBufs]);
        // ---- which of my key rows are real keys (written by the K producer)
        ok = warp_wait(&ms->info_full[gA % kInfoSlots], (gA / kInfoSlots) & 1, abort_flag);
        if (ok && hasB) ok = warp_wait(&ms->info_full[gB % kInfoSlots], (gB / kInfoSlots) & 1, abort_flag);
        if (!ok) break;
        const uint32_t infoA = ms->info[gA % kInfoSlots];
        const uint32_t infoB = hasB ? ms->info[gB % kInfoSlots] : 0u;
        const bool validA = (uint32_t)(r & 63) < ((infoA >> (8 * half)) & 0xFFu);
        const bool validB = hasB && (uint32_t)(r & 63) < ((infoB >> (8 * half)) & 0xFFu);

        if (tA == 0) {
          // seed the running max from the first step
          float v[kQCols];
#pragma unroll
          for (int q = 0; q < kQCols; ++q)
            v[q] = fmaxf(validA ? x[q] * c : -INFINITY, validB ? x[q + kQCols] * c : -INFINITY);
          const float mx = wg_reduce_cols<true>(v, red, quarter, lane, r, wg, ok);
          if (!ok) break;
          if (r < kQCols) m2[r] = (mx == -INFINITY) ? 0.f : mx;
          if (!(ok = wg())) break;
        }
        // ---- x <- s * c - m2 (log2 domain); rows outside the kept set -> -inf
        float lmax = -INFINITY;
#pragma unroll
        for (int q4 = 0; q4 < kQCols / 4; ++q4) {
          const float4 m4 = reinterpret_cast<const float4*>(m2)[q4];
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = 4 * q4 + e;
            x[q] = validA ? fmaf(x[q], c, -mm[e]) : -INFINITY;
            x[q + kQCols] = validB ? fmaf(x[q + kQCols], c, -mm[e]) : -INFINITY;
            lmax = fmaxf(lmax, fmaxf(x[q], x[q + kQCols]));
          }
        }
        if (lmax > kRescaleThreshold) {
          // rare: ask the next step to raise m for these queries (logits are
          // exact meanwhile up to 2^100 above m; beyond that they are clamped
          // and the call reports a device error)
#pragma unroll
          for (int q = 0; q < kQCols; ++q) {
            const float ex = fmaxf(x[q], x[q + kQCols]);
            if (ex > kRescaleThreshold) atomicMax(&raise_req[par][q], __float_as_uint(ex));
          }
          flag[par] = 1;
          if (lmax > kExpClamp) record_error(a.status, SBATTN_ERR_DEVICE);
        }
        // ---- p = 2^x, partial row sums, bf16 P^T rows into shared memory:
        // row r of P^T holds 64 queries (128 B, 128-byte swizzle); this
        // work-group owns its 16-byte chunks 4g .. 4g + 3
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
          if (tile == 1 && !hasB) break;
          const uint32_t gx = gA + tile;
          uint32_t pk[kQCols / 2];
#pragma unroll
          for (int q = 0; q < kQCols; q += 2) {
            const float p0 = fast_exp2(fminf(x[tile * kQCols + q], kExpClamp));
            const float p1 = fast_exp2(fminf(x[tile * kQCols + q + 1], kExpClamp));
            l[q] += p0;
            l[q + 1] += p1;
            pk[q >> 1] = pack_bf16x2(p0, p1);
          }
          ok = warp_wait(&ms->p_empty[gx % kPStages], ((gx / kPStages) & 1) ^ 1, abort_flag);
          if (!ok) break;
          uint8_t* prow = smem + kOffP + (gx % kPStages) * kPBytes + r * 128;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(prow + (((4 * g + c4) ^ (r & 7)) * 16)) =
                make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
        }
        if (!ok) break;
        fence_proxy_async_smem();
        mbar_arrive(&ms->p_full[gA % kPStages]);
        if (hasB) mbar_arrive(&ms->p_full[gB % kPStages]);
      }
      if (!ok) break;
      gt += it.ntiles;

      // ---- epilogue: (sum of the partial O^T) / l -> out ----
      ok = warp_wait(&ms->o_full, on & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      {
        // a flag raised by the item's last step is moot: O is complete; clear it
        // once every thread has finished that step (the o_full wait above)
        float v[kQCols];
#pragma unroll
        for (int q = 0; q < kQCols; ++q) v[q] = l[q];
        const float lsum = wg_reduce_cols<false>(v, red, quarter, lane, r, wg, ok);
        if (!ok) break;
        if (r < kQCols) {
          alpha[r] = lsum > 0.f ? 1.0f / lsum : 0.f;
          raise_req[0][r] = 0u;
          raise_req[1][r] = 0u;
        }
        if (r == 0) flag[0] = flag[1] = 0;
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
  const long total = (long)a.B * a.H * a.nblk;
  const int grid = (int)(total < sms ? total : sms);
  attention_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], a);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace sbattn
