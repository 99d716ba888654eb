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
// Softmax warps own one TMEM lane each, i.e. one KEY row across the 64
// queries.  The per-query running maximum m is therefore shared: it is seeded
// from the first tile of the item (one cross-lane reduction per item) and
// only raised when a tile holds a logit more than 2^8 above it (a rare,
// work-group-uniform rescale of O in TMEM and of the partial row sums).  Each
// thread keeps 64 partial row sums; they are reduced once per item.
//
// Roles (256 threads, one CTA per SM, persistent over items):
//   warp 0: TMA producer for Q and K tiles     warp 1: TMA producer for V tiles
//   warp 2: TMEM allocator + MMA issuer        warp 3: idle
//   warps 4-7: softmax + epilogue (TMEM lane quarter = warp % 4)
// Every mbarrier wait is bounded (2 s); on expiry the kernel records
// SBATTN_ERR_TIMEOUT, waits for its own copies and MMAs, frees TMEM and exits.
#include "internal.h"

namespace sbattn {

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS0 = 0, kColS1 = 64, kColO = 128;

constexpr int kQBytes = 64 * 128 * 2;    // [2 channel halves][64 rows][128 B]
constexpr int kKVBytes = 128 * 128 * 2;  // [2 channel halves][128 rows][128 B]
constexpr int kPBytes = 128 * 64 * 2;    // [128 keys][64 queries] bf16
constexpr int kStages = 2;               // Q, K, V and P are each double-buffered
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kStages * kQBytes;
constexpr int kOffV = kOffK + kStages * kKVBytes;
constexpr int kOffP = kOffV + kStages * kKVBytes;
constexpr int kOffMisc = kOffP + kStages * kPBytes;

constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
  uint64_t q_full[kStages], q_empty[kStages];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[kStages], p_empty[kStages];
  uint64_t o_full, o_empty, drain;
  uint64_t wg_bar;   // barrier of the 128 softmax threads (bounded wait)
  uint32_t tmem_base;
  int abort;
  int flag[2];
  float m2[64];      // running max per query, scaled to log2 units
  float alpha[64];   // rescale factors / final 1/l
  float raise[64];   // increase of m in the current rescale
  float red[4][64];  // cross-warp reduction scratch
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

// Transpose-reduce 64 per-lane values across the warp: afterwards v[0], v[1]
// hold the reduction over all 32 lanes of columns 2*lane and 2*lane + 1.
template <bool kMax>
SB_DEV void warp_reduce_cols(float (&v)[64], int lane) {
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
  SB_RED_ROUND(16, 32)
  SB_RED_ROUND(8, 16)
  SB_RED_ROUND(4, 8)
  SB_RED_ROUND(2, 4)
  SB_RED_ROUND(1, 2)
#undef SB_RED_ROUND
}

// Barrier of the 128 softmax threads on an mbarrier, so that it is bounded
// like every other wait: a thread that gave up elsewhere cannot leave the
// others stuck.  Returns false on timeout / abort.
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

// Work-group (128 softmax threads) reduction of v over all key lanes, per
// query column; result for column r (< 64) is returned to thread r.
template <bool kMax>
SB_DEV float wg_reduce_cols(float (&v)[64], Misc* ms, int quarter, int lane, int r, WgSync& wg, bool& ok) {
  warp_reduce_cols<kMax>(v, lane);
  ms->red[quarter][2 * lane] = v[0];
  ms->red[quarter][2 * lane + 1] = v[1];
  ok = wg();
  float res = 0.f;
  if (r < 64) {
    const float a = ms->red[0][r], b = ms->red[1][r], c = ms->red[2][r], d = ms->red[3][r];
    res = kMax ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
  }
  return res;
}

SB_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

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
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ms->q_full[s], 1);
      mbar_init(&ms->q_empty[s], 1);
      mbar_init(&ms->k_full[s], 1);
      mbar_init(&ms->k_empty[s], 1);
      mbar_init(&ms->v_full[s], 1);
      mbar_init(&ms->v_empty[s], 1);
      mbar_init(&ms->p_full[s], 128);
      mbar_init(&ms->p_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ms->s_full[s], 1);
      mbar_init(&ms->s_empty[s], 128);
    }
    mbar_init(&ms->o_full, 1);
    mbar_init(&ms->o_empty, 128);
    mbar_init(&ms->drain, 1);
    mbar_init(&ms->wg_bar, 128);
    ms->abort = 0;
    ms->flag[0] = ms->flag[1] = -1;
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
    uint32_t tcount = 0, qcount = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const Item it = decode_item(a, item);
      if (it.ntiles == 0) continue;
      if (is_k && lane == 0) {
        const int qs = qcount % kStages;
        ok = mbar_wait(&ms->q_empty[qs], ((qcount / kStages) & 1) ^ 1, abort_flag);
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
        int j1 = cur.get(2 * t);
        int j2 = (2 * t + 1 < it.cnt) ? cur.get(2 * t + 1) : j1;
        if (j1 < 0 || j1 >= a.nblk) j1 = it.i;  // masked by the softmax warps
        if (j2 < 0 || j2 >= a.nblk) j2 = it.i;
        if (lane == 0) {
          const int st = tcount % kStages;
          ok = mbar_wait(&empty[st], ((tcount / kStages) & 1) ^ 1, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(&full[st], kKVBytes);
            uint8_t* dst = smem + (is_k ? kOffK : kOffV) + st * kKVBytes;
            tma_load_4d(dst, tm, &full[st], 0, it.h, j1 * kBlock, it.b);
            tma_load_4d(dst + 8192, tm, &full[st], 0, it.h, j2 * kBlock, it.b);
            tma_load_4d(dst + 16384, tm, &full[st], 64, it.h, j1 * kBlock, it.b);
            tma_load_4d(dst + 24576, tm, &full[st], 64, it.h, j2 * kBlock, it.b);
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
        for (int s = 0; s < kStages; ++s) {
          // the most recent phase armed on slot s has parity ((n_s - 1) & 1)
          const uint32_t n_s = (tcount + kStages - 1 - s) / kStages;
          if (n_s > 0)
            while (!mbar_try_wait(&full[s], (n_s - 1) & 1) && global_timer_ns() - t0 < 100000000ull) {
            }
          const uint32_t nq = (qcount + kStages - 1 - s) / kStages;
          if (is_k && nq > 0)
            while (!mbar_try_wait(&ms->q_full[s], (nq - 1) & 1) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
      }
      __syncwarp();
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t kcount = 0, vcount = 0, scount = 0, pcount = 0, qcount = 0, ocount = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const Item it = decode_item(a, item);
      if (it.ntiles == 0) continue;
      if (lane == 0) {
        const int qs = qcount % kStages;
        ok = mbar_wait(&ms->q_full[qs], (qcount / kStages) & 1, abort_flag);
        const uint32_t q_addr = sbase + kOffQ + qs * kQBytes;
        auto issue_qk = [&](int t) -> bool {
          const int ks = kcount % kStages;
          if (!mbar_wait(&ms->k_full[ks], (kcount / kStages) & 1, abort_flag)) return false;
          const int sb = scount & 1;
          if (!mbar_wait(&ms->s_empty[sb], ((scount >> 1) & 1) ^ 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t k_addr = sbase + kOffK + ks * kKVBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tmem + (sb ? kColS1 : kColS0), smem_desc(k_addr + off, 16, 1024, kSwizzle128B),
                      smem_desc(q_addr + qoff, 16, 1024, kSwizzle128B), kIdescQK, kk > 0);
          }
          umma_commit(&ms->s_full[sb]);
          umma_commit(&ms->k_empty[ks]);
          if (t == it.ntiles - 1) umma_commit(&ms->q_empty[qs]);
          ++kcount;
          ++scount;
          return true;
        };
        if (ok) ok = issue_qk(0);
        for (int t = 0; t < it.ntiles && ok; ++t) {
          if (t + 1 < it.ntiles) ok = issue_qk(t + 1);
          if (!ok) break;
          if (t == 0) ok = mbar_wait(&ms->o_empty, (ocount & 1) ^ 1, abort_flag);
          const int ps = pcount % kStages, vs = vcount % kStages;
          if (ok) ok = mbar_wait(&ms->p_full[ps], (pcount / kStages) & 1, abort_flag);
          if (ok) ok = mbar_wait(&ms->v_full[vs], (vcount / kStages) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v_addr = sbase + kOffV + vs * kKVBytes;
          const uint32_t p_addr = sbase + kOffP + ps * kPBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            umma_bf16(tmem + kColO, smem_desc(v_addr + kk * 2048, 16384, 1024, kSwizzle128B),
                      smem_desc(p_addr + kk * 2048, 8192, 1024, kSwizzle128B), kIdescPV, (t > 0 || kk > 0));
          }
          umma_commit(&ms->p_empty[ps]);
          umma_commit(&ms->v_empty[vs]);
          ++pcount;
          ++vcount;
        }
        if (ok) umma_commit(&ms->o_full);
      }
      ++qcount;
      ++ocount;
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
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
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: key row of S, channel of O
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c = a.scale * kLog2e;
    uint32_t scount = 0, pcount = 0, ocount = 0;
    WgSync wg{&ms->wg_bar, abort_flag, 0};
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const Item it = decode_item(a, item);
      if (it.bad_cnt && r == 0) record_error(a.status, SBATTN_ERR_DEVICE);
      uint16_t* obase = a.out + (((size_t)it.b * a.N + (size_t)it.i * kBlock) * a.H + it.h) * kHeadDim + r;
      const int qrows = min(kBlock, a.N - it.i * kBlock);
      if (it.ntiles == 0) {
        for (int q = 0; q < qrows; ++q) obase[(size_t)q * a.H * kHeadDim] = 0;
        continue;
      }
      KeptCursor cur;
      cur.init(a.kept_idx + (size_t)item * a.K_capacity, it.cnt, lane);
      float l[64];
#pragma unroll
      for (int q = 0; q < 64; ++q) l[q] = 0.f;

      for (int t = 0; t < it.ntiles; ++t) {
        // which key does my lane hold in this tile?
        const int j_lo = cur.get(2 * t);
        const int j_hi = (2 * t + 1 < it.cnt) ? cur.get(2 * t + 1) : -1;
        const int jb = r < 64 ? j_lo : j_hi;
        const bool real = r < 64 || 2 * t + 1 < it.cnt;
        const bool jb_ok = jb >= 0 && jb < a.nblk;
        if (real && !jb_ok) record_error(a.status, SBATTN_ERR_DEVICE);
        const bool valid = jb_ok && (jb * kBlock + (r & 63)) < a.N;

        const int sb = scount & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&ms->s_full[sb], (scount >> 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        float x[64];
        {
          uint32_t raw[32];
          tmem_ld_32cols(lane_addr + (sb ? kColS1 : kColS0), raw);
          uint32_t raw2[32];
          tmem_ld_32cols(lane_addr + (sb ? kColS1 : kColS0) + 32, raw2);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            x[q] = __uint_as_float(raw[q]);
            x[q + 32] = __uint_as_float(raw2[q]);
          }
        }
        tc_fence_before();
        mbar_arrive(&ms->s_empty[sb]);
        const uint32_t tile_id = scount;
        ++scount;

        if (t == 0) {
          // seed the running max from this tile
          float v[64];
#pragma unroll
          for (int q = 0; q < 64; ++q) v[q] = valid ? x[q] * c : -INFINITY;
          const float mx = wg_reduce_cols<true>(v, ms, quarter, lane, r, wg, ok);
          if (!ok) break;
          if (r < 64) ms->m2[r] = (mx == -INFINITY) ? 0.f : mx;
          if (!(ok = wg())) break;
        }
        // x <- s * c - m2 (log2 domain)
        float lmax = -INFINITY;
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 m4 = reinterpret_cast<const float4*>(ms->m2)[q4];
          x[4 * q4 + 0] = valid ? fmaf(x[4 * q4 + 0], c, -m4.x) : -INFINITY;
          x[4 * q4 + 1] = valid ? fmaf(x[4 * q4 + 1], c, -m4.y) : -INFINITY;
          x[4 * q4 + 2] = valid ? fmaf(x[4 * q4 + 2], c, -m4.z) : -INFINITY;
          x[4 * q4 + 3] = valid ? fmaf(x[4 * q4 + 3], c, -m4.w) : -INFINITY;
          lmax = fmaxf(lmax, fmaxf(fmaxf(x[4 * q4], x[4 * q4 + 1]), fmaxf(x[4 * q4 + 2], x[4 * q4 + 3])));
        }
        if (t > 0) {
          const bool need = __any_sync(0xffffffffu, lmax > kRescaleThreshold);
          if (need && lane == 0) ms->flag[tile_id & 1] = (int)tile_id;
          if (!(ok = wg())) break;
          if (ms->flag[tile_id & 1] == (int)tile_id) {
            // ---- rare path: raise m, rescale O and the partial sums ----
            float v[64];
#pragma unroll
            for (int q = 0; q < 64; ++q) v[q] = x[q];
            const float mt = wg_reduce_cols<true>(v, ms, quarter, lane, r, wg, ok);
            if (!ok) break;
            if (r < 64) {
              const float up = fmaxf(mt, 0.f);
              ms->raise[r] = up;
              ms->alpha[r] = fast_exp2(-up);
              ms->m2[r] += up;
            }
            if (!(ok = wg())) break;
            // every PV issued so far must be complete before O is touched
            const uint32_t prev = pcount - 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&ms->p_empty[prev % kStages], (prev / kStages) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t o[32];
              tmem_ld_32cols(lane_addr + kColO + half * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * ms->alpha[half * 32 + q]);
              tmem_st_32cols(lane_addr + kColO + half * 32, o);
            }
            tmem_wait_st();
            tc_fence_before();
            // partial sums follow O; x was relative to the old maximum
#pragma unroll
            for (int q = 0; q < 64; ++q) {
              l[q] *= ms->alpha[q];
              x[q] -= ms->raise[q];
            }
          }
        }
        // p = 2^x, partial row sums, pack to bf16
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 64; q += 2) {
          const float p0 = fast_exp2(x[q]), p1 = fast_exp2(x[q + 1]);
          l[q] += p0;
          l[q + 1] += p1;
          pk[q >> 1] = pack_bf16x2(p0, p1);
        }
        const int ps = pcount % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&ms->p_empty[ps], ((pcount / kStages) & 1) ^ 1, abort_flag));
        if (!ok) break;
        {
          uint8_t* prow = smem + kOffP + ps * kPBytes + r * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int phys = ch ^ (r & 7);
            *reinterpret_cast<uint4*>(prow + phys * 16) =
                make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&ms->p_full[ps]);
        ++pcount;
      }
      if (!ok) break;

      // ---- epilogue: O^T / l -> out ----
      ok = __all_sync(0xffffffffu, mbar_wait(&ms->o_full, ocount & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      {
        float v[64];
#pragma unroll
        for (int q = 0; q < 64; ++q) v[q] = l[q];
        const float lsum = wg_reduce_cols<false>(v, ms, quarter, lane, r, wg, ok);
        if (!ok) break;
        if (r < 64) ms->alpha[r] = lsum > 0.f ? 1.0f / lsum : 0.f;
        if (!(ok = wg())) break;
      }
      uint32_t o0[32], o1[32];
      tmem_ld_32cols(lane_addr + kColO, o0);
      tmem_ld_32cols(lane_addr + kColO + 32, o1);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ms->o_empty);
      ++ocount;
      const size_t row_stride = (size_t)a.H * kHeadDim;
#pragma unroll
      for (int q = 0; q < 64; ++q) {
        const float o = __uint_as_float(q < 32 ? o0[q] : o1[q - 32]) * ms->alpha[q];
        if (q < qrows) obase[(size_t)q * row_stride] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
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
