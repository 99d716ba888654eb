// SubBlock block selection (xiaodao.ai "MiniMax-H3 的 6.24 倍，不能直接算成六倍
// 产能", section "6.24 倍里，真正有损的部分大约是三倍": query and key are cut into
// 64-token blocks, the key blocks that contribute little are estimated and
// only the high-scoring ones are kept; chat-gpts.plus "MiniMax-H3 在 8×H200 上
// 基准测试…", section "事件核心：发生了什么": blocks below a threshold are
// skipped).
//
// Scores on tensor cores.  A work item is 128 query blocks of one (batch,
// head), one per TMEM lane, so that a thread owns a query block's whole score
// row and selects within it alone.  The block scores s_ij = q_bar_i . k_bar_j
// are fp32 dot products; the tensor core computes them from tf32 pieces:
// x = hi + lo with hi = x with its low 13 mantissa bits cleared (exactly a
// tf32 value) and lo = x - hi, and s = hi_q.hi_k + hi_q.lo_k + lo_q.hi_k
// (kind::tf32, fp32 accumulation; the dropped lo.lo term and the tf32
// reading of lo leave an error of a few 1e-6 of |q_bar_i| |k_bar_j|).
//   * Q pieces: each selector thread loads its query block's mean, splits it
//     and stores hi / lo into its own TMEM lane (the A operand, read from
//     tensor memory).
//   * K pieces: a TMA warp streams k_bar in stages of 128 key blocks x 32
//     channels (one 128-byte swizzle row of fp32 per key block), four stages
//     deep; four converter warps split each stage in place into hi (where TMA
//     wrote it) and lo (a second buffer with the same swizzled positions).
//   * One thread issues the MMAs: per channel chunk of a group of 256 key
//     blocks (two stages) 4 K-steps x 3 products x 2 tiles, M = 128 query
//     blocks, N = 128 keys, K = 8 channels, into two accumulators of 128 TMEM
//     columns (the two tiles' chains interleave).
// Exact top-K: an 8-bit radix select on order-preserving 32-bit keys of the
// fp32 scores, four passes (most significant digit first), each counting in a
// per-row histogram (u16, shared memory) the digits of the keys that match
// the digits found so far; then an output pass writes, in ascending key
// block order, the diagonal, every score above the selected value and the
// lowest-indexed ties.  The scores are recomputed by the tensor core in every
// pass: deterministic, so all passes see the same values.  Threshold mode
// (keep s >= tau) and the trivial budgets need the output pass only.
//
// Roles (384 threads, one CTA per SM, persistent over work items):
//   warp 0: TMA producer           warp 1: TMEM allocator + MMA issuer
//   warps 4-7: converters          warps 8-11: selectors (TMEM lane quarter = warp % 4)
// Every mbarrier wait is bounded; on expiry the kernel stores nothing more,
// lets its own copies and MMAs finish, frees TMEM and returns.
#include "internal.h"

namespace sbattn {

namespace {

constexpr int kThreads = 384;
constexpr int kRows = 128;                    // query blocks per work item (MMA M)
constexpr int kTileN = 128;                   // key blocks per MMA (N)
constexpr int kGroupTiles = 2;                // accumulators per group
constexpr int kGroupKeys = kTileN * kGroupTiles;      // 256
constexpr int kChunkD = 32;                   // channels per stage (128 bytes of fp32)
constexpr int kChunks = kHeadDim / kChunkD;   // 4
constexpr int kStages = 4;                    // a stage: one tile of 128 keys x one chunk of 32 channels
constexpr int kHalfBytes = kTileN * kChunkD * 4;      // 16 KB: hi (TMA target) or lo
constexpr int kStageBytes = 2 * kHalfBytes;
constexpr int kBins = 256;
constexpr int kHistBytes = kBins * kRows * 2;         // u16 counts, [bin][row]
constexpr int kOffHist = kStages * kStageBytes;       // 128 KB
constexpr int kOffMisc = kOffHist + kHistBytes;       // 192 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQhi = 0, kColQlo = 128, kColD = 256;
constexpr int kRadixPasses = 4;

struct Misc {
  uint64_t raw_full[kStages], conv_full[kStages], stage_empty[kStages];
  uint64_t d_full, d_empty;  // the group's accumulators
  uint64_t q_ready, q_empty;  // the item's Q pieces in TMEM
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
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

// Monotone map from float to uint32 (larger float -> larger key); adding
// +0 first turns -0 into +0, so that the two zeros are equal keys.
SB_DEV uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

SB_DEV uint32_t tf32_hi(uint32_t u) { return u & 0xFFFFE000u; }

// The schedule every role walks: work items (128 query blocks of one
// batch-head) strided over the grid, passes, groups of 256 key blocks and the
// four channel chunks of a group.
struct Plan {
  int items, row_blocks, groups, passes;
  SB_DEV void init(const SelectArgs& a) {
    row_blocks = (a.nblk + kRows - 1) / kRows;
    items = a.B * a.H * row_blocks;
    groups = (a.nblk + kGroupKeys - 1) / kGroupKeys;
    const bool radix = !a.threshold_mode && a.keep > 1 && a.keep < a.nblk;
    passes = radix ? kRadixPasses + 1 : 1;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    select_kernel(const __grid_constant__ CUtensorMap tm_k, SelectArgs a, uint64_t wait_limit_ns) {
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
    mbar_init(&ms->d_full, 1);
    mbar_init(&ms->d_empty, 128);
    mbar_init(&ms->q_ready, 128);
    mbar_init(&ms->q_empty, 1);
    mbar_init(&ms->drain, 1);
    ms->abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_k);
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // histograms start at zero; every radix pass clears the bins it read
  for (int e = threadIdx.x; e < kHistBytes / 16; e += kThreads)
    reinterpret_cast<uint4*>(smem + kOffHist)[e] = make_uint4(0u, 0u, 0u, 0u);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  volatile int* abort_flag = &ms->abort;
  const WaitCtl wc{abort_flag, wait_limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------- TMA
    bool ok = true;
    uint32_t sc = 0;
    if (lane == 0) {
      for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x) {
        const int bh = item / pl.row_blocks;
        for (int pass = 0; pass < pl.passes && ok; ++pass)
          for (int g = 0; g < pl.groups && ok; ++g)
            for (int c = 0; c < kChunks && ok; ++c)
              for (int t = 0; t < kGroupTiles && ok; ++t) {
                const int s = sc % kStages;
                if (!(ok = mbar_wait(&ms->stage_empty[s], ((sc / kStages) & 1) ^ 1, wc))) break;
                mbar_arrive_expect_tx(&ms->raw_full[s], kHalfBytes);
                tma_load_3d(smem + s * kStageBytes, &tm_k, &ms->raw_full[s], c * kChunkD, g * kGroupKeys + t * kTileN,
                            bh);
                ++sc;
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
      uint32_t sc = 0, gc = 0, ic = 0;
      for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x, ++ic) {
        if (!(ok = mbar_wait(&ms->q_ready, ic & 1, wc))) break;
        for (int pass = 0; pass < pl.passes && ok; ++pass)
          for (int g = 0; g < pl.groups && ok; ++g, ++gc) {
            if (!(ok = mbar_wait(&ms->d_empty, (gc & 1) ^ 1, wc))) break;
            tc_fence_after();
            for (int c = 0; c < kChunks && ok; ++c, sc += kGroupTiles) {
              // the chunk's two stages (tile 0, tile 1) are consecutive in the ring
              const int s0 = sc % kStages, s1 = (sc + 1) % kStages;
              if (!(ok = mbar_wait(&ms->conv_full[s0], (sc / kStages) & 1, wc) &&
                         mbar_wait(&ms->conv_full[s1], ((sc + 1) / kStages) & 1, wc)))
                break;
              tc_fence_after();
              const uint32_t st_addr[2] = {smem_addr(smem + s0 * kStageBytes), smem_addr(smem + s1 * kStageBytes)};
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t ks = (uint32_t)(c * 4 + kk);  // K-step of 8 channels
                const uint32_t ahi = tmem + kColQhi + ks * 8, alo = tmem + kColQlo + ks * 8;
                const uint32_t first = (c == 0 && kk == 0) ? 0u : 1u;
                // +32 bytes per K-step inside the 128-byte row = +2 in the address field
                uint64_t bhi[2], blo[2];
#pragma unroll
                for (int t = 0; t < kGroupTiles; ++t) {
                  bhi[t] = smem_desc(st_addr[t], 16, 1024, kSwizzle128B) + (uint64_t)(kk * 2);
                  blo[t] = smem_desc(st_addr[t] + kHalfBytes, 16, 1024, kSwizzle128B) + (uint64_t)(kk * 2);
                }
#pragma unroll
                for (int t = 0; t < kGroupTiles; ++t) umma_tf32_ts(tmem + kColD + t * kTileN, ahi, bhi[t], first);
#pragma unroll
                for (int t = 0; t < kGroupTiles; ++t) umma_tf32_ts(tmem + kColD + t * kTileN, ahi, blo[t], 1u);
#pragma unroll
                for (int t = 0; t < kGroupTiles; ++t) umma_tf32_ts(tmem + kColD + t * kTileN, alo, bhi[t], 1u);
              }
              umma_commit(&ms->stage_empty[s0]);
              umma_commit(&ms->stage_empty[s1]);
            }
            if (ok) umma_commit(&ms->d_full);
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
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------- converters
    const int tid = threadIdx.x - 128;
    uint32_t sc = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x)
      for (int pass = 0; pass < pl.passes && ok; ++pass)
        for (int g = 0; g < pl.groups && ok; ++g)
          for (int c = 0; c < kChunks * kGroupTiles && ok; ++c, ++sc) {
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
    if (!ok && threadIdx.x == 128) *abort_flag = 1;
  } else if (warp >= 8) {
    // ------------------------------------------------------------- selectors
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = query block of the item
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    uint16_t* hist = reinterpret_cast<uint16_t*>(smem + kOffHist);  // [bin][row]
    uint32_t gc = 0, ic = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < pl.items && ok; item += gridDim.x, ++ic) {
      const int bh = item / pl.row_blocks;
      const int i = (item - bh * pl.row_blocks) * kRows + r;  // my query block
      const bool row = i < a.nblk;
      // ---- my query block's mean, split into tf32 pieces, into my TMEM lane
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ms->q_empty, (ic & 1) ^ 1, wc)))) break;
      tc_fence_after();
      {
        const float4* qrow = reinterpret_cast<const float4*>(a.q_bar + ((size_t)bh * a.nblk + (row ? i : 0)) * kHeadDim);
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
          uint32_t hv[32], lv[32];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 v = row ? __ldg(qrow + part * 8 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t h = tf32_hi(__float_as_uint(f[k]));
              hv[4 * e + k] = h;
              lv[4 * e + k] = __float_as_uint(f[k] - __uint_as_float(h));
            }
          }
          tmem_st_32cols(lane_addr + kColQhi + part * 32, hv);
          tmem_st_32cols(lane_addr + kColQlo + part * 32, lv);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ms->q_ready);
      }
      // ---- selection state of my row
      uint32_t prefix = 0, mask = 0;
      int remaining = a.keep - 1;  // off-diagonal blocks to keep (budget mode)
      int shift = 24;
      int32_t* out = a.kept_idx + ((size_t)bh * a.nblk + (row ? i : 0)) * a.K_capacity;
      float* srow = a.scores != nullptr && row ? a.scores + ((size_t)bh * a.nblk + i) * a.nblk : nullptr;
      int written = 0, eq_taken = 0;
      bool output = false;
      // per element of a chunk of my score row: count its digit (radix pass,
      // fire-and-forget shared-memory atomic on my 16-bit half of a word; the
      // neighbouring row owns the other half) or decide and write it (output)
      const uint32_t inc = 1u << ((r & 1) * 16);
      uint32_t* hw = reinterpret_cast<uint32_t*>(smem + kOffHist) + (r >> 1);  // + bin * 64
      auto scan_chunk = [&](const uint32_t (&v)[32], int j0) {
        if (!output) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = j0 + e;
            const uint32_t key = order_key(__uint_as_float(v[e]));
            if (j < a.nblk && j != i && (key & mask) == prefix) atomicAdd(hw + ((key >> shift) & 0xFFu) * 64, inc);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = j0 + e;
            if (j >= a.nblk) continue;  // (fully unrolled: v stays in registers)
            const float sv = __uint_as_float(v[e]);
            const uint32_t key = order_key(sv);
            if (srow != nullptr) srow[j] = sv;
            bool take;
            if (j == i) {
              take = true;
            } else if (a.threshold_mode) {
              take = sv >= a.tau;
            } else if (a.keep <= 1) {
              take = false;
            } else if (a.keep >= a.nblk) {
              take = true;
            } else {
              take = key > prefix || (key == prefix && eq_taken < remaining);
              if (key == prefix && take) ++eq_taken;
            }
            if (take && written < a.K_capacity) out[written++] = j;  // bounded by the row's capacity
          }
        }
      };
      for (int pass = 0; pass < pl.passes && ok; ++pass) {
        output = pass == pl.passes - 1;
        for (int g = 0; g < pl.groups && ok; ++g, ++gc) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ms->d_full, gc & 1, wc)))) break;
          tc_fence_after();
          // the group's 256 scores in eight 32-column chunks; the load of the
          // next chunk is in flight while one is processed
          uint32_t va[32], vb[32];
          tmem_ld_32cols(lane_addr + kColD, va);
#pragma unroll 1
          for (int part = 0; part < kGroupKeys / 32; part += 2) {
            tmem_wait_ld_regs(va);
            tmem_ld_32cols(lane_addr + kColD + (part + 1) * 32, vb);
            if (row) scan_chunk(va, g * kGroupKeys + part * 32);
            tmem_wait_ld_regs(vb);
            if (part + 2 < kGroupKeys / 32) tmem_ld_32cols(lane_addr + kColD + (part + 2) * 32, va);
            if (row) scan_chunk(vb, g * kGroupKeys + (part + 1) * 32);
          }
          tc_fence_before();
          mbar_arrive(&ms->d_empty);
        }
        if (!ok) break;
        if (!output && row) {
          // ---- the digit of the remaining-th largest among the matching keys;
          // clear the bins for the next pass
          int cum = 0, digit = -1, above = 0;
#pragma unroll 4
          for (int b = kBins - 1; b >= 0; --b) {
            uint16_t* h = hist + b * kRows + r;
            const int cnt = *h;
            *h = 0;
            if (digit < 0) {
              if (cum + cnt >= remaining) {
                digit = b;
                above = cum;
              } else {
                cum += cnt;
              }
            }
          }
          prefix |= (uint32_t)digit << shift;
          mask |= 0xFFu << shift;
          remaining -= above;
          shift -= 8;
        }
      }
      if (!ok) break;
      if (row) {
        for (int e = written; e < a.K_capacity; ++e) out[e] = -1;
        a.kept_cnt[(size_t)bh * a.nblk + i] = written;
      }
    }
    if (!ok) {
      tmem_wait_ld();
      if (r == 0) *abort_flag = 1;
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

// [B*H, nblk, 128] fp32 seen as 3-D (d, key block, batch-head); a box is 32
// channels x 128 key blocks, 128-byte swizzle; key blocks past nblk read 0.
int make_pooled_map(CUtensorMap* map, const float* base, int nblk, int BH) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess || p == nullptr)
    return SBATTN_ERR_CUDA;
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(p);
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)nblk, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 4, (cuuint64_t)nblk * kHeadDim * 4};
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
  CUtensorMap map;
  int rc = make_pooled_map(&map, a.k_bar, a.nblk, a.B * a.H);
  if (rc != SBATTN_OK) return rc;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return SBATTN_ERR_CUDA;
  const long items = (long)a.B * a.H * ((a.nblk + kRows - 1) / kRows);
  const int grid = (int)(items < sms ? items : sms);
  select_kernel<<<grid, kThreads, kSmemBytes, stream>>>(map, a, kWaitLimitNs);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace sbattn
