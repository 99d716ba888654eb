// SubBlock block selection (xiaodao.ai "MiniMax-H3 的 6.24 倍，不能直接算成六倍
// 产能", section "6.24 倍里，真正有损的部分大约是三倍": query and key are cut into
// 64-token blocks, the key blocks that contribute little are estimated and
// only the high-scoring ones are kept; chat-gpts.plus "MiniMax-H3 在 8×H200 上
// 基准测试…", section "事件核心：发生了什么": blocks below a threshold are
// skipped).
//
// One CTA owns R query blocks of one (batch, head).  Phase 1 computes their
// full score rows s_ij = q_bar_i . k_bar_j into shared memory: each thread
// owns key blocks j = tid, tid + 256, ... and dots its pooled key row against
// the R pooled query rows (fp32, channel order 0..127, broadcast from shared
// memory).  Phase 2 gives each warp one row: a 4-pass, 8-bit radix select on
// order-preserving 32-bit keys finds the (K-1)-th largest off-diagonal score
// exactly, then one ascending ballot-compaction pass writes the diagonal, every
// score above that value and the lowest-indexed ties, already sorted.
#include "internal.h"

namespace sbattn {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Monotone map from float to uint32 (larger float -> larger key); -0 -> +0.
SB_DEV uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

SB_DEV uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exact key of the need-th largest element of row[0..n) excluding index
// `skip`, and how many elements equal to it must be taken (the others above
// it are all taken).  Warp-collective; hist: 256 words of this warp's smem.
SB_DEV void radix_select(const float* row, int n, int skip, int need, uint32_t* hist, uint32_t& tau,
                         int& need_eq) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  int remaining = need;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      uint32_t key = 0;
      bool ok = false;
      if (j < n && j != skip) {
        key = order_key(row[j]);
        ok = (key & pmask) == prefix;
      }
      const uint32_t act = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        const uint32_t digit = (key >> shift) & 0xFFu;
        const uint32_t peers = __match_any_sync(act, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
      }
    }
    __syncwarp();
    // lane l owns bins [8l, 8l+8); count elements in bins above each lane's range
    int local = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) local += (int)hist[8 * lane + e];
    int suf = local;  // inclusive suffix sum over lanes >= this lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += t;
    }
    const int above_lane = suf - local;
    const uint32_t hit = __ballot_sync(0xffffffffu, above_lane < remaining && remaining <= suf);
    const int src = __ffs(hit) - 1;
    int digit = 0, above = 0;
    if (lane == src) {
      int cum = above_lane;
      for (int b = 8 * lane + 7; b >= 8 * lane; --b) {
        const int cnt = (int)hist[b];
        if (cum + cnt >= remaining) {
          digit = b;
          above = cum;
          break;
        }
        cum += cnt;
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    prefix |= (uint32_t)digit << shift;
    pmask |= 0xFFu << shift;
    remaining -= above;
    __syncwarp();
  }
  tau = prefix;
  need_eq = remaining;
}

template <int R>
__global__ void __launch_bounds__(kThreads) select_kernel(SelectArgs a, int ld) {
  extern __shared__ float4 smem4[];
  float* qs = reinterpret_cast<float*>(smem4);  // [R][128]
  float* sc = qs + R * kHeadDim;                // [R][ld]
  uint32_t* hist = reinterpret_cast<uint32_t*>(sc + (size_t)R * ld);  // [warps][256]

  const int tid = threadIdx.x;
  const int groups = (a.nblk + R - 1) / R;
  const int bh = blockIdx.x / groups;
  const int r0 = (blockIdx.x - bh * groups) * R;
  const int rows = min(R, a.nblk - r0);

  const float* qb = a.q_bar + ((size_t)bh * a.nblk + r0) * kHeadDim;
  for (int e = tid; e < R * kHeadDim; e += kThreads) qs[e] = (e / kHeadDim) < rows ? qb[e] : 0.f;
  __syncthreads();

  // ---- phase 1: score rows ------------------------------------------------
  const float* kb = a.k_bar + (size_t)bh * a.nblk * kHeadDim;
  for (int j = tid; j < a.nblk; j += kThreads) {
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const float4* kr = reinterpret_cast<const float4*>(kb + (size_t)j * kHeadDim);
#pragma unroll 4
    for (int d4 = 0; d4 < kHeadDim / 4; ++d4) {
      const float4 kv = __ldg(kr + d4);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 qv = reinterpret_cast<const float4*>(qs + r * kHeadDim)[d4];
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) sc[r * ld + j] = acc[r];
  }
  __syncthreads();

  if (a.scores != nullptr) {
    for (int r = 0; r < rows; ++r) {
      float* dst = a.scores + ((size_t)bh * a.nblk + r0 + r) * a.nblk;
      for (int j = tid; j < a.nblk; j += kThreads) dst[j] = sc[r * ld + j];
    }
  }

  // ---- phase 2: one warp per row -------------------------------------------
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t lt = lanemask_lt();
  for (int r = warp; r < rows; r += kWarps) {
    const int i = r0 + r;  // query block = diagonal key block
    const float* row = sc + r * ld;
    const size_t orow = (size_t)bh * a.nblk + i;
    int32_t* out = a.kept_idx + orow * a.K_capacity;

    int mode;  // 0: diagonal only, 1: everything, 2: radix select, 3: threshold
    uint32_t tau = 0;
    int need_eq = 0;
    if (a.threshold_mode) {
      mode = 3;
    } else if (a.keep <= 1) {
      mode = 0;
    } else if (a.keep >= a.nblk) {
      mode = 1;
    } else {
      mode = 2;
      radix_select(row, a.nblk, i, a.keep - 1, hist + warp * 256, tau, need_eq);
    }

    int written = 0, eq_taken = 0;
    for (int j0 = 0; j0 < a.nblk; j0 += 32) {
      const int j = j0 + lane;
      const bool inr = j < a.nblk;
      const bool diag = inr && j == i;
      bool take = diag;
      bool eq = false;
      if (inr && !diag) {
        if (mode == 1) {
          take = true;
        } else if (mode == 2) {
          const uint32_t key = order_key(row[j]);
          take = key > tau;
          eq = key == tau;
        } else if (mode == 3) {
          take = row[j] >= a.tau;
        }
      }
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      if (eq) take = (eq_taken + __popc(eqb & lt)) < need_eq;
      const uint32_t tb = __ballot_sync(0xffffffffu, take);
      if (take) out[written + __popc(tb & lt)] = j;
      written += __popc(tb);
      eq_taken += __popc(eqb);
    }
    for (int e = written + lane; e < a.K_capacity; e += 32) out[e] = -1;
    if (lane == 0) a.kept_cnt[orow] = written;
  }
}

size_t select_smem_bytes(int R, int ld) {
  return ((size_t)R * kHeadDim + (size_t)R * ld) * sizeof(float) + (size_t)kWarps * 256 * sizeof(uint32_t);
}

constexpr size_t kSmemBudget = 100 * 1024;     // preferred: several CTAs per SM
constexpr size_t kSmemMax = 227 * 1024;

template <int R>
int launch_R(const SelectArgs& a, int ld, cudaStream_t stream) {
  const size_t smem = select_smem_bytes(R, ld);
  auto k = select_kernel<R>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SBATTN_ERR_CUDA;
  const long groups = (a.nblk + R - 1) / R;
  const long grid = groups * (long)a.B * a.H;
  k<<<(unsigned)grid, kThreads, smem, stream>>>(a, ld);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace

int select_max_nblk() {
  // R = 1 must fit: 128 + ld floats + histograms
  return (int)((kSmemMax - kWarps * 256 * sizeof(uint32_t)) / sizeof(float)) - kHeadDim - 4;
}

int launch_select(const SelectArgs& a, cudaStream_t stream) {
  const int ld = (a.nblk + 3) & ~3;  // keep rows 16-byte aligned
  if (select_smem_bytes(8, ld) <= kSmemBudget) return launch_R<8>(a, ld, stream);
  if (select_smem_bytes(4, ld) <= kSmemBudget) return launch_R<4>(a, ld, stream);
  if (select_smem_bytes(2, ld) <= kSmemBudget) return launch_R<2>(a, ld, stream);
  if (select_smem_bytes(1, ld) <= kSmemMax) return launch_R<1>(a, ld, stream);
  return SBATTN_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace sbattn
