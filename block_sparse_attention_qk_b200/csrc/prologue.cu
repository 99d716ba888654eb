// Fused per-head QK-RMSNorm + 3D RoPE (xiaodao.ai "MiniMax-H3 的 6.24 倍，不能
// 直接算成六倍产能", section "先把近两倍的免费收益拿走": one kernel for QK RMSNorm
// and 3D RoPE), optionally emitting the 64-token block means that the SubBlock
// selector scores (same page, section "6.24 倍里，真正有损的部分大约是三倍").
//
// HBM-bound.  Mapping: a CTA owns one 64-token block of one batch and 8 heads
// (128 "columns" of 16 bytes = 8 channels each); each thread walks the block's
// tokens in order, so a warp reads and writes 512 contiguous bytes per token
// (two heads x 256 B) with 128-bit accesses (read-only-path loads and plain
// write-back stores: faster here than the streaming cache hints), the rows of
// the next two tokens loaded ahead.  The 16 threads of a row reduce
// the sum of squares with 4 xor-shuffles.  The (cos, sin) table of every grid
// position and rotary frequency is built once per CTA in shared memory from
// fp64 sin/cos; CTAs are persistent over blocks so the table cost is
// amortised.  Pooled means are summed in token order in fp32 from the
// bf16-rounded outputs, so they are exactly what a separate pass over the
// stored outputs computes.
#include "internal.h"

namespace sbattn {

namespace {

constexpr int kThreads = 128;       // 8 heads x 16 chunks
constexpr int kChunks = kHeadDim / 8;  // 16-byte chunks per row
constexpr int kAhead = 2;              // tokens loaded ahead

SB_DEV void bf16x8_to_f32(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

SB_DEV uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// Rotation-table layout: entries (cos, sin) for axis a at
// tab[off_a + pos * (D_a / 2) + m].
struct RopeTable {
  int off[3];
  int half[3];   // D_a / 2
  int extent[3]; // T, Hh, W
  int entries;
};

template <bool kNormRope, bool kPool>
__global__ void __launch_bounds__(kThreads) prologue_kernel(PrologueArgs a, RopeTable rt) {
  extern __shared__ float2 tab[];
  __shared__ double inv_freq[kHeadDim / 2];  // theta^(-2m/D) per section pair

  if constexpr (kNormRope) {
    for (int p = threadIdx.x; p < kHeadDim / 2; p += kThreads) {
      const int axis = p < rt.half[0] ? 0 : (p < rt.half[0] + rt.half[1] ? 1 : 2);
      const int m = p - (axis > 0 ? rt.half[0] : 0) - (axis > 1 ? rt.half[1] : 0);
      inv_freq[p] = pow((double)a.theta, -(2.0 * m) / (2.0 * rt.half[axis]));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < rt.entries; e += kThreads) {
      const int axis = (e >= rt.off[2]) ? 2 : (e >= rt.off[1]) ? 1 : 0;
      const int local = e - rt.off[axis];
      const int pos = local / rt.half[axis];
      const int m = local - pos * rt.half[axis];
      const int pair = m + (axis > 0 ? rt.half[0] : 0) + (axis > 1 ? rt.half[1] : 0);
      double sn, cs;
      sincos((double)pos * inv_freq[pair], &sn, &cs);  // angle pos * theta^(-2m/D) in fp64
      tab[e] = make_float2((float)cs, (float)sn);
    }
    __syncthreads();
  }

  const int col = blockIdx.x * kThreads + threadIdx.x;
  const bool active = col < a.H * kChunks;
  const int h = active ? col / kChunks : 0;
  const int c = col % kChunks;
  const int b = blockIdx.z;

  float wq[8], wk[8];
  int axis = 0, m0 = 0;
  if constexpr (kNormRope) {
    uint4 vq = *reinterpret_cast<const uint4*>(a.w_q + c * 8);
    uint4 vk = *reinterpret_cast<const uint4*>(a.w_k + c * 8);
    bf16x8_to_f32(vq, wq);
    bf16x8_to_f32(vk, wk);
    const int pair0 = c * 4;  // first of the 4 rotation pairs this thread owns
    const int h_t = rt.half[0], h_h = rt.half[1];
    if (pair0 < h_t) {
      axis = 0; m0 = pair0;
    } else if (pair0 < h_t + h_h) {
      axis = 1; m0 = pair0 - h_t;
    } else {
      axis = 2; m0 = pair0 - h_t - h_h;
    }
  }

  const size_t row_stride = (size_t)a.H * kHeadDim;  // elements between tokens
  const size_t base = ((size_t)b * a.N * a.H + h) * kHeadDim + c * 8;
  const float inv_d = 1.0f / (float)kHeadDim;

  for (int blk = blockIdx.y; blk < a.nblk; blk += gridDim.y) {
    const int n0 = blk * kBlock;
    const int n1 = min(a.N, n0 + kBlock);
    float qs[8], ks[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qs[e] = ks[e] = 0.f;

    // grid coordinates of token n0, advanced incrementally
    int pt = 0, ph = 0, pw = 0;
    if constexpr (kNormRope) {
      pt = n0 / (a.Hh * a.W);
      int rem = n0 - pt * a.Hh * a.W;
      ph = rem / a.W;
      pw = rem - ph * a.W;
    }

    // the rows of the next kAhead tokens are loaded ahead (a ring of kAhead
    // registers per tensor, indexed by the token's position in the ring, so
    // the loop is unrolled by kAhead), keeping 2 * kAhead 16-byte loads in
    // flight per thread
    uint4 rq[kAhead], rk[kAhead];
#pragma unroll
    for (int i = 0; i < kAhead; ++i) {
      rq[i] = rk[i] = make_uint4(0, 0, 0, 0);
      if (active && n0 + i < n1) {
        rq[i] = __ldg(reinterpret_cast<const uint4*>(a.q + base + (size_t)(n0 + i) * row_stride));
        rk[i] = __ldg(reinterpret_cast<const uint4*>(a.k + base + (size_t)(n0 + i) * row_stride));
      }
    }
    for (int nb = n0; nb < n1; nb += kAhead) {
#pragma unroll
      for (int i = 0; i < kAhead; ++i) {
        const int n = nb + i;
        if (n >= n1) break;  // (the same for every thread of the CTA)
        const size_t off = base + (size_t)n * row_stride;
        const uint4 vq = rq[i], vk = rk[i];
        if (active && n + kAhead < n1) {
          rq[i] = __ldg(reinterpret_cast<const uint4*>(a.q + off + kAhead * row_stride));
          rk[i] = __ldg(reinterpret_cast<const uint4*>(a.k + off + kAhead * row_stride));
        }
        float xq[8], xk[8];
        bf16x8_to_f32(vq, xq);
        bf16x8_to_f32(vk, xk);
        if constexpr (kNormRope) {
          float ssq = 0.f, ssk = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ssq = fmaf(xq[e], xq[e], ssq);
            ssk = fmaf(xk[e], xk[e], ssk);
          }
#pragma unroll
          for (int o = 8; o >= 1; o >>= 1) {  // the 16 threads of one row
            ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
            ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
          }
          const float rq_ = 1.0f / sqrtf(ssq * inv_d + a.eps);
          const float rk_ = 1.0f / sqrtf(ssk * inv_d + a.eps);
          const int pos = axis == 0 ? pt : (axis == 1 ? ph : pw);
          const float2* cs = tab + rt.off[axis] + pos * rt.half[axis] + m0;
          uint32_t oq[4], ok[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 t = cs[p];
            float a0 = xq[2 * p] * rq_ * wq[2 * p], a1 = xq[2 * p + 1] * rq_ * wq[2 * p + 1];
            float y0 = a0 * t.x - a1 * t.y, y1 = a0 * t.y + a1 * t.x;
            oq[p] = pack_bf16x2_rn(y0, y1);
            a0 = xk[2 * p] * rk_ * wk[2 * p];
            a1 = xk[2 * p + 1] * rk_ * wk[2 * p + 1];
            y0 = a0 * t.x - a1 * t.y;
            y1 = a0 * t.y + a1 * t.x;
            ok[p] = pack_bf16x2_rn(y0, y1);
          }
          const uint4 wq4 = make_uint4(oq[0], oq[1], oq[2], oq[3]);
          const uint4 wk4 = make_uint4(ok[0], ok[1], ok[2], ok[3]);
          if (active) {
            *reinterpret_cast<uint4*>(a.q_out + off) = wq4;
            *reinterpret_cast<uint4*>(a.k_out + off) = wk4;
          }
          if constexpr (kPool) {
            bf16x8_to_f32(wq4, xq);
            bf16x8_to_f32(wk4, xk);
          }
          if (++pw == a.W) {
            pw = 0;
            if (++ph == a.Hh) { ph = 0; ++pt; }
          }
        }
        if constexpr (kPool) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            qs[e] += xq[e];
            ks[e] += xk[e];
          }
        }
      }
    }

    if constexpr (kPool) {
      if (active) {
        const float inv = 1.0f / (float)(n1 - n0);
        const size_t po = (((size_t)b * a.H + h) * a.nblk + blk) * kHeadDim + c * 8;
        float4* pq = reinterpret_cast<float4*>(a.q_pool + po);
        float4* pk = reinterpret_cast<float4*>(a.k_pool + po);
        pq[0] = make_float4(qs[0] * inv, qs[1] * inv, qs[2] * inv, qs[3] * inv);
        pq[1] = make_float4(qs[4] * inv, qs[5] * inv, qs[6] * inv, qs[7] * inv);
        pk[0] = make_float4(ks[0] * inv, ks[1] * inv, ks[2] * inv, ks[3] * inv);
        pk[1] = make_float4(ks[4] * inv, ks[5] * inv, ks[6] * inv, ks[7] * inv);
      }
    }
  }
}

RopeTable make_table(const PrologueArgs& a) {
  RopeTable rt{};
  const int ext[3] = {a.T, a.Hh, a.W};
  const int dims[3] = {a.dim_t, a.dim_h, a.dim_w};
  int off = 0;
  for (int i = 0; i < 3; ++i) {
    rt.off[i] = off;
    rt.half[i] = dims[i] / 2;
    rt.extent[i] = ext[i];
    off += ext[i] * (dims[i] / 2);
  }
  rt.entries = off;
  return rt;
}

// Persistent grid: exactly as many CTAs as fit on the GPU at once (so there
// is no partial second wave), split over column groups and batches.
template <typename Kernel>
int grid_y_for(Kernel k, size_t smem, int nblk, int col_groups, int B, int sm_count) {
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  long want = (long)sm_count * per_sm / ((long)col_groups * B);
  if (want < 1) want = 1;
  if (want > nblk) want = nblk;
  return (int)want;
}

}  // namespace

size_t prologue_table_bytes(int T, int Hh, int W, int dim_t, int dim_h, int dim_w) {
  return ((size_t)T * (dim_t / 2) + (size_t)Hh * (dim_h / 2) + (size_t)W * (dim_w / 2)) * sizeof(float2);
}

int launch_prologue(const PrologueArgs& a, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int col_groups = (a.H * kChunks + kThreads - 1) / kThreads;
  const RopeTable rt = make_table(a);
  const size_t smem = (size_t)rt.entries * sizeof(float2);
  auto k = a.q_pool != nullptr ? prologue_kernel<true, true> : prologue_kernel<true, false>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SBATTN_ERR_CUDA;
  dim3 grid(col_groups, grid_y_for(k, smem, a.nblk, col_groups, a.B, sms), a.B);
  k<<<grid, kThreads, smem, stream>>>(a, rt);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

int launch_pool(const PrologueArgs& a, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int col_groups = (a.H * kChunks + kThreads - 1) / kThreads;
  auto k = prologue_kernel<false, true>;
  dim3 grid(col_groups, grid_y_for(k, 0, a.nblk, col_groups, a.B, sms), a.B);
  RopeTable rt{};
  k<<<grid, kThreads, 0, stream>>>(a, rt);
  return cudaGetLastError() == cudaSuccess ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace sbattn
