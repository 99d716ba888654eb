// C ABI of the library: argument validation (entirely on the host, before any
// CUDA call), tensor-map creation and kernel launches.  See include/sbattn.h.
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace sbattn {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int nblk_of(long long N) { return (int)((N + kBlock - 1) / kBlock); }

// Common checks of a [B, N, H, d] activation set.
int check_dims(long long B, long long N, long long H, long long d) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return SBATTN_ERR_INVALID_ARG;
  if (d != kHeadDim) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  // item and element indices must stay in range of the kernels' integer types
  if (B * H * ((N + kBlock - 1) / kBlock) > 0x7FFFFFFFLL) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  if (N > 0x7FFFFFFFLL - kBlock) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  return SBATTN_OK;
}

// Output checks shared by every selection entry point.
int check_select_outputs(const int32_t* kept_idx, const int32_t* kept_cnt, const float* scores) {
  if (!kept_idx || !kept_cnt) return SBATTN_ERR_INVALID_ARG;
  if (!aligned16(kept_idx) || !aligned16(kept_cnt) || (scores && !aligned16(scores))) return SBATTN_ERR_MISALIGNED;
  return SBATTN_OK;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

// Tensor map over a [B, N, H, 128] bf16 tensor seen as 4-D (d, H, N, B); a
// box is 64 channels x 1 head x 64 tokens with 128-byte swizzle, which lands
// in shared memory as 64 rows of 128 bytes (the canonical tcgen05 operand
// tile).  Tokens past N read as zero.
int make_bf16_row_map(CUtensorMap* map, const void* base, int B, int N, int H) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return SBATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)H * kHeadDim * 2,
                                 (cuuint64_t)N * H * kHeadDim * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBlock, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SBATTN_OK : SBATTN_ERR_CUDA;
}

}  // namespace sbattn

using namespace sbattn;

extern "C" {

SBATTN_API const char* sbattn_strerror(int status) {
  switch (status) {
    case SBATTN_OK: return "ok";
    case SBATTN_ERR_INVALID_ARG: return "invalid argument";
    case SBATTN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SBATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SBATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case SBATTN_ERR_CUDA: return "CUDA runtime error";
    case SBATTN_ERR_DEVICE: return "device-side check failed";
    case SBATTN_ERR_TIMEOUT: return "bounded wait inside a kernel ran out";
    case SBATTN_ERR_CAPACITY: return "kept-list capacity smaller than the budget";
    default: return "unknown status";
  }
}

SBATTN_API int sbattn_check_status(const int32_t* status, void* stream) {
  if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u)) return SBATTN_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();  // clear a non-sticky error so that later calls start clean
    return SBATTN_ERR_CUDA;
  }
  if (status == nullptr) return SBATTN_OK;
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return SBATTN_ERR_CUDA;
  }
  if (v == SBATTN_OK) return SBATTN_OK;
  return (v >= SBATTN_ERR_INVALID_ARG && v <= SBATTN_ERR_CAPACITY) ? v : SBATTN_ERR_DEVICE;
}

SBATTN_API int sbattn_version(void) { return 1 * 10000 + 0 * 100 + 0; }

SBATTN_API int sbattn_keep_count(int nblk, double sparsity, int* K_out) {
  if (K_out == nullptr || nblk < 1) return SBATTN_ERR_INVALID_ARG;
  if (!(sparsity >= 0.0 && sparsity <= 1.0)) return SBATTN_ERR_INVALID_ARG;  // also rejects NaN
  const long long micro = llround(sparsity * 1e6);
  const long long keep_num = (1000000LL - micro) * (long long)nblk;  // K = ceil(keep_num / 1e6)
  long long K = (keep_num + 999999LL) / 1000000LL;
  if (K < 1) K = 1;
  if (K > nblk) K = nblk;
  *K_out = (int)K;
  return SBATTN_OK;
}

SBATTN_API size_t sbattn_select_workspace_bytes(int B, int N, int H, int d) {
  if (check_dims(B, N, H, d) != SBATTN_OK) return 0;
  return 2ull * (size_t)B * H * nblk_of(N) * d * sizeof(float);
}

SBATTN_API int sbattn_qk_norm_rope(const uint16_t* q, const uint16_t* k, const uint16_t* w_q,
                                   const uint16_t* w_k, uint16_t* q_out, uint16_t* k_out, float* q_pool,
                                   float* k_pool, int B, int T, int Hh, int W, int H, int d, int dim_t,
                                   int dim_h, int dim_w, float theta, float eps, void* stream) {
  if (!q || !k || !w_q || !w_k || !q_out || !k_out) return SBATTN_ERR_INVALID_ARG;
  if ((q_pool == nullptr) != (k_pool == nullptr)) return SBATTN_ERR_INVALID_ARG;
  if (T < 1 || Hh < 1 || W < 1) return SBATTN_ERR_INVALID_ARG;
  if (!(isfinite(theta) && theta > 0.f) || !(isfinite(eps) && eps >= 0.f)) return SBATTN_ERR_INVALID_ARG;
  const long long N = (long long)T * Hh * W;
  int rc = check_dims(B, N, H, d);
  if (rc != SBATTN_OK) return rc;
  if (dim_t < 0 || dim_h < 0 || dim_w < 0 || dim_t % 8 || dim_h % 8 || dim_w % 8 || dim_t + dim_h + dim_w != d)
    return SBATTN_ERR_UNSUPPORTED_SHAPE;
  if (prologue_table_bytes(T, Hh, W, dim_t, dim_h, dim_w) > kMaxRopeTableBytes) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(w_q) || !aligned16(w_k) || !aligned16(q_out) ||
      !aligned16(k_out) || (q_pool && (!aligned16(q_pool) || !aligned16(k_pool))))
    return SBATTN_ERR_MISALIGNED;
  PrologueArgs a{};
  a.q = q; a.k = k; a.w_q = w_q; a.w_k = w_k;
  a.q_out = q_out; a.k_out = k_out; a.q_pool = q_pool; a.k_pool = k_pool;
  a.B = B; a.N = (int)N; a.H = H; a.T = T; a.Hh = Hh; a.W = W; a.nblk = nblk_of(N);
  a.dim_t = dim_t; a.dim_h = dim_h; a.dim_w = dim_w; a.theta = theta; a.eps = eps;
  return launch_prologue(a, static_cast<cudaStream_t>(stream));
}

SBATTN_API int sbattn_select_blocks_pooled(const float* q_bar, const float* k_bar, int B, int nblk, int H, int d,
                                           double sparsity, int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                           float* scores, void* stream) {
  if (!q_bar || !k_bar) return SBATTN_ERR_INVALID_ARG;
  int rc = check_dims(B, (long long)nblk * kBlock, H, d);
  if (rc != SBATTN_OK) return rc;
  if ((rc = check_select_outputs(kept_idx, kept_cnt, scores)) != SBATTN_OK) return rc;
  if (!aligned16(q_bar) || !aligned16(k_bar)) return SBATTN_ERR_MISALIGNED;
  int K = 0;
  if ((rc = sbattn_keep_count(nblk, sparsity, &K)) != SBATTN_OK) return rc;
  if (K_capacity < K) return SBATTN_ERR_CAPACITY;
  if (nblk > select_max_nblk()) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  SelectArgs a{};
  a.q_bar = q_bar; a.k_bar = k_bar; a.B = B; a.H = H; a.nblk = nblk; a.keep = K;
  a.threshold_mode = 0; a.tau = 0.f;
  a.kept_idx = kept_idx; a.kept_cnt = kept_cnt; a.K_capacity = K_capacity; a.scores = scores;
  return launch_select(a, static_cast<cudaStream_t>(stream));
}

SBATTN_API int sbattn_select_blocks_threshold(const float* q_bar, const float* k_bar, int B, int nblk, int H, int d,
                                              float tau, int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                              float* scores, void* stream) {
  if (!q_bar || !k_bar || isnan(tau)) return SBATTN_ERR_INVALID_ARG;
  int rc = check_dims(B, (long long)nblk * kBlock, H, d);
  if (rc != SBATTN_OK) return rc;
  if ((rc = check_select_outputs(kept_idx, kept_cnt, scores)) != SBATTN_OK) return rc;
  if (!aligned16(q_bar) || !aligned16(k_bar)) return SBATTN_ERR_MISALIGNED;
  if (K_capacity < nblk) return SBATTN_ERR_CAPACITY;
  if (nblk > select_max_nblk()) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  SelectArgs a{};
  a.q_bar = q_bar; a.k_bar = k_bar; a.B = B; a.H = H; a.nblk = nblk; a.keep = nblk;
  a.threshold_mode = 1; a.tau = tau;
  a.kept_idx = kept_idx; a.kept_cnt = kept_cnt; a.K_capacity = K_capacity; a.scores = scores;
  return launch_select(a, static_cast<cudaStream_t>(stream));
}

SBATTN_API int sbattn_select_blocks(const uint16_t* q_rot, const uint16_t* k_rot, int B, int N, int H, int d,
                                    double sparsity, int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                    float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q_rot || !k_rot) return SBATTN_ERR_INVALID_ARG;
  int rc = check_dims(B, N, H, d);
  if (rc != SBATTN_OK) return rc;
  if ((rc = check_select_outputs(kept_idx, kept_cnt, scores)) != SBATTN_OK) return rc;
  if (!aligned16(q_rot) || !aligned16(k_rot)) return SBATTN_ERR_MISALIGNED;
  const int nblk = nblk_of(N);
  int K = 0;
  if ((rc = sbattn_keep_count(nblk, sparsity, &K)) != SBATTN_OK) return rc;
  if (K_capacity < K) return SBATTN_ERR_CAPACITY;
  if (nblk > select_max_nblk()) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  const size_t need = sbattn_select_workspace_bytes(B, N, H, d);
  if (workspace == nullptr || workspace_bytes < need) return SBATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SBATTN_ERR_MISALIGNED;
  float* q_bar = static_cast<float*>(workspace);
  float* k_bar = q_bar + (size_t)B * H * nblk * d;
  PrologueArgs p{};
  p.q = q_rot; p.k = k_rot; p.q_pool = q_bar; p.k_pool = k_bar;
  p.B = B; p.N = N; p.H = H; p.nblk = nblk;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = launch_pool(p, s)) != SBATTN_OK) return rc;
  SelectArgs a{};
  a.q_bar = q_bar; a.k_bar = k_bar; a.B = B; a.H = H; a.nblk = nblk; a.keep = K;
  a.threshold_mode = 0; a.tau = 0.f;
  a.kept_idx = kept_idx; a.kept_cnt = kept_cnt; a.K_capacity = K_capacity; a.scores = scores;
  return launch_select(a, s);
}

static int forward_impl(const uint16_t* q_rot, const uint16_t* k_rot, const uint16_t* v, const int32_t* kept_idx,
                        const int32_t* kept_cnt, int K_capacity, uint16_t* out, int B, int N, int H, int d,
                        float softmax_scale, int32_t* status, unsigned long long wait_limit_ns, int withhold_v_tile,
                        void* stream) {
  if (!q_rot || !k_rot || !v || !kept_idx || !kept_cnt || !out) return SBATTN_ERR_INVALID_ARG;
  if (out == q_rot || out == k_rot || out == v) return SBATTN_ERR_INVALID_ARG;
  if (K_capacity < 1 || isnan(softmax_scale) || isinf(softmax_scale)) return SBATTN_ERR_INVALID_ARG;
  int rc = check_dims(B, N, H, d);
  if (rc != SBATTN_OK) return rc;
  if (!aligned16(q_rot) || !aligned16(k_rot) || !aligned16(v) || !aligned16(out) || !aligned16(kept_idx) ||
      !aligned16(kept_cnt) || (status && (reinterpret_cast<uintptr_t>(status) & 3u)))
    return SBATTN_ERR_MISALIGNED;
  AttentionArgs a{};
  a.q = q_rot; a.k = k_rot; a.v = v; a.kept_idx = kept_idx; a.kept_cnt = kept_cnt; a.out = out; a.status = status;
  a.B = B; a.N = N; a.H = H; a.nblk = nblk_of(N); a.K_capacity = K_capacity;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)d);
  a.wait_limit_ns = wait_limit_ns;
  a.withhold_v_tile = withhold_v_tile;
  return launch_attention(a, static_cast<cudaStream_t>(stream));
}

SBATTN_API int sbattn_forward(const uint16_t* q_rot, const uint16_t* k_rot, const uint16_t* v,
                              const int32_t* kept_idx, const int32_t* kept_cnt, int K_capacity, uint16_t* out,
                              int B, int N, int H, int d, float softmax_scale, int32_t* status, void* stream) {
  return forward_impl(q_rot, k_rot, v, kept_idx, kept_cnt, K_capacity, out, B, N, H, d, softmax_scale, status,
                      kWaitLimitNs, -1, stream);
}

SBATTN_API int sbattn_forward_diag(const uint16_t* q_rot, const uint16_t* k_rot, const uint16_t* v,
                                   const int32_t* kept_idx, const int32_t* kept_cnt, int K_capacity, uint16_t* out,
                                   int B, int N, int H, int d, float softmax_scale, int32_t* status,
                                   unsigned long long wait_limit_ns, int withhold_v_tile, void* stream) {
  if (wait_limit_ns < 1000000ull || wait_limit_ns > 10ull * kWaitLimitNs) return SBATTN_ERR_INVALID_ARG;
  if (withhold_v_tile < -1) return SBATTN_ERR_INVALID_ARG;
  return forward_impl(q_rot, k_rot, v, kept_idx, kept_cnt, K_capacity, out, B, N, H, d, softmax_scale, status,
                      wait_limit_ns, withhold_v_tile, stream);
}

SBATTN_API int sbattn_adaln_modulate(const uint16_t* x, const uint16_t* shift, const uint16_t* scale,
                                     uint16_t* out, int B, int N, int C, float eps, void* stream) {
  if (!x || !shift || !scale || !out) return SBATTN_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || C < 1 || !(isfinite(eps) && eps >= 0.f)) return SBATTN_ERR_INVALID_ARG;
  if ((long long)B * N * C > (1ll << 40)) return SBATTN_ERR_INVALID_ARG;
  if (C % 8 != 0 || C > kMaxAdaLNChannels) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(shift) || !aligned16(scale) || !aligned16(out)) return SBATTN_ERR_MISALIGNED;
  DitArgs a{};
  a.x = x; a.shift = shift; a.scale = scale; a.out = out;
  a.B = B; a.N = N; a.C = C; a.eps = eps;
  return launch_adaln(a, static_cast<cudaStream_t>(stream));
}

SBATTN_API int sbattn_swiglu(const uint16_t* gate, const uint16_t* up, uint16_t* out, int64_t rows, int F,
                             int64_t ld_in, void* stream) {
  if (!gate || !up || !out) return SBATTN_ERR_INVALID_ARG;
  if (rows < 1 || F < 8 || F % 8 != 0 || ld_in < F || ld_in % 8 != 0) return SBATTN_ERR_INVALID_ARG;
  if (rows > (1ll << 40) / ld_in) return SBATTN_ERR_INVALID_ARG;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(out)) return SBATTN_ERR_MISALIGNED;
  SwigluArgs a{};
  a.gate = gate; a.up = up; a.out = out;
  a.rows = rows; a.ld_in = ld_in; a.F = F;
  return launch_swiglu(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
