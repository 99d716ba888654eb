// Block selection without any caller-provided scratch memory.
//
// sbattn_select_blocks needs a device workspace for the pooled block means,
// which the caller normally allocates.  Some callers cannot allocate device
// memory at the point where they run the layer: for example a plugin-style
// host that hands the library only the layer's input and output buffers and
// owns every other byte of device memory itself, or a runtime that plans all
// device memory up front and forbids allocation once it is serving.  For
// them, this file keeps the scratch in a fixed, file-scope device array
// (sized by SBATTN_NOALLOC_MAX_POOLED_ROWS) that is part of the loaded
// library, so the call itself allocates nothing.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kRows = SBATTN_NOALLOC_MAX_POOLED_ROWS;                    // B*H*nblk limit
constexpr size_t kScratchFloats = 2 * kRows * sbattn::kHeadDim;             // q_bar and k_bar
static_assert(kScratchFloats * sizeof(float) == 4u << 20, "the header documents 4 MiB");

// Lives in every GPU that loads the library, until the process exits.  Host
// code must never hand this symbol to a kernel directly: on the host it is
// only a stand-in, not a device address; the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) float g_select_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_dev_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the first call on each device does it).
int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_dev_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return SBATTN_ERR_CUDA;
    g_dev_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_dev_ptr[dev];
  return SBATTN_OK;
}

}  // namespace

extern "C" SBATTN_API int sbattn_select_blocks_noalloc(const uint16_t* q_rot, const uint16_t* k_rot, int B, int N,
                                                       int H, int d, double sparsity, int32_t* kept_idx,
                                                       int32_t* kept_cnt, int K_capacity, float* scores,
                                                       void* stream) {
  using namespace sbattn;
  if (!q_rot || !k_rot || !kept_idx || !kept_cnt) return SBATTN_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1 || d < 1) return SBATTN_ERR_INVALID_ARG;
  if (d != kHeadDim) return SBATTN_ERR_UNSUPPORTED_SHAPE;
  const long long nblk = ((long long)N + kBlock - 1) / kBlock;
  if ((long long)B * H * nblk > (long long)kRows) return SBATTN_ERR_WORKSPACE;  // beyond the built-in scratch
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q_rot) | reinterpret_cast<uintptr_t>(k_rot) |
                        reinterpret_cast<uintptr_t>(kept_idx) | reinterpret_cast<uintptr_t>(kept_cnt) |
                        reinterpret_cast<uintptr_t>(scores);
  if (mis & 15u) return SBATTN_ERR_MISALIGNED;
  int K = 0;
  int rc = sbattn_keep_count((int)nblk, sparsity, &K);
  if (rc != SBATTN_OK) return rc;
  if (K_capacity < K) return SBATTN_ERR_CAPACITY;

  float* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch)) != SBATTN_OK) return rc;
  // The pooling kernel overwrites every pooled value it later reads, so the
  // scratch needs no clearing between calls.
  float* q_bar = scratch;
  float* k_bar = scratch + (size_t)B * H * nblk * kHeadDim;
  PrologueArgs p{};
  p.q = q_rot; p.k = k_rot; p.q_pool = q_bar; p.k_pool = k_bar;
  p.B = B; p.N = N; p.H = H; p.nblk = (int)nblk;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = launch_pool(p, s)) != SBATTN_OK) return rc;
  SelectArgs a{};
  a.q_bar = q_bar; a.k_bar = k_bar; a.B = B; a.H = H; a.nblk = (int)nblk; a.keep = K;
  a.threshold_mode = 0; a.tau = 0.f;
  a.kept_idx = kept_idx; a.kept_cnt = kept_cnt; a.K_capacity = K_capacity; a.scores = scores;
  return launch_select(a, s);
}
