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
struct Cached {
  CUcontext ctx;  // context the address belongs to
  float* ptr;
};
Cached g_cache[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

// Device address of the scratch array in the current device's current
// context.  It is looked up (cudaGetSymbolAddress, with that device current)
// on the first call in each context and again whenever the current context of
// the device changes (after cudaDeviceReset, or when the caller makes another
// context current), so a cached address never outlives its context.  Under
// CUDA's lazy module loading the lookup is also what loads the module holding
// the array, i.e. the moment its 4 MiB are created on that device.
int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBATTN_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return SBATTN_ERR_CUDA;
  CUcontext ctx = nullptr;  // stays null until the runtime has made a context current
  if (get_ctx(&ctx) != CUDA_SUCCESS) return SBATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_cache[dev];
  if (c.ptr == nullptr || ctx == nullptr || c.ctx != ctx) {
    void* p = nullptr;  // the lookup also makes the device's primary context current if none is
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return SBATTN_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return SBATTN_ERR_CUDA;
    c.ctx = ctx;
    c.ptr = static_cast<float*>(p);
  }
  *out = c.ptr;
  return SBATTN_OK;
}

}  // namespace

extern "C" SBATTN_API int sbattn_select_blocks_noalloc(const uint16_t* q_rot, const uint16_t* k_rot, int B, int N,
                                                       int H, int d, double sparsity, int32_t* kept_idx,
                                                       int32_t* kept_cnt, int K_capacity, float* scores,
                                                       void* stream) {
  using namespace sbattn;
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
  // the one check of its own: the problem must fit the built-in scratch
  if ((long long)B * H * nblk > (long long)kRows) return SBATTN_ERR_WORKSPACE;

  float* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch)) != SBATTN_OK) return rc;
  // The pooling kernel overwrites every pooled value it later reads, so the
  // scratch needs no clearing between calls.
  float* q_bar = scratch;
  float* k_bar = scratch + (size_t)B * H * nblk * kHeadDim;
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
