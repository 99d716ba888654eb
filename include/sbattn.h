/*
 * sbattn.h -- C ABI of the block-sparse video attention library (sm_100a).
 *
 * The library computes one video-DiT attention layer's hot path:
 *   1. sbattn_qk_norm_rope    fused per-head QK-RMSNorm + 3D RoPE;
 *   2. sbattn_select_blocks   SubBlock block selection: 64-token blocks,
 *                             mean-pooled block scores, per query block the
 *                             diagonal key block plus the top-scoring ones;
 *   3. sbattn_forward         attention over the kept key blocks only.
 *
 * Sources (web pages, cited by title and section):
 *   [p3] xiaodao.ai "MiniMax-H3 的 6.24 倍，不能直接算成六倍产能":
 *        section "先把近两倍的免费收益拿走" -- fused QK RMSNorm and 3D RoPE
 *        kernel, fewer intermediate tensors, memory traffic and launches;
 *        section "6.24 倍里，真正有损的部分大约是三倍" -- SubBlock cuts query
 *        and key into 64-token blocks, estimates which key blocks contribute
 *        little and keeps only the high-scoring ones for a block-sparse
 *        attention kernel; sparsity 0.75 keeps about a quarter.
 *   [p4] chat-gpts.plus "MiniMax-H3 在 8×H200 上基准测试：无损加速 1.95×，
 *        最高 6.24×（SSIM 0.76-0.91）", section "事件核心：发生了什么" --
 *        SubBlock skips attention blocks below a threshold.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Activations are bfloat16 bit patterns (uint16_t), contiguous, laid out
 *    [B, N, H, d] (batch, token, head, channel; channel fastest), the layout a
 *    fused QKV projection writes and the output projection reads.
 *  - d must be 128.  N is the token count; tokens are cut into nblk =
 *    ceil(N / 64) blocks of 64 (the last one may be partial).
 *  - All tensor pointers are DEVICE pointers owned by the caller and must be
 *    16-byte aligned.  The library allocates and frees nothing, keeps no state
 *    between calls, never synchronises, and launches only on `stream`
 *    (a cudaStream_t passed as void*; NULL means the legacy default stream).
 *  - Every call returns an int status (SBATTN_OK on success).  Argument
 *    errors are detected on the host before anything is launched; a call that
 *    returns an error has launched nothing.  SBATTN_ERR_CUDA reports a launch
 *    failure (cudaGetLastError after the launch).
 *  - Calls are asynchronous: results are ready once the stream reaches them.
 */
#ifndef SBATTN_H
#define SBATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SBATTN_API __attribute__((visibility("default")))
#else
#define SBATTN_API
#endif

/* ---- status codes ------------------------------------------------------ */
#define SBATTN_OK                    0
#define SBATTN_ERR_INVALID_ARG       1  /* null pointer, negative size, bad number */
#define SBATTN_ERR_UNSUPPORTED_SHAPE 2  /* d != 128, N != T*Hh*W, bad RoPE split, too large */
#define SBATTN_ERR_MISALIGNED        3  /* a tensor pointer is not 16-byte aligned */
#define SBATTN_ERR_WORKSPACE         4  /* workspace missing or too small */
#define SBATTN_ERR_CUDA              5  /* CUDA runtime error at launch */
#define SBATTN_ERR_DEVICE            6  /* a device-side check failed (see status word) */
#define SBATTN_ERR_TIMEOUT           7  /* a bounded wait inside a kernel ran out */
#define SBATTN_ERR_CAPACITY          8  /* kept-list capacity smaller than the budget */

#define SBATTN_BLOCK 64                 /* tokens per block ([p3], "6.24 倍里…") */

/* Human-readable name of a status code (static string, never NULL). */
SBATTN_API const char* sbattn_strerror(int status);

/* Waits until `stream` has finished all work queued on it so far, then
 * reports the first error found (this call synchronises; use it in tests,
 * debug paths or at the end of a step, not inside a timed loop):
 *   SBATTN_ERR_CUDA  an asynchronous CUDA error surfaced (a failed kernel);
 *   the nonzero code a kernel stored in the device status word `status`
 *                    (SBATTN_ERR_DEVICE or SBATTN_ERR_TIMEOUT, see
 *                    sbattn_forward), read back with one 4-byte copy on
 *                    `stream`;
 *   SBATTN_OK        otherwise.
 *   status   optional device int32 (NULL: only the stream is checked); it is
 *            read, not cleared.  4-byte aligned, else MISALIGNED.
 * The library keeps no global error state: the status word is the caller's.
 */
SBATTN_API int sbattn_check_status(const int32_t* status, void* stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
SBATTN_API int sbattn_version(void);

/* ---- 1. fused QK-RMSNorm + 3D RoPE -------------------------------------
 * [p3] "先把近两倍的免费收益拿走": QK RMSNorm and 3D RoPE fused in one kernel.
 *
 * For every (b, n, h) and X in {Q, K}, with x the d-vector of that row:
 *     r = 1 / sqrt(mean_c(x_c^2) + eps);   y = x * r * w_X   (w_X: [d])
 * then the 3D rotary embedding: token n of the T x Hh x W latent grid sits at
 * t = n / (Hh*W), h = (n / W) % Hh, w = n % W; channels [0, dim_t) rotate with
 * t, [dim_t, dim_t+dim_h) with h, the last dim_w with w; inside a section of
 * size D starting at channel o, the pair (o+2m, o+2m+1) turns by
 * pos * theta^(-2m/D):  (a, b) -> (a cos - b sin, a sin + b cos).
 * Arithmetic in fp32, output rounded to bf16 (nearest even).
 *
 *   q, k          [B, N, H, d] bf16 input, N = T*Hh*W
 *   w_q, w_k      [d] bf16 RMSNorm weights (shared by all heads)
 *   q_out, k_out  [B, N, H, d] bf16 output; may alias q / k (in place)
 *   dim_t+dim_h+dim_w == d, each even and a multiple of 8
 *   q_pool, k_pool  optional (may be NULL, both or neither): fp32
 *                 [B, H, nblk, d] block means of q_out / k_out, i.e. the
 *                 pooled vectors sbattn_select_blocks_pooled consumes; writing
 *                 them here saves re-reading q_out / k_out.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (d != 128, bad split, grid whose
 * rotation table exceeds 160 KiB), MISALIGNED, CUDA.
 */
SBATTN_API int sbattn_qk_norm_rope(const uint16_t* q, const uint16_t* k,
                                   const uint16_t* w_q, const uint16_t* w_k,
                                   uint16_t* q_out, uint16_t* k_out,
                                   float* q_pool, float* k_pool,
                                   int B, int T, int Hh, int W, int H, int d,
                                   int dim_t, int dim_h, int dim_w,
                                   float theta, float eps, void* stream);

/* ---- 2. block selection (SubBlock, budget form) -------------------------
 * [p3] "6.24 倍里，真正有损的部分大约是三倍".
 *
 * Kept blocks per query block: K = ceil((1 - s) * nblk), with s read as a
 * decimal of at most six fractional digits (s_micro = llround(s * 1e6);
 * K = ceil((1e6 - s_micro) * nblk / 1e6) in exact integer arithmetic),
 * clamped to [1, nblk].  Rejects s outside [0, 1] or NaN with INVALID_ARG.
 * Host-only; needs no GPU.
 */
SBATTN_API int sbattn_keep_count(int nblk, double sparsity, int* K_out);

/* Workspace bytes sbattn_select_blocks needs: two fp32 [B, H, nblk, d]
 * pooled tensors (2 * B*H*nblk*d*4 bytes).  Returns 0 on invalid sizes. */
SBATTN_API size_t sbattn_select_workspace_bytes(int B, int N, int H, int d);

/* For every (b, h) and query block i:
 *   q_bar_i = mean of the (up to) 64 rows of q_rot in block i (k_bar likewise);
 *   score s_ij = q_bar_i . k_bar_j  (fp32; computed on the tensor cores from
 *   tf32 pieces of each operand, three products, within a few 1e-6 of
 *   |q_bar_i| |k_bar_j| of the exact dot product; the selection below is
 *   exact on these scores);
 *   kept(i) = {i} + the K-1 highest-scoring j != i (equal scores: lower j
 *   first), written sorted ascending.
 *
 *   q_rot, k_rot  [B, N, H, d] bf16 (the prologue's output)
 *   kept_idx      [B, H, nblk, K_capacity] int32 output; row (b,h,i) holds
 *                 its kept block ids in entries [0, kept_cnt); entries past
 *                 kept_cnt are set to -1
 *   kept_cnt      [B, H, nblk] int32 output (= K for every row)
 *   K_capacity    >= K, else SBATTN_ERR_CAPACITY
 *   scores        optional fp32 [B, H, nblk, nblk] output of s_ij (NULL to skip)
 *   workspace     device scratch of >= sbattn_select_workspace_bytes bytes,
 *                 16-byte aligned; its contents on entry do not matter
 */
SBATTN_API int sbattn_select_blocks(const uint16_t* q_rot, const uint16_t* k_rot,
                                    int B, int N, int H, int d, double sparsity,
                                    int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                    float* scores, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Same selection from already pooled fp32 [B, H, nblk, d] block means (as
 * written by sbattn_qk_norm_rope's q_pool / k_pool).  No workspace. */
SBATTN_API int sbattn_select_blocks_pooled(const float* q_bar, const float* k_bar,
                                           int B, int nblk, int H, int d, double sparsity,
                                           int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                           float* scores, void* stream);

/* Threshold form ([p4] "事件核心…": blocks scoring below a threshold are
 * skipped): kept(i) = {i} + every j != i with s_ij >= tau, sorted ascending;
 * kept_cnt varies per row (1..nblk); K_capacity must be >= nblk.
 * Inputs are pooled means as for sbattn_select_blocks_pooled. */
SBATTN_API int sbattn_select_blocks_threshold(const float* q_bar, const float* k_bar,
                                              int B, int nblk, int H, int d, float tau,
                                              int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                              float* scores, void* stream);

/* Same selection as sbattn_select_blocks, for callers that cannot allocate
 * device memory when they run the layer -- a plugin-style host that passes
 * the library only the layer's inputs and outputs and owns all other device
 * memory, or a runtime that plans its memory up front and forbids allocation
 * once serving.  The pages have no counterpart to this call; it exists only
 * for such callers.
 *
 * The pooled block means live in a fixed scratch array compiled into the
 * library (4 MiB of device memory, held until the process exits), so the
 * call allocates nothing and takes no workspace.  Limit: B * H * ceil(N/64)
 * <= SBATTN_NOALLOC_MAX_POOLED_ROWS; larger problems are rejected with
 * SBATTN_ERR_WORKSPACE before anything is launched (use sbattn_select_blocks
 * with a workspace for them).
 *
 * Warm-up: the first call in each context looks up that device's address of
 * the array (with the device current).  Under CUDA's lazy module loading
 * (the default) that lookup is also what loads the library module holding
 * the array, so the first call on a device is the one that creates its
 * 4 MiB; until then the array does not exist on that device.  Make one call
 * on every device before the point where allocation becomes forbidden, and
 * before any stream capture.  The address is cached per device and looked up
 * again when the device's current context changes (after cudaDeviceReset or
 * when another context is made current).
 *
 * All calls on a device share the one array and each call overwrites every
 * value it reads, so nothing needs clearing between calls; but calls whose
 * work overlaps on the GPU (different streams, or different host threads,
 * without ordering between them) race on it.
 * Other arguments, outputs and errors as for sbattn_select_blocks.
 */
#define SBATTN_NOALLOC_MAX_POOLED_ROWS 4096
SBATTN_API int sbattn_select_blocks_noalloc(const uint16_t* q_rot, const uint16_t* k_rot,
                                            int B, int N, int H, int d, double sparsity,
                                            int32_t* kept_idx, int32_t* kept_cnt, int K_capacity,
                                            float* scores, void* stream);

/* ---- 3. block-sparse attention -----------------------------------------
 * [p3] "6.24 倍里…": only the kept key blocks enter the attention kernel.
 *
 * For every (b, h) and query block i with S = tokens of the kept key blocks
 * kept_idx[b,h,i,0:kept_cnt[b,h,i]]:
 *     O_i = softmax(Q_i K_S^T * scale) V_S      (non-causal; keys outside S
 *                                                contribute nothing)
 * bf16 tensor-core products with fp32 accumulation and an fp32 softmax.
 *
 *   q_rot, k_rot, v [B, N, H, d] bf16
 *   kept_idx        [B, H, nblk, K_capacity] int32, each entry in [0, nblk),
 *                   no repeats within a row (any order)
 *   kept_cnt        [B, H, nblk] int32, each in [1, K_capacity]
 *   out             [B, N, H, d] bf16 output (must not alias the inputs)
 *   softmax_scale   <= 0 selects 1/sqrt(d)
 *   status          optional device int32 (may be NULL).  If given, the
 *                   kernel stores a nonzero SBATTN_ERR_* code there when a
 *                   kept index or count is out of range (that block/row is
 *                   skipped; DEVICE) or when a bounded internal wait runs out
 *                   (TIMEOUT); it never clears it.  Zero it before the call
 *                   and read it after the stream has reached the call (e.g.
 *                   with sbattn_check_status).
 * The softmax is exact for any logit range: the running maximum of a query
 * is raised before any weight of a step is computed whenever the step's
 * logits exceed it by more than 2^8 (so every weight is at most 2^8).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (d != 128), MISALIGNED, CUDA.
 */
SBATTN_API int sbattn_forward(const uint16_t* q_rot, const uint16_t* k_rot, const uint16_t* v,
                              const int32_t* kept_idx, const int32_t* kept_cnt, int K_capacity,
                              uint16_t* out, int B, int N, int H, int d,
                              float softmax_scale, int32_t* status, void* stream);

/* Failure-detection form of sbattn_forward (the pages have no counterpart;
 * it exists so that tests can show that the kernel's internal waits are
 * bounded).  Same computation and arguments, plus:
 *   wait_limit_ns    limit of every bounded wait inside the kernel, in
 *                    [1 ms, 20 s] (sbattn_forward uses 2 s)
 *   withhold_v_tile  -1 for a normal call; t >= 0 makes every CTA skip the
 *                    copy of its t-th V tile (counted in the CTA's own order
 *                    of kept-block pairs), so the wait for that tile runs out:
 *                    the kernel then stores SBATTN_ERR_TIMEOUT in `status`,
 *                    lets its own copies and matrix products finish, frees
 *                    its tensor memory and returns; the outputs of the call
 *                    are undefined, the device stays usable.
 * Errors: as sbattn_forward; INVALID_ARG for a limit or tile out of range.
 */
SBATTN_API int sbattn_forward_diag(const uint16_t* q_rot, const uint16_t* k_rot, const uint16_t* v,
                                   const int32_t* kept_idx, const int32_t* kept_cnt, int K_capacity,
                                   uint16_t* out, int B, int N, int H, int d, float softmax_scale,
                                   int32_t* status, unsigned long long wait_limit_ns, int withhold_v_tile,
                                   void* stream);

/* ---- 4. fused DiT-block elementwise steps around attention -------------
 * [p3] "先把近两倍的免费收益拿走": the lossless gain also comes from fused
 * AdaLN and SwiGLU kernels (fewer intermediate tensors, memory passes and
 * launches).  The page names the operations only; these are the standard
 * DiT definitions.
 *
 * AdaLN: for every token row x (C channels) of sample b,
 *     y = (x - mean(x)) / sqrt(var(x) + eps) * (1 + scale_b) + shift_b
 * with the biased (1/C) variance and no learned LayerNorm affine; shift and
 * scale are the per-sample conditioning vectors.  One pass: fp32 statistics
 * and arithmetic, output rounded to bf16 (nearest even).
 *
 *   x            [B, N, C] bf16 input
 *   shift, scale [B, C] bf16 conditioning vectors
 *   out          [B, N, C] bf16 output; may alias x (in place)
 *   C            a multiple of 8, at most 6144 (a row is held in registers)
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (C), MISALIGNED, CUDA.
 */
SBATTN_API int sbattn_adaln_modulate(const uint16_t* x, const uint16_t* shift, const uint16_t* scale,
                                     uint16_t* out, int B, int N, int C, float eps, void* stream);

/* SwiGLU: out[r, f] = silu(gate[r, f]) * up[r, f], silu(a) = a / (1 + e^-a),
 * fp32 arithmetic, output rounded to bf16 (nearest even).
 *
 *   gate, up     bf16 rows of F elements, row r at gate + r * ld_in (the two
 *                halves of a fused [rows, 2F] projection output have
 *                ld_in = 2F and up = gate + F; separate tensors ld_in = F)
 *   out          [rows, F] bf16, contiguous; must not overlap gate / up
 *   F, ld_in     multiples of 8, ld_in >= F
 * Errors: INVALID_ARG, MISALIGNED, CUDA.
 */
SBATTN_API int sbattn_swiglu(const uint16_t* gate, const uint16_t* up, uint16_t* out,
                             int64_t rows, int F, int64_t ld_in, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SBATTN_H */
