"""Plain fp64 CPU oracle for SubBlock-style block-sparse attention with its fused
QK-RMSNorm + 3D-RoPE prologue.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
baseline leg of the benchmark may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from the product package: the two share no code.

Sources (web pages; cited by page title and section):

* [p3] xiaodao.ai, "MiniMax-H3 的 6.24 倍，不能直接算成六倍产能"
  - section "先把近两倍的免费收益拿走": the lossless runtime gain comes from
    fused kernels, among them one that applies QK RMSNorm and 3D RoPE.
  - section "6.24 倍里，真正有损的部分大约是三倍": SubBlock cuts query and key
    into 64-token blocks, estimates which key blocks contribute little, and
    sends only the high-scoring blocks to a block-sparse attention kernel;
    sparsity 0.75 means about 75 % of the key blocks may be dropped, so about
    a quarter is kept.
* [p4] chat-gpts.plus, "MiniMax-H3 在 8×H200 上基准测试：无损加速 1.95×，最高
  6.24×（SSIM 0.76-0.91）", section "事件核心：发生了什么": SubBlock skips
  attention blocks that fall below a threshold (the threshold phrasing; the
  budget phrasing of [p3] is the one implemented by `select_blocks`, the
  threshold one by `select_blocks_threshold`).

The pages print no formula.  Where they leave a step open, the plainest reading
consistent with the rest is taken, stated in each docstring:

* block importance: mean-pool the post-prologue Q and K over each 64-token
  block, score key block j for query block i by the plain dot product of the
  pooled vectors;
* budget: K = ceil((1 - s) * nblk) kept blocks per query block, the query
  block's own (diagonal) key block always among them, the rest the
  highest-scoring off-diagonal blocks, equal scores resolved towards the lower
  block index, the kept list sorted ascending;
* RMSNorm per (token, head) over the head dimension d with a learned weight of
  length d (one for Q, one for K), eps inside the square root, then RoPE;
* 3D RoPE: the head dimension is split into a t, an h and a w section; inside a
  section of size D, the interleaved pair (2m, 2m+1) is rotated by the angle
  pos * theta**(-2m / D) with (a, b) -> (a cos - b sin, a sin + b cos);
  token n of a T x Hh x W latent grid sits at t = n // (Hh W),
  h = (n // W) % Hh, w = n % W;
* attention is non-causal and the softmax runs over the kept keys only, scaled
  by 1 / sqrt(d) unless a scale is given.

Every function here is the definition written out in float64, with NumPy's
matmul / sort as the only library steps; no blocking, fusion or reordering.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

BLOCK = 64  # [p3] "6.24 倍里…": query and key are cut into 64-token blocks


# ----------------------------------------------------------------------------
# budget
# ----------------------------------------------------------------------------

def sparsity_micro(sparsity: float) -> int:
    """Sparsity as an integer count of millionths.

    The budget is read as a decimal number with at most six fractional digits,
    so that e.g. s = 0.18 means exactly 18/100 and not the binary double
    nearest to it.  The double s is multiplied by 1e6 in IEEE double precision
    and rounded half away from zero; the rounding is done exactly with
    fractions so that values such as 0.49999999999999994 are not rounded up by
    an intermediate double addition.
    """
    if not isinstance(sparsity, (float, int)) or math.isnan(sparsity):
        raise ValueError("sparsity must be a finite number")
    if sparsity < 0.0 or sparsity > 1.0:
        raise ValueError("sparsity must lie in [0, 1]")
    x = float(sparsity) * 1e6  # one IEEE double multiplication
    return int(math.floor(Fraction(x) + Fraction(1, 2)))


def keep_count(nblk: int, sparsity: float) -> int:
    """Number of key blocks kept per query block, diagonal included.

    [p3] "6.24 倍里…": sparsity s allows dropping about a fraction s of the key
    blocks, so about (1 - s) of them is kept (s = 0.75 keeps about a quarter).
    Reading: K = ceil((1 - s) * nblk), evaluated exactly on the decimal value of
    s (see `sparsity_micro`), clamped to [1, nblk] because the diagonal block is
    always kept.
    """
    if nblk < 1:
        raise ValueError("nblk must be >= 1")
    keep = Fraction(10**6 - sparsity_micro(sparsity), 10**6) * nblk
    k = math.ceil(keep)
    return max(1, min(nblk, k))


# ----------------------------------------------------------------------------
# prologue: RMSNorm then 3D RoPE
# ----------------------------------------------------------------------------

def token_positions(T: int, Hh: int, W: int) -> np.ndarray:
    """(t, h, w) integer coordinates of every token of a T x Hh x W latent grid,
    row-major: token n = (t * Hh + h) * W + w.  Shape [N, 3], int64."""
    n = np.arange(T * Hh * W, dtype=np.int64)
    return np.stack([n // (Hh * W), (n // W) % Hh, n % W], axis=1)


def rope_angles(T: int, Hh: int, W: int, dims=(32, 48, 48), theta: float = 10000.0) -> np.ndarray:
    """Rotation angle of every (token, pair): shape [N, d/2], float64.

    [p3] "先把近两倍…" names a 3D RoPE.  Reading: the head dimension is split
    into consecutive t, h and w sections of sizes dims; pair m of a section of
    size D (channels offset + 2m, offset + 2m + 1) turns by
    pos_axis * theta**(-2m / D).
    """
    pos = token_positions(T, Hh, W).astype(np.float64)
    cols = []
    for axis, D in enumerate(dims):
        if D % 2:
            raise ValueError("every RoPE section must have an even size")
        m = np.arange(D // 2, dtype=np.float64)
        inv_freq = theta ** (-2.0 * m / D)
        cols.append(pos[:, axis:axis + 1] * inv_freq[None, :])
    return np.concatenate(cols, axis=1)


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Per-row RMSNorm over the last axis: y = x / sqrt(mean(x**2) + eps) * w.

    [p3] "先把近两倍…" names QK RMSNorm; reading: over the head dimension of
    each (token, head) row, eps inside the square root, one weight of length d.
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def rope_3d(y: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate interleaved channel pairs of y [B, N, H, d] by angles [N, d/2]:
    (a, b) -> (a cos - b sin, a sin + b cos)."""
    y = np.asarray(y, dtype=np.float64)
    a = y[..., 0::2]
    b = y[..., 1::2]
    c = np.cos(angles)[None, :, None, :]
    s = np.sin(angles)[None, :, None, :]
    out = np.empty_like(y)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def qk_norm_rope(q, k, w_q, w_k, T, Hh, W, dims=(32, 48, 48), theta=10000.0, eps=1e-6):
    """Fused prologue of [p3] "先把近两倍…": RMSNorm of Q and K per (token,
    head) with their own weights, then the same 3D RoPE on both.

    q, k: [B, N, H, d] (any float dtype; promoted to float64), N = T*Hh*W.
    Returns float64 (q_rot, k_rot).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if q.shape[1] != T * Hh * W or k.shape != q.shape:
        raise ValueError("q and k must be [B, T*Hh*W, H, d]")
    if sum(dims) != q.shape[-1]:
        raise ValueError("RoPE sections must sum to d")
    ang = rope_angles(T, Hh, W, dims, theta)
    return (rope_3d(rms_norm(q, w_q, eps), ang),
            rope_3d(rms_norm(k, w_k, eps), ang))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned
    as float64.  Done in one step from float64 (no intermediate float32
    rounding).  bfloat16 keeps 8 significant bits and float32's exponent
    range; values are assumed finite and below the bfloat16 maximum."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    _, e = np.frexp(x[nz])           # |x| = f * 2**e with f in [0.5, 1)
    e = np.maximum(e - 1, -126)      # exponent of the leading bit; subnormal floor
    ulp = np.ldexp(1.0, e - 7)       # spacing of bf16 values in that binade
    out[nz] = np.rint(x[nz] / ulp) * ulp  # rint rounds half to even
    return out


# ----------------------------------------------------------------------------
# block selection
# ----------------------------------------------------------------------------

def block_pool(x: np.ndarray) -> np.ndarray:
    """Mean of each 64-token block, per (batch, head): x [B, N, H, d] ->
    [B, H, nblk, d] float64.

    [p3] "6.24 倍里…": blocks are 64 tokens; reading of "estimate": the block's
    mean vector.  A trailing partial block is averaged over its valid tokens.
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, H, d = x.shape
    nblk = -(-N // BLOCK)
    out = np.empty((B, H, nblk, d))
    for i in range(nblk):
        lo, hi = i * BLOCK, min(N, (i + 1) * BLOCK)
        out[:, :, i, :] = x[:, lo:hi].mean(axis=1)
    return out


def block_scores(q_bar: np.ndarray, k_bar: np.ndarray) -> np.ndarray:
    """Score of key block j for query block i: the dot product of the pooled
    vectors, s_ij = q_bar_i . k_bar_j.  [B, H, nblk, nblk] float64."""
    return np.einsum("bhid,bhjd->bhij", q_bar, k_bar)


def select_row(scores_row: np.ndarray, i: int, K: int) -> np.ndarray:
    """Kept key blocks of query block i from its score row.

    The diagonal block i is always kept; the other K - 1 are the
    highest-scoring j != i, equal scores going to the lower j; the list is
    returned sorted ascending (int64)."""
    nblk = scores_row.shape[0]
    others = np.array([j for j in range(nblk) if j != i], dtype=np.int64)
    # full stable sort by (-score, j): lexsort's last key is the primary one
    order = np.lexsort((others, -scores_row[others]))
    kept = np.concatenate([[i], others[order[:K - 1]]])
    return np.sort(kept)


def select_blocks(q_rot, k_rot, sparsity: float):
    """SubBlock selection of [p3] "6.24 倍里…" in its budget form.

    q_rot, k_rot: post-prologue [B, N, H, d].  Returns
    (kept_idx int64 [B, H, nblk, K], kept_cnt int64 [B, H, nblk], scores).
    """
    q_bar, k_bar = block_pool(q_rot), block_pool(k_rot)
    s = block_scores(q_bar, k_bar)
    B, H, nblk, _ = s.shape
    K = keep_count(nblk, sparsity)
    idx = np.empty((B, H, nblk, K), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for i in range(nblk):
                idx[b, h, i] = select_row(s[b, h, i], i, K)
    return idx, np.full((B, H, nblk), K, dtype=np.int64), s


def select_blocks_threshold(q_rot, k_rot, tau: float):
    """Threshold form of SubBlock ([p4] "事件核心…": blocks scoring below a
    threshold are skipped).  Reading: keep the diagonal block and every
    off-diagonal key block with score >= tau; variable count per row.

    Returns (kept_idx padded with -1 to nblk columns, kept_cnt, scores)."""
    q_bar, k_bar = block_pool(q_rot), block_pool(k_rot)
    s = block_scores(q_bar, k_bar)
    B, H, nblk, _ = s.shape
    idx = np.full((B, H, nblk, nblk), -1, dtype=np.int64)
    cnt = np.zeros((B, H, nblk), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for i in range(nblk):
                row = [j for j in range(nblk) if j == i or s[b, h, i, j] >= tau]
                idx[b, h, i, :len(row)] = row
                cnt[b, h, i] = len(row)
    return idx, cnt, s


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    """Numerically stable softmax in float64."""
    m = np.max(x, axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def attention_block(q, k, v, kept, b, h, i, scale=None) -> np.ndarray:
    """Output rows of query block i of (batch b, head h).

    O_i = softmax(Q_i K_S^T * scale) V_S where S is the union of the tokens of
    the kept key blocks (non-causal; dropped blocks contribute nothing).
    """
    N, d = q.shape[1], q.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    lo, hi = i * BLOCK, min(N, (i + 1) * BLOCK)
    toks = np.concatenate([np.arange(j * BLOCK, min(N, (j + 1) * BLOCK)) for j in kept])
    Qi = np.asarray(q[b, lo:hi, h, :], dtype=np.float64)
    Ks = np.asarray(k[b, toks, h, :], dtype=np.float64)
    Vs = np.asarray(v[b, toks, h, :], dtype=np.float64)
    P = softmax(Qi @ Ks.T * scale, axis=-1)
    return P @ Vs


def block_sparse_attention(q, k, v, kept_idx, kept_cnt, scale=None) -> np.ndarray:
    """Block-sparse attention of every query block over its kept key blocks.
    q, k, v [B, N, H, d]; kept_idx [B, H, nblk, >=cnt]; returns float64 O."""
    B, N, H, d = q.shape
    nblk = -(-N // BLOCK)
    out = np.empty((B, N, H, d))
    for b in range(B):
        for h in range(H):
            for i in range(nblk):
                kept = kept_idx[b, h, i, :kept_cnt[b, h, i]]
                out[b, i * BLOCK:min(N, (i + 1) * BLOCK), h, :] = attention_block(q, k, v, kept, b, h, i, scale)
    return out


def dense_attention(q, k, v, scale=None) -> np.ndarray:
    """Plain softmax attention of every query over every key, per head."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = np.einsum("bnhd,bmhd->bhnm", q, k) * scale
    return np.einsum("bhnm,bmhd->bnhd", softmax(s, axis=-1), v)


# ----------------------------------------------------------------------------
# the fused elementwise steps either side of attention in the DiT block
# ([p3] "先把近两倍的免费收益拿走": the lossless gain includes fused AdaLN and
# SwiGLU kernels).  The page names them only; the readings below are the
# standard DiT definitions:
#
# * AdaLN: LayerNorm of each token's hidden vector without a learned affine
#   (mean and biased variance over the C channels, eps inside the square
#   root), then modulated by the per-sample conditioning vectors shift and
#   scale: y = x_hat * (1 + scale) + shift;
# * SwiGLU: the gated activation between the MLP's two projections,
#   out = silu(gate) * up with silu(a) = a / (1 + exp(-a)), gate and up being
#   the two halves of the first projection's output.


def layer_norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """LayerNorm over the last axis without affine parameters:
    (x - mean) / sqrt(var + eps) with the biased (1/C) variance."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def adaln_modulate(x: np.ndarray, shift: np.ndarray, scale: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """AdaLN of x [B, N, C] with per-sample shift, scale [B, C]:
    layer_norm(x) * (1 + scale) + shift, float64."""
    shift = np.asarray(shift, dtype=np.float64)[:, None, :]
    scale = np.asarray(scale, dtype=np.float64)[:, None, :]
    return layer_norm(x, eps) * (1.0 + scale) + shift


def silu(a: np.ndarray) -> np.ndarray:
    """a * sigmoid(a) = a / (1 + exp(-a)) in float64 (exp(-a) may overflow to
    inf for very negative a, giving the correct limit -0)."""
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def swiglu(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """SwiGLU gating: silu(gate) * up, elementwise, float64."""
    return silu(gate) * np.asarray(up, dtype=np.float64)
