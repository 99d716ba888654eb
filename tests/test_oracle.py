"""Pins of the fp64 oracle against what the definitions and the pages fix.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a float ceil) fails at least one of
them.  CPU only.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import sbattn_oracle as orc
from block_sparse_attention_qk_b200.inputs import WORKLOADS, custom_workload, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def _f64(t):
    return t.to(torch.float64).numpy()


# ---------------------------------------------------------------- budget ----

def test_keep_count_golden():
    rows = _golden_rows("keep_count.txt")
    assert len(rows) >= 10
    for nblk, s, K in rows:
        assert orc.keep_count(int(nblk), float(s)) == int(K), (nblk, s, K)


def test_keep_count_about_a_quarter():
    # "sparsity 0.75 keeps about a quarter of the key blocks"
    for nblk in (4, 17, 252, 1953, 3843):
        K = orc.keep_count(nblk, 0.75)
        assert 0.25 <= K / nblk < 0.25 + 1.0 / nblk + 1e-12


def test_keep_count_exact_not_float_ceil():
    # the float expression gives 124 here; the decimal reading gives 123
    assert math.ceil((1 - 0.18) * 150) == 124
    assert orc.keep_count(150, 0.18) == 123
    # brute force against exact decimal arithmetic on a grid of (s, n)
    from decimal import Decimal
    for s100 in range(0, 101):
        s = s100 / 100
        for n in (1, 3, 64, 150, 999, 1953):
            exact = math.ceil(Decimal(100 - s100) * n / Decimal(100))
            assert orc.keep_count(n, s) == max(1, min(n, exact)), (s, n)


def test_keep_count_rejects_bad_sparsity():
    for bad in (-0.01, 1.01, float("nan"), float("inf")):
        with pytest.raises(ValueError):
            orc.keep_count(10, bad)


def test_sparsity_micro_half_rounding():
    assert orc.sparsity_micro(0.25) == 250000
    assert orc.sparsity_micro(0.0000015) == 2   # 1.5 -> 2 (half away from zero)
    assert orc.sparsity_micro(1.0) == 10**6


# ------------------------------------------------------------- RMSNorm ----

def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(50, 128)) * rng.uniform(0.01, 10, size=(50, 1))
    w = rng.normal(1.0, 0.1, size=128)
    eps = 1e-6
    y = orc.rms_norm(x, w, eps)
    ms = np.mean(x * x, axis=-1)
    got = np.sqrt(np.mean((y / w) ** 2, axis=-1))
    np.testing.assert_allclose(got, np.sqrt(ms / (ms + eps)), rtol=1e-12)
    # the weight multiplies channel by channel
    np.testing.assert_allclose(orc.rms_norm(x, np.ones(128), eps) * w, y, rtol=1e-13)


def test_rmsnorm_eps_inside_sqrt():
    # one tiny row where eps dominates: y = x / sqrt(ms + eps)
    x = np.full((1, 128), 1e-4)
    y = orc.rms_norm(x, np.ones(128), 1e-6)
    np.testing.assert_allclose(y, 1e-4 / math.sqrt(1e-8 + 1e-6), rtol=1e-12)


# ---------------------------------------------------------------- RoPE ----

def test_rope_golden_unit_vectors():
    T, Hh, W = 2, 3, 2
    ang = orc.rope_angles(T, Hh, W)
    rows = _golden_rows("rope_unit_vectors.txt")
    assert len(rows) >= 6
    for t, h, w, cin, ca, va, cb, vb in rows:
        n = (int(t) * Hh + int(h)) * W + int(w)
        y = np.zeros((1, T * Hh * W, 1, 128))
        y[0, n, 0, int(cin)] = 1.0
        out = orc.rope_3d(y, ang)[0, n, 0]
        assert out[int(ca)] == pytest.approx(float(va), abs=1e-15)
        assert out[int(cb)] == pytest.approx(float(vb), abs=1e-15)
        others = np.delete(out, [int(ca), int(cb)])
        assert np.all(others == 0.0)


def test_rope_position_zero_identity_and_norm():
    rng = np.random.default_rng(1)
    T, Hh, W = 3, 4, 5
    y = rng.normal(size=(1, T * Hh * W, 2, 128))
    out = orc.rope_3d(y, orc.rope_angles(T, Hh, W))
    np.testing.assert_array_equal(out[:, 0], y[:, 0])
    # every interleaved pair keeps its length
    np.testing.assert_allclose(np.hypot(out[..., 0::2], out[..., 1::2]),
                               np.hypot(y[..., 0::2], y[..., 1::2]), rtol=1e-12)


def test_rope_relative_offset_invariance():
    # q.k after RoPE depends only on the (dt, dh, dw) offset between the tokens
    rng = np.random.default_rng(2)
    T, Hh, W = 6, 7, 9
    ang = orc.rope_angles(T, Hh, W)
    pos = orc.token_positions(T, Hh, W)
    idx = {tuple(p): n for n, p in enumerate(pos)}
    for _ in range(40):
        q = rng.normal(size=128)
        k = rng.normal(size=128)
        p1 = rng.integers(0, [3, 3, 4])
        p2 = rng.integers(0, [3, 3, 4])
        delta = rng.integers(0, [3, 4, 5])
        dots = []
        for sh in (np.zeros(3, int), delta):
            n1, n2 = idx[tuple(p1 + sh)], idx[tuple(p2 + sh)]
            y = np.zeros((1, T * Hh * W, 1, 128))
            y[0, n1, 0] = q
            qr = orc.rope_3d(y, ang)[0, n1, 0]
            y = np.zeros((1, T * Hh * W, 1, 128))
            y[0, n2, 0] = k
            kr = orc.rope_3d(y, ang)[0, n2, 0]
            dots.append(qr @ kr)
        assert dots[0] == pytest.approx(dots[1], rel=1e-12, abs=1e-12)


def test_rope_single_axis_is_textbook_complex_rotation():
    # positions (0, h, 0): only the h section turns, by the 1D RoPE of size 48,
    # written here as multiplication by a unit complex number
    rng = np.random.default_rng(3)
    T, Hh, W = 1, 11, 1
    y = rng.normal(size=(1, Hh, 1, 128))
    out = orc.rope_3d(y, orc.rope_angles(T, Hh, W))
    for h in range(Hh):
        z = y[0, h, 0, 32:80:2] + 1j * y[0, h, 0, 33:80:2]
        freq = np.array([10000.0 ** (-(2 * m) / 48) for m in range(24)])
        zr = z * np.exp(1j * h * freq)
        np.testing.assert_allclose(out[0, h, 0, 32:80:2], zr.real, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out[0, h, 0, 33:80:2], zr.imag, rtol=1e-12, atol=1e-14)
        np.testing.assert_array_equal(out[0, h, 0, :32], y[0, h, 0, :32])
        np.testing.assert_array_equal(out[0, h, 0, 80:], y[0, h, 0, 80:])


def test_qk_norm_rope_rotation_keeps_row_norm():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl)
    qr, kr = orc.qk_norm_rope(_f64(x["q"]), _f64(x["k"]), _f64(x["w_q"]), _f64(x["w_k"]), wl.T, wl.Hh, wl.W)
    for inp, w, out in ((x["q"], x["w_q"], qr), (x["k"], x["w_k"], kr)):
        normed = orc.rms_norm(_f64(inp), _f64(w))
        np.testing.assert_allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(normed, axis=-1), rtol=1e-12)
        # token 0 sits at the origin of the grid: no rotation at all
        np.testing.assert_allclose(out[:, 0], normed[:, 0], rtol=0, atol=0)


# ------------------------------------------------------ bf16 rounding ----

def test_round_to_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(4)
    x32 = (rng.normal(size=20000) * np.exp(rng.uniform(-20, 20, size=20000))).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.round_to_bf16(x32.astype(np.float64)), ref)


def test_round_to_bf16_ties_to_even():
    v = np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 0.0, 2**-130])
    np.testing.assert_array_equal(orc.round_to_bf16(v)[:4], [1.0, 1 + 2**-6, -1.0, 0.0])


# --------------------------------------------------------- selection ----

def test_pool_and_scores_closed_forms():
    B, N, H, d = 1, 192, 1, 128
    x = np.zeros((B, N, H, d))
    for i in range(3):
        x[0, i * 64:(i + 1) * 64, 0, 0] = np.arange(64) + 100 * i  # mean 31.5 + 100 i
    pooled = orc.block_pool(x)
    np.testing.assert_allclose(pooled[0, 0, :, 0], [31.5, 131.5, 231.5])
    assert np.all(pooled[..., 1:] == 0)
    qb = np.zeros((1, 1, 3, d)); qb[..., 0] = 1.0
    kb = np.zeros((1, 1, 3, d)); kb[0, 0, :, 0] = [5.0, -2.0, 7.0]
    s = orc.block_scores(qb, kb)
    np.testing.assert_array_equal(s[0, 0], [[5, -2, 7]] * 3)
    # a trailing partial block is averaged over its valid tokens
    x2 = np.ones((1, 100, 1, d)); x2[0, 64:] = 3.0
    np.testing.assert_allclose(orc.block_pool(x2)[0, 0, :, 0], [1.0, 3.0])


def _dominance_ok(row, i, kept):
    # every kept off-diagonal block beats every dropped one (ties: lower index)
    off = [j for j in kept if j != i]
    dropped = [j for j in range(len(row)) if j not in kept]
    return all(row[a] > row[b] or (row[a] == row[b] and a < b) for a in off for b in dropped)


def test_select_row_brute_force_enumeration():
    rng = np.random.default_rng(5)
    for trial in range(60):
        nblk = int(rng.integers(1, 8))
        row = rng.integers(-3, 4, size=nblk).astype(np.float64)  # many ties on purpose
        i = int(rng.integers(0, nblk))
        K = int(rng.integers(1, nblk + 1))
        others = [j for j in range(nblk) if j != i]
        winners = [set(c) | {i} for c in itertools.combinations(others, K - 1)
                   if _dominance_ok(row, i, set(c) | {i})]
        assert len(winners) == 1
        got = orc.select_row(row, i, K)
        assert set(got.tolist()) == winners[0]
        assert list(got) == sorted(got)


def test_select_blocks_structure_and_nesting():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl)
    qr, kr = orc.qk_norm_rope(_f64(x["q"]), _f64(x["k"]), _f64(x["w_q"]), _f64(x["w_k"]), wl.T, wl.Hh, wl.W)
    prev = None
    for s in (0.0, 0.25, 0.5, 0.75, 1.0):
        idx, cnt, _ = orc.select_blocks(qr, kr, s)
        K = orc.keep_count(wl.nblk, s)
        assert idx.shape == (wl.B, wl.H, wl.nblk, K)
        assert np.all(cnt == K)
        for b, h, i in itertools.product(range(wl.B), range(wl.H), range(wl.nblk)):
            row = idx[b, h, i]
            assert i in row and len(set(row)) == K and list(row) == sorted(row)
            if prev is not None:  # a higher sparsity keeps a subset
                assert set(row) <= set(prev[b, h, i])
        prev = idx
    idx0, _, _ = orc.select_blocks(qr, kr, 0.0)
    assert np.all(idx0 == np.arange(wl.nblk))
    idx1, _, _ = orc.select_blocks(qr, kr, 1.0)
    assert np.all(idx1[..., 0] == np.arange(wl.nblk)[None, None, :])


def test_select_blocks_tie_break_lower_index():
    d = 128
    q = np.ones((1, 64 * 6, 1, d))
    k = np.ones((1, 64 * 6, 1, d))  # all scores equal
    idx, _, _ = orc.select_blocks(q, k, 0.5)  # K = 3
    for i in range(6):
        expect = sorted({i} | set([j for j in range(6) if j != i][:2]))
        assert list(idx[0, 0, i]) == expect


def test_threshold_selection_matches_budget_at_kth_score():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl)
    qr, kr = orc.qk_norm_rope(_f64(x["q"]), _f64(x["k"]), _f64(x["w_q"]), _f64(x["w_k"]), wl.T, wl.Hh, wl.W)
    idx, cnt, s = orc.select_blocks_threshold(qr, kr, -np.inf)
    assert np.all(cnt == wl.nblk)
    idx, cnt, s = orc.select_blocks_threshold(qr, kr, np.inf)
    assert np.all(cnt == 1) and np.all(idx[..., 0] == np.arange(wl.nblk))
    # with no ties, tau = the (K-1)-th largest off-diagonal score reproduces the budget
    bidx, _, _ = orc.select_blocks(qr, kr, 0.5)
    K = orc.keep_count(wl.nblk, 0.5)
    for h in range(wl.H):
        for i in range(wl.nblk):
            off = np.sort(np.delete(s[0, h, i], i))[::-1]
            tidx, tcnt, _ = orc.select_blocks_threshold(qr[:, :, h:h + 1], kr[:, :, h:h + 1], off[K - 2])
            assert list(tidx[0, 0, i, :tcnt[0, 0, i]]) == list(bidx[0, h, i])


# --------------------------------------------------------- attention ----

def _tiny_rot():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl)
    qr, kr = orc.qk_norm_rope(_f64(x["q"]), _f64(x["k"]), _f64(x["w_q"]), _f64(x["w_k"]), wl.T, wl.Hh, wl.W)
    return wl, qr, kr, _f64(x["v"])


def _sdpa(q, k, v):
    # torch's scaled_dot_product_attention in float64 on the CPU, [B, N, H, d] layout
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))
    return o.permute(0, 2, 1, 3).numpy()


def test_sparsity_zero_equals_dense_and_sdpa():
    wl = custom_workload(B=2, H=3, T=2, Hh=4, W=24, sparsity=0.0, seed=11)  # 192 tokens, 3 blocks
    x = make_inputs(wl)
    q, k, v = _f64(x["q"]), _f64(x["k"]), _f64(x["v"])
    idx, cnt, _ = orc.select_blocks(q, k, 0.0)
    out = orc.block_sparse_attention(q, k, v, idx, cnt)
    np.testing.assert_allclose(out, orc.dense_attention(q, k, v), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out, _sdpa(q, k, v), rtol=1e-10, atol=1e-12)


def test_single_kept_block_is_local_attention():
    wl, q, k, v = _tiny_rot()
    idx, cnt, _ = orc.select_blocks(q, k, 1.0)  # K = 1: the diagonal only
    out = orc.block_sparse_attention(q, k, v, idx, cnt)
    for i in range(wl.nblk):
        sl = slice(i * 64, (i + 1) * 64)
        np.testing.assert_allclose(out[:, sl], _sdpa(q[:, sl], k[:, sl], v[:, sl]), rtol=1e-10, atol=1e-12)


def test_rows_are_convex_combinations():
    wl, q, k, _ = _tiny_rot()
    idx, cnt, _ = orc.select_blocks(q, k, 0.5)  # K = 2 -> 128 keys per query
    # constant V: every output equals the constant
    c = np.linspace(-1, 1, 128)
    v = np.broadcast_to(c, q.shape).copy()
    np.testing.assert_allclose(orc.block_sparse_attention(q, k, v, idx, cnt), v, rtol=1e-12)
    # one-hot V over the 128 kept keys: the output row IS the softmax row
    for h in range(wl.H):
        for i in range(wl.nblk):
            kept = idx[0, h, i]
            toks = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in kept])
            vv = np.zeros_like(q)
            vv[0, toks, h, np.arange(128)] = 1.0
            P = orc.attention_block(q, k, vv, kept, 0, h, i)
            assert np.all(P >= 0)
            np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=1e-13)


def test_kept_order_and_dropped_blocks_do_not_matter():
    wl, q, k, v = _tiny_rot()
    idx, cnt, _ = orc.select_blocks(q, k, 0.5)
    base = orc.block_sparse_attention(q, k, v, idx, cnt)
    perm = idx[..., ::-1].copy()
    np.testing.assert_allclose(orc.block_sparse_attention(q, k, v, perm, cnt), base, rtol=1e-13, atol=1e-15)
    # scribbling on a dropped key block leaves query block 0 of head 0 alone,
    # scribbling on a kept one does not
    kept0 = set(idx[0, 0, 0].tolist())
    dropped = [j for j in range(wl.nblk) if j not in kept0][0]
    kept_off = [j for j in kept0 if j != 0][0]
    for j, changes in ((dropped, False), (kept_off, True)):
        k2, v2 = k.copy(), v.copy()
        k2[0, j * 64:(j + 1) * 64, 0] += 3.0
        v2[0, j * 64:(j + 1) * 64, 0] -= 5.0
        o2 = orc.attention_block(q, k2, v2, idx[0, 0, 0], 0, 0, 0)
        assert (not np.allclose(o2, base[0, 0:64, 0])) == changes


def test_explicit_scale_matches_default():
    wl, q, k, v = _tiny_rot()
    idx, cnt, _ = orc.select_blocks(q, k, 0.5)
    a = orc.block_sparse_attention(q, k, v, idx, cnt)
    b = orc.block_sparse_attention(q, k, v, idx, cnt, scale=1 / math.sqrt(128))
    np.testing.assert_array_equal(a, b)
    c = orc.block_sparse_attention(q, k, v, idx, cnt, scale=0.5)
    assert not np.allclose(a, c)


# ---------------------------------------------------------------- AdaLN / SwiGLU

def test_layer_norm_hand_example():
    # x = (1, 2, 3, 4): mean 5/2, biased variance 5/4, eps 0
    y = orc.layer_norm(np.array([1.0, 2.0, 3.0, 4.0]), eps=0.0)
    s = math.sqrt(1.25)
    np.testing.assert_allclose(y, [-1.5 / s, -0.5 / s, 0.5 / s, 1.5 / s], rtol=0, atol=1e-15)


def test_layer_norm_moments_closed_form():
    # rows of y have mean 0 and variance var / (var + eps) exactly: catches a
    # dropped mean, an unbiased variance or eps outside the square root
    rng = np.random.default_rng(11)
    x = rng.normal(2.0, 0.01, size=(3, 5, 64))
    eps = 1e-4
    y = orc.layer_norm(x, eps)
    var = x.var(axis=-1)
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(axis=-1), var / (var + eps), rtol=1e-12)


def test_layer_norm_is_affine_invariant():
    rng = np.random.default_rng(12)
    x = rng.normal(size=(2, 3, 48))
    np.testing.assert_allclose(orc.layer_norm(3.5 * x - 7.0, 0.0), orc.layer_norm(x, 0.0), atol=1e-12)


def test_adaln_modulation_special_cases():
    rng = np.random.default_rng(13)
    x = rng.normal(size=(2, 4, 32))
    shift = rng.normal(size=(2, 32))
    zero = np.zeros((2, 32))
    # scale = shift = 0 -> plain LayerNorm; scale = -1 -> shift regardless of x
    np.testing.assert_allclose(orc.adaln_modulate(x, zero, zero), orc.layer_norm(x), atol=1e-15)
    np.testing.assert_allclose(orc.adaln_modulate(x, shift, -np.ones((2, 32))),
                               np.broadcast_to(shift[:, None, :], x.shape), atol=1e-15)
    # constant rows normalise to 0 -> shift
    c = np.full((2, 4, 32), 3.25)
    np.testing.assert_allclose(orc.adaln_modulate(c, shift, rng.normal(size=(2, 32))),
                               np.broadcast_to(shift[:, None, :], c.shape), atol=1e-15)
    # (1 + scale), per sample: doubling the normalised row needs scale = 1
    np.testing.assert_allclose(orc.adaln_modulate(x, zero, np.ones((2, 32))), 2 * orc.layer_norm(x), atol=1e-14)
    # sample b uses its own vectors
    s2 = np.stack([np.zeros(32), np.full(32, 5.0)])
    y = orc.adaln_modulate(x, s2, zero)
    np.testing.assert_allclose(y[1] - y[0], 5.0 + orc.layer_norm(x)[1] - orc.layer_norm(x)[0], atol=1e-13)


def test_silu_values_and_identity():
    assert orc.silu(np.array(0.0)) == 0.0
    np.testing.assert_allclose(orc.silu(np.array([1.0, -1.0])), [1 / (1 + math.exp(-1)), -1 / (1 + math.e)], rtol=1e-15)
    a = np.linspace(-30, 30, 121)
    # silu(a) - silu(-a) = a (a * (sigmoid(a) + sigmoid(-a)))
    np.testing.assert_allclose(orc.silu(a) - orc.silu(-a), a, atol=1e-13)
    big = orc.silu(np.array([-1000.0, 1000.0]))
    assert big[0] == 0.0 and big[1] == 1000.0
    # silu against torch's SiLU on the same fp64 values
    np.testing.assert_allclose(orc.silu(a), torch.nn.functional.silu(torch.from_numpy(a)).numpy(), rtol=1e-14, atol=1e-300)


def test_swiglu_gates_up():
    rng = np.random.default_rng(14)
    g = rng.normal(size=(5, 16))
    u = rng.normal(size=(5, 16))
    np.testing.assert_allclose(orc.swiglu(g, np.ones_like(g)), orc.silu(g), atol=0)
    np.testing.assert_allclose(orc.swiglu(g, 2 * u), 2 * orc.swiglu(g, u), rtol=1e-15)
    assert not np.allclose(orc.swiglu(g, u), orc.swiglu(u, g))  # gate and up are not interchangeable
