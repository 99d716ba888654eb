"""GPU parity of each stage through the C ABI, stage by stage.

Every stage is fed inputs that come from the seeded generator or from the
oracle (never from another CUDA stage) and is compared with the oracle on
those same inputs:
  prologue   raw Q, K, weights             -> vs oracle fp64 prologue
  selection  oracle prologue rounded to bf16 -> vs oracle selection
  attention  oracle prologue (bf16), V, oracle kept lists -> vs oracle attention
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_qk_b200 as sb
from block_sparse_attention_qk_b200.inputs import WORKLOADS, custom_workload, make_inputs
from oracle import sbattn_oracle as orc

from .parity import (check_attention, check_kept_structure, check_prologue, check_selection, f64, oracle_prologue,
                     to_bf16_tensor)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

# grids spanning several tiles and a ragged tail (N % 64 != 0)
CASES = {
    "tiny": WORKLOADS["tiny"],
    "dense": WORKLOADS["dense"],
    "dense_s075": WORKLOADS["dense"].with_sparsity(0.75),
    # K = 61: an odd number of tiles per item, ~14 items per CTA
    "dense_odd": WORKLOADS["dense"].with_sparsity(0.76),
    "ragged": custom_workload("ragged", B=2, H=3, T=3, Hh=7, W=13, sparsity=0.6, seed=21),  # N = 273
    "odd_keep": custom_workload("odd_keep", B=1, H=4, T=2, Hh=16, W=30, sparsity=0.5, seed=22),  # nblk 15, K 8
    "one_block": custom_workload("one_block", B=1, H=2, T=1, Hh=5, W=7, sparsity=0.5, seed=23),  # N = 35
}


# heads compared element by element (the kernels always run every head); the
# dense check's fp64 attention is costly, so two of its eight heads are used
HEADS = {"dense": (0, 5), "dense_s075": (1, 6), "dense_odd": (2, 7)}

_ORACLE_ATTN = {}


def oracle_attention(name, wl, qr16, kr16, v, idx, cnt, sparsity, scale=None):
    """Oracle attention of the compared heads (NaN elsewhere), cached per case."""
    key = (name, sparsity, scale)
    if key not in _ORACLE_ATTN:
        heads = HEADS.get(name, tuple(range(wl.H)))
        ref = np.full(qr16.shape, np.nan)
        for h in heads:
            sl = slice(h, h + 1)
            ref[:, :, sl] = orc.block_sparse_attention(qr16[:, :, sl], kr16[:, :, sl], v[:, :, sl], idx[:, sl],
                                                       cnt[:, sl], scale)
        _ORACLE_ATTN[key] = ref
    return _ORACLE_ATTN[key]


def compared(got, ref):
    m = ~np.isnan(ref[0, 0, :, 0])
    return got[:, :, m], ref[:, :, m]


@pytest.fixture(scope="module")
def data():
    torch.cuda.init()
    cache = {}

    def get(name):
        if name not in cache:
            wl = CASES[name]
            x = make_inputs(wl)  # CPU draw; copied to the device below
            qr, kr, qr16, kr16 = oracle_prologue(x, wl)
            cache[name] = (wl, x, qr, kr, qr16, kr16)
        return cache[name]

    return get


def _dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


# ------------------------------------------------------------------ prologue

@pytest.mark.parametrize("name", list(CASES))
def test_prologue_matches_oracle(data, name):
    wl, x, qr, kr, _, _ = data(name)
    d = _dev(x)
    q_rot, k_rot, q_bar, k_bar = sb.qk_norm_rope(d["q"], d["k"], d["w_q"], d["w_k"], (wl.T, wl.Hh, wl.W), pool=True)
    torch.cuda.synchronize()
    check_prologue(f64(q_rot), qr, "q")
    check_prologue(f64(k_rot), kr, "k")
    # fused block means: the mean of the stored outputs, within the prologue
    # tolerance averaged over the block
    for gbar, ref in ((q_bar, qr), (k_bar, kr)):
        refbar = orc.block_pool(ref)
        bound = orc.block_pool(4e-3 * np.maximum(1.0, np.abs(ref)))
        assert np.all(np.abs(f64(gbar) - refbar) <= bound)


def test_prologue_in_place_and_pool_agrees_with_separate_pass(data):
    wl, x, qr, _, _, _ = data("ragged")
    d = _dev(x)
    q_sep, k_sep = sb.qk_norm_rope(d["q"], d["k"], d["w_q"], d["w_k"], (wl.T, wl.Hh, wl.W))
    q_in, k_in = d["q"].clone(), d["k"].clone()
    sb.qk_norm_rope(q_in, k_in, d["w_q"], d["w_k"], (wl.T, wl.Hh, wl.W), q_out=q_in, k_out=k_in)
    torch.cuda.synchronize()
    assert torch.equal(q_in, q_sep) and torch.equal(k_in, k_sep)
    # fused pooling equals the pooling pass of sbattn_select_blocks (same sum order)
    _, _, q_bar, k_bar = sb.qk_norm_rope(d["q"], d["k"], d["w_q"], d["w_k"], (wl.T, wl.Hh, wl.W), pool=True)
    i1, c1, s1 = sb.select_blocks(q_sep, k_sep, 0.6, return_scores=True)
    i2, c2, s2 = sb.select_blocks_pooled(q_bar, k_bar, 0.6, return_scores=True)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2) and torch.equal(i1, i2) and torch.equal(c1, c2)


# ----------------------------------------------------------------- selection

@pytest.mark.parametrize("name", list(CASES))
def test_selection_matches_oracle(data, name):
    wl, x, _, _, qr16, kr16 = data(name)
    q_rot, k_rot = to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV)
    idx, cnt, scores = sb.select_blocks(q_rot, k_rot, wl.sparsity, return_scores=True)
    torch.cuda.synchronize()
    ref_idx, ref_cnt, ref_scores = orc.select_blocks(qr16, kr16, wl.sparsity)
    K = orc.keep_count(wl.nblk, wl.sparsity)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    check_kept_structure(gidx, gcnt, wl.nblk, K)
    q_bar, k_bar = orc.block_pool(qr16), orc.block_pool(kr16)
    cs = np.linalg.norm(q_bar, axis=-1)[..., None] * np.max(np.linalg.norm(k_bar, axis=-1), axis=-1)[..., None, None]
    assert np.all(np.abs(f64(scores) - ref_scores) <= 1e-5 * cs), "scores off"
    check_selection(gidx, gcnt, ref_idx, ref_scores, q_bar, k_bar)


def test_selection_ties_go_to_lower_index():
    # identical blocks: every score ties; the kept list is the diagonal plus
    # the lowest other indices
    wl = custom_workload("ties", B=1, H=2, T=1, Hh=6, W=64, sparsity=0.5)  # nblk 6, K 3
    q = torch.ones((1, wl.N, 2, 128), dtype=torch.bfloat16, device=DEV)
    idx, cnt = sb.select_blocks(q, q.clone(), 0.5)
    for i in range(6):
        expect = sorted({i} | set([j for j in range(6) if j != i][:2]))
        assert idx[0, 0, i].tolist() == expect and idx[0, 1, i].tolist() == expect


def test_selection_extremes_and_capacity_padding(data):
    wl, x, _, _, qr16, kr16 = data("odd_keep")
    q_rot, k_rot = to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV)
    idx, cnt = sb.select_blocks(q_rot, k_rot, 0.0)
    assert torch.equal(idx[0, 0].cpu(), torch.arange(wl.nblk, dtype=torch.int32).repeat(wl.nblk, 1))
    idx, cnt = sb.select_blocks(q_rot, k_rot, 1.0, capacity=5)
    assert torch.all(cnt == 1)
    assert torch.equal(idx[..., 0].cpu(), torch.arange(wl.nblk, dtype=torch.int32).expand(1, wl.H, wl.nblk))
    assert torch.all(idx[..., 1:] == -1)


def test_threshold_selection_matches_oracle(data):
    wl, x, _, _, qr16, kr16 = data("odd_keep")
    q_bar = torch.from_numpy(orc.block_pool(qr16)).float().to(DEV)
    k_bar = torch.from_numpy(orc.block_pool(kr16)).float().to(DEV)
    _, _, ref_scores = orc.select_blocks(qr16, kr16, 0.5)
    tau = float(np.median(ref_scores))
    idx, cnt, scores = sb.select_blocks_threshold(q_bar, k_bar, tau, return_scores=True)
    torch.cuda.synchronize()
    gs = f64(scores)
    for h in range(wl.H):
        for i in range(wl.nblk):
            c = int(cnt[0, h, i])
            got = idx[0, h, i, :c].tolist()
            # decided on the GPU's own fp32 scores (the rule is a comparison)
            expect = [j for j in range(wl.nblk) if j == i or gs[0, h, i, j] >= np.float32(tau)]
            assert got == expect
            assert torch.all(idx[0, h, i, c:] == -1)
    # and the GPU scores are the oracle's (same bound as the budget path)
    qb, kb = orc.block_pool(qr16), orc.block_pool(kr16)
    cs = np.linalg.norm(qb, axis=-1)[..., None] * np.max(np.linalg.norm(kb, axis=-1), axis=-1)[..., None, None]
    assert np.all(np.abs(gs - ref_scores) <= 1e-5 * cs), "threshold-path scores off"
    ref_idx, ref_cnt, _ = orc.select_blocks_threshold(qr16, kr16, tau)
    rows_same = np.mean([set(idx[0, h, i, :cnt[0, h, i]].tolist()) == set(ref_idx[0, h, i, :ref_cnt[0, h, i]].tolist())
                         for h in range(wl.H) for i in range(wl.nblk)])
    assert rows_same >= 0.99


# ----------------------------------------------------------------- attention

def _attn_case(data, name, sparsity=None, permute=False, seed=0):
    wl, x, _, _, qr16, kr16 = data(name)
    s = wl.sparsity if sparsity is None else sparsity
    ref_idx, ref_cnt, _ = orc.select_blocks(qr16, kr16, s)
    idx = ref_idx.copy()
    if permute:  # any order of the kept list is allowed
        rng = np.random.default_rng(seed)
        for row in idx.reshape(-1, idx.shape[-1]):
            rng.shuffle(row)
    q_rot, k_rot = to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV)
    v = x["v"].to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = sb.forward(q_rot, k_rot, v, torch.from_numpy(idx).int().to(DEV), torch.from_numpy(ref_cnt).int().to(DEV),
                     status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle_attention(name, wl, qr16, kr16, f64(x["v"]), ref_idx, ref_cnt, s)
    got, ref = compared(f64(out), ref)
    return got, ref, wl, (qr16, kr16, f64(x["v"]))


@pytest.mark.parametrize("name", list(CASES))
def test_attention_matches_oracle(data, name):
    got, ref, _, _ = _attn_case(data, name)
    check_attention(got, ref)


def test_attention_dense_equals_dense_softmax(data):
    got, _, wl, (q, k, v) = _attn_case(data, "dense", sparsity=0.0)
    h = HEADS["dense"]
    check_attention(got, orc.dense_attention(q[:, :, h], k[:, :, h], v[:, :, h]))


@pytest.mark.parametrize("name", ["dense_s075", "ragged", "odd_keep"])
def test_attention_kept_order_does_not_matter(data, name):
    got, ref, _, _ = _attn_case(data, name, permute=True, seed=5)
    check_attention(got, ref)


@pytest.mark.parametrize("s", [1.0, 0.9, 0.5, 0.0])
def test_attention_budget_sweep(data, s):
    got, ref, _, _ = _attn_case(data, "odd_keep", sparsity=s)
    check_attention(got, ref)


def test_attention_rescale_path():
    # a later kept block whose logits exceed the first tile's maximum by far
    # more than 2^8 forces the running-maximum rescale of O and the row sums
    rng = np.random.default_rng(7)
    B, H, nblk, d = 1, 2, 6, 128
    N = nblk * 64
    q = rng.normal(size=(B, N, H, d))
    k = rng.normal(size=(B, N, H, d)) * 0.3
    v = rng.normal(size=(B, N, H, d))
    # key n of block 4 is twice query n of block 0: logit about 2*128/sqrt(128)
    # = 22.6 against about 1 in the first tile of query block 0
    k[:, 4 * 64:5 * 64] = 2.0 * q[:, 0:64]
    q, k, v = orc.round_to_bf16(q), orc.round_to_bf16(k), orc.round_to_bf16(v)
    idx = np.array([[[[i, (i + 1) % nblk, (i + 2) % nblk, 4] if i not in (2, 3, 4) else [i, 0, 1, 5]
                      for i in range(nblk)]] * H]).reshape(B, H, nblk, 4)
    cnt = np.full((B, H, nblk), 4)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = sb.forward(to_bf16_tensor(q, DEV), to_bf16_tensor(k, DEV), to_bf16_tensor(v, DEV),
                     torch.from_numpy(idx).int().to(DEV), torch.from_numpy(cnt).int().to(DEV), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = orc.block_sparse_attention(q, k, v, idx, cnt)
    # the logits here span a wide range: the softmax of query block 0 is
    # dominated by block 4, as it must be
    check_attention(f64(out), ref)


def test_attention_explicit_scale(data):
    wl, x, _, _, qr16, kr16 = data("tiny")
    ref_idx, ref_cnt, _ = orc.select_blocks(qr16, kr16, 0.5)
    out = sb.forward(to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV), x["v"].to(DEV),
                     torch.from_numpy(ref_idx).int().to(DEV), torch.from_numpy(ref_cnt).int().to(DEV), scale=0.03)
    torch.cuda.synchronize()
    check_attention(f64(out), oracle_attention("tiny", wl, qr16, kr16, f64(x["v"]), ref_idx, ref_cnt, 0.5, 0.03))


def test_attention_bad_indices_are_reported_and_masked(data):
    wl, x, _, _, qr16, kr16 = data("odd_keep")
    ref_idx, ref_cnt, _ = orc.select_blocks(qr16, kr16, 0.5)
    idx = ref_idx.copy()
    cnt = ref_cnt.copy()
    idx[0, 1, 3, -1] = wl.nblk + 7     # out of range: skipped, reported
    cnt[0, 2, 5] = 0                   # empty row: zeros, reported
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = sb.forward(to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV), x["v"].to(DEV),
                     torch.from_numpy(idx).int().to(DEV), torch.from_numpy(cnt).int().to(DEV), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6  # SBATTN_ERR_DEVICE
    got = f64(out)
    ref = orc.block_sparse_attention(qr16, kr16, f64(x["v"]), ref_idx, ref_cnt)
    ref_bad = orc.attention_block(qr16, kr16, f64(x["v"]), ref_idx[0, 1, 3, :-1], 0, 1, 3)
    ref[0, 3 * 64:4 * 64, 1] = ref_bad
    ref[0, 5 * 64:6 * 64, 2] = 0.0
    check_attention(got, ref)
