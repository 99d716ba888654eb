"""GPU tests of the selection kernel's paths, on pooled block means.

The kernel places a histogram window from a sample of each score row, keeps
the few blocks of the boundary bin in shared memory and cuts among them; when
a bin holds too many blocks it falls back to radix levels on the score and
then on the block index.  Each path is driven here by inputs built for it and
compared with the oracle's selection on the same pooled means:

  * sample far from the bulk: every sampled key block scores far above the
    rest, so the window misses the boundary (fallback on score bytes);
  * mass ties: all scores equal, so the boundary is decided by block index
    alone (fallback on index bytes);
  * twin blocks: every score appears twice, so the boundary bin holds exact
    ties that the cut resolves by block index (fast path);
  * several tiles per row in threshold mode, where the second selector
    warpgroup's blocks are moved behind the first's, and the trivial budgets;
  * long rows: up to 16 tiles compaction and output share one pass, beyond
    that they are two passes, and beyond 4096 blocks the rows are written
    without the shared bitmask.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_qk_b200 as sb
from oracle import sbattn_oracle as orc

from .parity import check_kept_structure, check_selection

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _oracle_budget(q_bar, k_bar, sparsity):
    s = orc.block_scores(q_bar, k_bar)
    B, H, nblk, _ = s.shape
    K = orc.keep_count(nblk, sparsity)
    idx = np.empty((B, H, nblk, K), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for i in range(nblk):
                idx[b, h, i] = orc.select_row(s[b, h, i], i, K)
    return idx, s, K


def _run_budget(q_bar, k_bar, sparsity):
    qd = torch.from_numpy(q_bar.astype(np.float32)).to(DEV)
    kd = torch.from_numpy(k_bar.astype(np.float32)).to(DEV)
    idx, cnt, scores = sb.select_blocks_pooled(qd, kd, sparsity, return_scores=True)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy(), scores.cpu().numpy()


def _check_budget(q_bar, k_bar, sparsity):
    ref_idx, ref_s, K = _oracle_budget(q_bar, k_bar, sparsity)
    gidx, gcnt, gs = _run_budget(q_bar, k_bar, sparsity)
    nblk = q_bar.shape[2]
    check_kept_structure(gidx, gcnt, nblk, K)
    return check_selection(gidx, gcnt, ref_idx, ref_s, q_bar, k_bar), gidx, ref_idx


def test_sample_far_from_the_bulk_falls_back_to_radix_levels():
    rng = np.random.default_rng(51)
    B, H, nblk, d = 1, 2, 1000, 128          # 8 tiles; every 8th block is sampled
    u = rng.normal(size=(B, H, 1, d))
    q_bar = 3.0 * u + rng.normal(size=(B, H, nblk, d))
    k_bar = rng.normal(size=(B, H, nblk, d))
    k_bar[:, :, ::8] += 3.0 * u               # the sampled blocks score ~9 |u|^2 higher
    q_bar, k_bar = q_bar.astype(np.float32).astype(np.float64), k_bar.astype(np.float32).astype(np.float64)
    stats, gidx, ref_idx = _check_budget(q_bar, k_bar, 0.75)
    assert stats["decision_agreement"] > 0.9999


def test_mass_ties_are_cut_by_block_index():
    B, H, nblk, d = 1, 2, 300, 128           # 3 tiles per row, 2 rows of items
    q_bar = np.ones((B, H, nblk, d))
    k_bar = np.full((B, H, nblk, d), 0.5)
    gidx, gcnt, gs = _run_budget(q_bar, k_bar, 0.6)
    K = orc.keep_count(nblk, 0.6)
    assert np.all(gs == 64.0)
    for i in (0, 1, 119, 120, 121, 150, 299):
        expect = sorted({i} | set([j for j in range(nblk) if j != i][:K - 1]))
        assert gidx[0, 0, i].tolist() == expect and gidx[0, 1, i].tolist() == expect
    assert np.all(gcnt == K)


def test_twin_blocks_tie_at_the_boundary_and_go_to_the_lower_index():
    rng = np.random.default_rng(52)
    B, H, nblk, d = 1, 3, 400, 128
    q_bar = rng.normal(size=(B, H, nblk, d)).astype(np.float32).astype(np.float64)
    k_bar = rng.normal(size=(B, H, nblk, d)).astype(np.float32).astype(np.float64)
    k_bar[:, :, 1::2] = k_bar[:, :, 0::2]     # block 2m+1 repeats block 2m: every score has a twin
    stats, gidx, ref_idx = _check_budget(q_bar, k_bar, 0.75)
    # twins are bit-identical on both sides, so a boundary between twins is no
    # near tie: only the lower of the two may be kept alone
    s = orc.block_scores(q_bar, k_bar)
    for h in range(H):
        for i in range(0, nblk, 7):
            kept = set(gidx[0, h, i].tolist()) - {i}
            for j in kept:
                twin = j ^ 1
                if twin != i and twin not in kept and s[0, h, i, twin] == s[0, h, i, j]:
                    assert j < twin, (h, i, j)


@pytest.mark.parametrize("nblk", [300, 513])
def test_threshold_over_several_tiles(nblk):
    rng = np.random.default_rng(53 + nblk)
    B, H, d = 1, 2, 128
    q_bar = rng.normal(size=(B, H, nblk, d)).astype(np.float32).astype(np.float64)
    k_bar = rng.normal(size=(B, H, nblk, d)).astype(np.float32).astype(np.float64)
    s = orc.block_scores(q_bar, k_bar)
    tau = float(np.median(s))
    qd = torch.from_numpy(q_bar.astype(np.float32)).to(DEV)
    kd = torch.from_numpy(k_bar.astype(np.float32)).to(DEV)
    idx, cnt = sb.select_blocks_threshold(qd, kd, tau)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    scale = np.linalg.norm(q_bar, axis=-1)[..., None] * np.max(np.linalg.norm(k_bar, axis=-1), axis=-1)[..., None, None]
    for h in range(H):
        for i in range(nblk):
            row = gidx[0, h, i]
            c = int(gcnt[0, h, i])
            assert np.all(row[c:] == -1)
            got = row[:c]
            assert np.all(np.diff(got) > 0), "ascending"
            ref = set(j for j in range(nblk) if j == i or s[0, h, i, j] >= tau)
            for j in set(got.tolist()) ^ ref:
                assert abs(s[0, h, i, j] - tau) <= 1e-5 * scale[0, h, i, 0], (h, i, j)


def test_trivial_budgets_over_several_tiles():
    rng = np.random.default_rng(54)
    B, H, nblk, d = 1, 2, 300, 128
    q_bar = rng.normal(size=(B, H, nblk, d)).astype(np.float32)
    k_bar = rng.normal(size=(B, H, nblk, d)).astype(np.float32)
    qd, kd = torch.from_numpy(q_bar).to(DEV), torch.from_numpy(k_bar).to(DEV)
    idx, cnt = sb.select_blocks_pooled(qd, kd, 0.0)
    assert torch.all(cnt == nblk)
    assert torch.equal(idx.cpu(), torch.arange(nblk, dtype=torch.int32).expand(B, H, nblk, nblk))
    idx, cnt = sb.select_blocks_pooled(qd, kd, 1.0, capacity=4)
    assert torch.all(cnt == 1)
    assert torch.equal(idx[..., 0].cpu(), torch.arange(nblk, dtype=torch.int32).expand(B, H, nblk))
    assert torch.all(idx[..., 1:] == -1)


@pytest.mark.parametrize("nblk", [2100, 4200])
def test_long_rows_take_the_two_pass_and_direct_output_forms(nblk):
    """Rows of more than 16 tiles run compaction and output as two passes
    (2100 blocks: 17 tiles, the kept blocks still gathered in the bitmask);
    beyond 4096 blocks the bitmask does not fit and each warpgroup writes its
    tiles' blocks itself (4200 blocks)."""
    rng = np.random.default_rng(55 + nblk)
    B, H, d = 1, 1, 128
    u = rng.normal(size=(B, H, nblk, d))
    q_bar = (rng.normal(size=(B, H, nblk, d)) + 0.5 * u).astype(np.float32).astype(np.float64)
    k_bar = (rng.normal(size=(B, H, nblk, d)) + 0.5 * u).astype(np.float32).astype(np.float64)
    stats, gidx, ref_idx = _check_budget(q_bar, k_bar, 0.75)
    assert stats["decision_agreement"] > 0.9999
