"""GPU tests of the attention kernel's edges, through the C ABI:

  * failure detection: a bounded wait inside the kernel runs out (one V copy
    is withheld), the kernel reports SBATTN_ERR_TIMEOUT in the caller's
    status word and returns, and the next normal call on the same device
    matches the oracle;
  * threshold selection feeding attention: kept lists of varying length
    (from 1 block to every block, padded with -1) are attended correctly;
  * logit range: with a large explicit softmax scale a later kept block
    exceeds the first tile's maximum by hundreds of log2 units, and the
    result is still the exact softmax.
"""

import ctypes
import time

import numpy as np
import pytest
import torch

import block_sparse_attention_qk_b200 as sb
from block_sparse_attention_qk_b200._lib import lib
from block_sparse_attention_qk_b200.inputs import custom_workload, make_inputs
from oracle import sbattn_oracle as orc

from .parity import check_attention, f64, oracle_prologue, to_bf16_tensor

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ERR_TIMEOUT = 7


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def case():
    torch.cuda.init()
    wl = custom_workload("edges", B=1, H=4, T=2, Hh=16, W=30, sparsity=0.5, seed=41)  # nblk 15, K 8: 4 tiles/item
    x = make_inputs(wl)
    _, _, qr16, kr16 = oracle_prologue(x, wl)
    return wl, x, qr16, kr16


def test_bounded_wait_runs_out_and_the_device_stays_usable(case):
    wl, x, qr16, kr16 = case
    idx, cnt, _ = orc.select_blocks(qr16, kr16, wl.sparsity)
    q, k, v = to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV), x["v"].to(DEV)
    kidx, kcnt = torch.from_numpy(idx).int().to(DEV), torch.from_numpy(cnt).int().to(DEV)
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    B, N, H, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    limit_ns = 50_000_000  # 50 ms
    t0 = time.perf_counter()
    # every CTA skips the copy of its second V tile: the PV issuer's wait for
    # it must run out, and every other role must then leave its waits
    rc = lib().sbattn_forward_diag(_p(q), _p(k), _p(v), _p(kidx), _p(kcnt), idx.shape[-1], _p(out), B, N, H, d,
                                   0.0, _p(status), limit_ns, 1, stream)
    assert rc == 0
    code = lib().sbattn_check_status(_p(status), stream)  # synchronises
    elapsed = time.perf_counter() - t0
    assert code == ERR_TIMEOUT
    assert int(status.item()) == ERR_TIMEOUT
    assert elapsed < 10.0
    # the same device, the same inputs, a normal call: correct results
    status.zero_()
    out2 = sb.forward(q, k, v, kidx, kcnt, status=status)
    sb.check_status(status)
    ref = orc.block_sparse_attention(qr16, kr16, f64(x["v"]), idx, cnt)
    check_attention(f64(out2), ref)


def test_diagnostic_call_without_withheld_tile_is_a_normal_call(case):
    wl, x, qr16, kr16 = case
    idx, cnt, _ = orc.select_blocks(qr16, kr16, wl.sparsity)
    q, k, v = to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV), x["v"].to(DEV)
    kidx, kcnt = torch.from_numpy(idx).int().to(DEV), torch.from_numpy(cnt).int().to(DEV)
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    B, N, H, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib().sbattn_forward_diag(_p(q), _p(k), _p(v), _p(kidx), _p(kcnt), idx.shape[-1], _p(out), B, N, H, d,
                                   0.0, _p(status), 1_000_000_000, -1, stream)
    assert rc == 0
    assert lib().sbattn_check_status(_p(status), stream) == 0
    check_attention(f64(out), orc.block_sparse_attention(qr16, kr16, f64(x["v"]), idx, cnt))


@pytest.mark.parametrize("where", ["median", "all", "diagonal_only"])
def test_threshold_selection_feeds_attention(case, where):
    """The threshold form's kept lists (count varying per row, capacity nblk,
    -1 padding) go straight into the attention call and are attended
    exactly: the oracle runs on the GPU's own kept lists."""
    wl, x, qr16, kr16 = case
    q_bar = torch.from_numpy(orc.block_pool(qr16)).float().to(DEV)
    k_bar = torch.from_numpy(orc.block_pool(kr16)).float().to(DEV)
    _, _, ref_scores = orc.select_blocks(qr16, kr16, 0.5)
    tau = {"median": float(np.median(ref_scores)), "all": -1e30, "diagonal_only": 1e30}[where]
    idx, cnt = sb.select_blocks_threshold(q_bar, k_bar, tau)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = sb.forward(to_bf16_tensor(qr16, DEV), to_bf16_tensor(kr16, DEV), x["v"].to(DEV), idx, cnt, status=status)
    sb.check_status(status)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert gidx.shape[-1] == wl.nblk
    if where == "all":
        assert np.all(gcnt == wl.nblk)
    elif where == "diagonal_only":
        assert np.all(gcnt == 1)
    else:
        assert gcnt.min() < gcnt.max()  # ragged counts
    ref = orc.block_sparse_attention(qr16, kr16, f64(x["v"]), gidx, gcnt)
    check_attention(f64(out), ref)


@pytest.mark.parametrize("scale", [0.5, 2.0])
def test_logits_far_above_the_first_tile_are_exact(scale):
    """Key block 4 repeats twice the queries of block 0, so for query block 0
    its logits exceed those of the first tile by about 2 * 128 * scale in
    natural units (185 and 740 log2 units here): far beyond 2^8, and, for the
    larger scale, far beyond the float range of 2^x.  The running maximum must
    be raised before those weights are formed."""
    rng = np.random.default_rng(8)
    B, H, nblk, d = 1, 2, 6, 128
    N = nblk * 64
    q = rng.normal(size=(B, N, H, d))
    k = rng.normal(size=(B, N, H, d)) * 0.3
    v = rng.normal(size=(B, N, H, d))
    k[:, 4 * 64:5 * 64] = 2.0 * q[:, 0:64]
    q, k, v = orc.round_to_bf16(q), orc.round_to_bf16(k), orc.round_to_bf16(v)
    # query block 0 sees blocks 0, 1 (first tile), then 2, 3, 4, 5: block 4 in the second step
    idx = np.array([[[[0, 1, 2, 3, 4, 5]] + [[i] + [j for j in range(nblk) if j != i][:5] for i in range(1, nblk)]] * H])
    idx = np.sort(idx.reshape(B, H, nblk, 6), axis=-1)
    cnt = np.full((B, H, nblk), 6)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = sb.forward(to_bf16_tensor(q, DEV), to_bf16_tensor(k, DEV), to_bf16_tensor(v, DEV),
                     torch.from_numpy(idx).int().to(DEV), torch.from_numpy(cnt).int().to(DEV), scale=scale,
                     status=status)
    sb.check_status(status)
    got = f64(out)
    assert np.all(np.isfinite(got))
    check_attention(got, orc.block_sparse_attention(q, k, v, idx, cnt, scale))
