"""The allocation-free selection entry point, through the C ABI.

sbattn_select_blocks_noalloc serves callers that cannot allocate device
memory when they run the layer (a host that hands the library only the
layer's inputs and outputs, or a runtime that forbids allocation once it is
serving): its pooled-means scratch is an array built into the library.  It
must give exactly what sbattn_select_blocks gives with a caller workspace,
call after call, although every call reuses the same built-in array.

This file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

from block_sparse_attention_qk_b200 import build as sb_build
from block_sparse_attention_qk_b200._lib import lib
from block_sparse_attention_qk_b200.inputs import custom_workload, make_inputs
from oracle import sbattn_oracle as orc

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
MAX_ROWS = 4096  # SBATTN_NOALLOC_MAX_POOLED_ROWS


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _rotated(wl):
    # stored (bf16) prologue outputs of the oracle, as selection inputs
    x = make_inputs(wl)
    f = lambda t: t.to(torch.float64).numpy()
    qr, kr = orc.qk_norm_rope(f(x["q"]), f(x["k"]), f(x["w_q"]), f(x["w_k"]), wl.T, wl.Hh, wl.W)
    to = lambda a: torch.from_numpy(orc.round_to_bf16(a)).float().to(torch.bfloat16).to(DEV)
    return to(qr), to(kr)


def _outputs(B, H, nblk, K):
    return (torch.full((B, H, nblk, K), -7, dtype=torch.int32, device=DEV),
            torch.full((B, H, nblk), -7, dtype=torch.int32, device=DEV),
            torch.full((B, H, nblk, nblk), float("nan"), dtype=torch.float32, device=DEV))


def _run_both(L, q, k, sparsity):
    B, N, H, d = q.shape
    nblk = -(-N // 64)
    K = orc.keep_count(nblk, sparsity)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ref = _outputs(B, H, nblk, K)
    ws = torch.empty(L.sbattn_select_workspace_bytes(B, N, H, d), dtype=torch.uint8, device=DEV)
    rc = L.sbattn_select_blocks(_p(q), _p(k), B, N, H, d, sparsity, _p(ref[0]), _p(ref[1]), K, _p(ref[2]),
                                _p(ws), ws.numel(), stream)
    assert rc == 0
    got = _outputs(B, H, nblk, K)
    rc = L.sbattn_select_blocks_noalloc(_p(q), _p(k), B, N, H, d, sparsity, _p(got[0]), _p(got[1]), K,
                                        _p(got[2]), stream)
    assert rc == 0
    torch.cuda.synchronize()
    return ref, got


def test_no_alloc_selection_matches_workspace_entry_point_twice_in_a_row():
    sb_build.build()
    L = lib()
    # two calls in a row on the shared built-in scratch: a larger problem
    # first, then a smaller one that reuses the front of the same array
    big = custom_workload("big", B=2, H=6, T=4, Hh=16, W=40, sparsity=0.7, seed=31)   # 2*6*40 = 480 rows
    small = custom_workload("small", B=1, H=3, T=3, Hh=7, W=13, sparsity=0.5, seed=32)  # ragged N = 273
    for wl in (big, small):
        q, k = _rotated(wl)
        ref, got = _run_both(L, q, k, wl.sparsity)
        # the same kernels on the same inputs: scores and kept lists identical
        assert torch.equal(got[2], ref[2])
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1], ref[1])
        K = orc.keep_count(wl.nblk, wl.sparsity)
        assert torch.all(got[1] == K)


def test_no_alloc_selection_at_exactly_the_scratch_limit():
    """B * H * nblk == 4096: the pooled key means end at the last byte of the
    built-in array, so an off-by-one in the limit or the offsets would show."""
    sb_build.build()
    L = lib()
    wl = custom_workload("edge", B=1, H=64, T=1, Hh=64, W=64, sparsity=0.75, seed=33)  # N = 4096, nblk = 64
    assert wl.B * wl.H * wl.nblk == MAX_ROWS
    q, k = _rotated(wl)
    ref, got = _run_both(L, q, k, wl.sparsity)
    assert torch.equal(got[2], ref[2])
    assert torch.equal(got[0], ref[0])
    assert torch.equal(got[1], ref[1])


def test_no_alloc_calls_allocate_no_device_memory_after_the_first():
    """After one warm-up call on the device (which, under CUDA's lazy module
    loading, is when the library's built-in array comes into existence),
    further calls leave the device's free memory unchanged."""
    sb_build.build()
    L = lib()
    wl = custom_workload("mem", B=1, H=4, T=2, Hh=16, W=32, sparsity=0.5, seed=34)
    q, k = _rotated(wl)
    B, N, H, d = q.shape
    nblk = -(-N // 64)
    K = orc.keep_count(nblk, wl.sparsity)
    out = _outputs(B, H, nblk, K)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        rc = L.sbattn_select_blocks_noalloc(_p(q), _p(k), B, N, H, d, wl.sparsity, _p(out[0]), _p(out[1]), K,
                                            _p(out[2]), stream)
        assert rc == 0

    call()  # warm-up
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before


def test_no_alloc_rejects_problems_beyond_the_scratch():
    sb_build.build()
    L = lib()
    a = torch.zeros(16, dtype=torch.int32, device=DEV)  # never read: the call returns first
    # B*H*nblk = 1*33*128 = 4224 > 4096
    rc = L.sbattn_select_blocks_noalloc(_p(a), _p(a), 1, 128 * 64, 33, 128, 0.5, _p(a), _p(a), 64, None, None)
    assert rc == 4  # SBATTN_ERR_WORKSPACE
    assert L.sbattn_select_blocks_noalloc(_p(a), _p(a), 1, 64 * 64, MAX_ROWS // 64 + 1, 128, 0.5, _p(a), _p(a),
                                          64, None, None) == 4
    assert L.sbattn_select_blocks_noalloc(_p(a), _p(a), 1, 256, 2, 64, 0.5, _p(a), _p(a), 2, None, None) == 2
