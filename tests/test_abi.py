"""The C ABI library on the CPU: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before launching
anything (so these calls need no GPU).  Pointers passed here are never
dereferenced: validation returns first."""

import ctypes
import os
import re

import pytest
import torch

from block_sparse_attention_qk_b200 import build as sb_build
from block_sparse_attention_qk_b200._lib import SIGNATURES, lib
from oracle import sbattn_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbattn.h")

OK, INVALID, SHAPE, MISALIGNED, WORKSPACE, CUDA, DEVICE, TIMEOUT, CAPACITY = range(9)
A = 0x7F0000000000  # a 16-byte-aligned fake device address, never dereferenced


@pytest.fixture(scope="module")
def L():
    sb_build.build()
    return lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SBATTN_API\s+[\w\s\*]*?\b(sbattn_\w+)\s*\(", text)))


def test_header_declares_the_three_calls_and_binding_matches():
    names = declared_symbols()
    for n in ("sbattn_qk_norm_rope", "sbattn_select_blocks", "sbattn_forward"):
        assert n in names
    assert sorted(SIGNATURES) == names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_macros_match(L):
    text = open(HEADER).read()
    codes = dict((m, int(v)) for m, v in re.findall(r"#define (SBATTN_(?:OK|ERR_\w+))\s+(\d+)", text))
    assert codes["SBATTN_OK"] == OK and codes["SBATTN_ERR_CAPACITY"] == CAPACITY
    for code in codes.values():
        assert L.sbattn_strerror(code)
    assert L.sbattn_strerror(999) == b"unknown status"
    assert L.sbattn_version() >= 10000


def _keep(L, nblk, s):
    out = ctypes.c_int(-1)
    rc = L.sbattn_keep_count(nblk, s, ctypes.byref(out))
    return rc, out.value


def test_keep_count_bit_exact_with_oracle(L):
    for s100 in range(0, 101):
        for s in (s100 / 100, s100 / 100 + 1e-7, s100 / 100 - 3e-7):
            if not 0.0 <= s <= 1.0:
                continue
            for n in (1, 2, 3, 4, 7, 63, 64, 150, 252, 999, 1953, 3843, 100000):
                rc, K = _keep(L, n, s)
                assert rc == OK and K == orc.keep_count(n, s), (n, s)


def test_keep_count_golden(L):
    path = os.path.join(os.path.dirname(__file__), "golden", "keep_count.txt")
    for line in open(path):
        line = line.split("#", 1)[0].split()
        if line:
            assert _keep(L, int(line[0]), float(line[1])) == (OK, int(line[2]))


def test_keep_count_rejects(L):
    for s in (-0.001, 1.001, float("nan"), float("inf")):
        assert _keep(L, 10, s)[0] == INVALID
    assert _keep(L, 0, 0.5)[0] == INVALID
    assert L.sbattn_keep_count(10, 0.5, None) == INVALID


def test_workspace_bytes(L):
    assert L.sbattn_select_workspace_bytes(1, 124992, 40, 128) == 2 * 1 * 40 * 1953 * 128 * 4
    assert L.sbattn_select_workspace_bytes(2, 100, 3, 128) == 2 * 2 * 3 * 2 * 128 * 4  # partial block
    assert L.sbattn_select_workspace_bytes(1, 100, 3, 64) == 0


def _prologue(L, **kw):
    args = dict(q=A, k=A, w_q=A, w_k=A, q_out=A, k_out=A, q_pool=None, k_pool=None, B=1, T=2, Hh=8, W=16, H=2,
                d=128, dt=32, dh=48, dw=48, theta=10000.0, eps=1e-6, stream=None)
    args.update(kw)
    return L.sbattn_qk_norm_rope(*args.values())


def test_prologue_validation(L):
    assert _prologue(L, q=None) == INVALID
    assert _prologue(L, q_pool=A) == INVALID           # pools come in pairs
    assert _prologue(L, d=64, dt=16, dh=24, dw=24) == SHAPE
    assert _prologue(L, dt=30, dh=50) == SHAPE          # not multiples of 8
    assert _prologue(L, dt=32, dh=48, dw=40) == SHAPE   # does not sum to d
    assert _prologue(L, T=0) == INVALID
    assert _prologue(L, theta=-1.0) == INVALID
    assert _prologue(L, eps=float("nan")) == INVALID
    assert _prologue(L, q=A + 2) == MISALIGNED
    assert _prologue(L, k_out=A + 8) == MISALIGNED
    assert _prologue(L, T=4000, Hh=4000, W=4000) == SHAPE  # rotation table too large / too many blocks


def _select(L, **kw):
    args = dict(q=A, k=A, B=1, N=256, H=2, d=128, s=0.5, idx=A, cnt=A, cap=2, scores=None, ws=A,
                ws_bytes=1 << 20, stream=None)
    args.update(kw)
    return L.sbattn_select_blocks(*args.values())


def test_select_validation(L):
    assert _select(L, q=None) == INVALID
    assert _select(L, idx=None) == INVALID
    assert _select(L, d=96) == SHAPE
    assert _select(L, s=float("nan")) == INVALID
    assert _select(L, s=1.5) == INVALID
    assert _select(L, cap=1) == CAPACITY                 # K = 2 at s = 0.5, nblk = 4
    assert _select(L, ws=None) == WORKSPACE
    assert _select(L, ws_bytes=100) == WORKSPACE
    assert _select(L, ws=A + 4) == MISALIGNED
    assert _select(L, idx=A + 4) == MISALIGNED
    assert _select(L, N=0) == INVALID


def test_select_pooled_and_threshold_validation(L):
    f = L.sbattn_select_blocks_pooled
    assert f(A, A, 1, 4, 2, 128, 0.5, A, A, 1, None, None) == CAPACITY
    assert f(None, A, 1, 4, 2, 128, 0.5, A, A, 2, None, None) == INVALID
    assert f(A, A, 1, 4, 2, 100, 0.5, A, A, 2, None, None) == SHAPE
    g = L.sbattn_select_blocks_threshold
    assert g(A, A, 1, 4, 2, 128, 0.0, A, A, 3, None, None) == CAPACITY  # needs nblk entries
    assert g(A, A, 1, 4, 2, 128, float("nan"), A, A, 4, None, None) == INVALID
    assert g(A, A, 1, 4, 2, 128, 0.0, A + 1, A, 4, None, None) == MISALIGNED


def _forward(L, **kw):
    args = dict(q=A, k=A, v=A, idx=A, cnt=A, cap=2, out=A + 4096, B=1, N=256, H=2, d=128, scale=0.0,
                status=None, stream=None)
    args.update(kw)
    return L.sbattn_forward(*args.values())


def test_forward_validation(L):
    assert _forward(L, v=None) == INVALID
    assert _forward(L, out=A) == INVALID                 # aliases q
    assert _forward(L, cap=0) == INVALID
    assert _forward(L, scale=float("nan")) == INVALID
    assert _forward(L, d=256) == SHAPE
    assert _forward(L, H=0) == INVALID
    assert _forward(L, idx=A + 12) == MISALIGNED
    assert _forward(L, status=A + 2) == MISALIGNED
    assert _forward(L, B=1 << 20, N=1 << 20, H=1 << 10) == SHAPE  # item count overflows int32


def test_forward_diag_validation(L):
    """The failure-detection form: its limit and withheld tile are checked on
    the host before anything else (no GPU needed)."""
    args = (A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x400000, 4, A + 0x500000, 1, 256, 2, 128, 0.0, None)
    assert L.sbattn_forward_diag(*args, 999_999, -1, None) == INVALID          # limit below 1 ms
    assert L.sbattn_forward_diag(*args, 20_000_000_001, -1, None) == INVALID   # above 20 s
    assert L.sbattn_forward_diag(*args, 50_000_000, -2, None) == INVALID
    bad = (A, A + 0x100000, None) + args[3:]
    assert L.sbattn_forward_diag(*bad, 50_000_000, 0, None) == INVALID       # then the usual checks


def _adaln(L, x=A, shift=A + 0x1000, scale=A + 0x2000, out=A + 0x100000, B=2, N=300, C=5120, eps=1e-6):
    return L.sbattn_adaln_modulate(x, shift, scale, out, B, N, C, eps, None)


def test_adaln_validation(L):
    assert _adaln(L, x=None) == INVALID
    assert _adaln(L, shift=None) == INVALID
    assert _adaln(L, N=0) == INVALID
    assert _adaln(L, eps=float("nan")) == INVALID
    assert _adaln(L, eps=-1.0) == INVALID
    assert _adaln(L, C=5124) == SHAPE          # not a multiple of 8
    assert _adaln(L, C=8192) == SHAPE          # more channels than a warp holds
    assert _adaln(L, scale=A + 0x2008) == MISALIGNED
    assert _adaln(L, out=A + 4) == MISALIGNED


def _swiglu(L, gate=A, up=A + 0x10000, out=A + 0x100000, rows=100, F=13824, ld=13824):
    return L.sbattn_swiglu(gate, up, out, rows, F, ld, None)


def test_swiglu_validation(L):
    assert _swiglu(L, up=None) == INVALID
    assert _swiglu(L, rows=0) == INVALID
    assert _swiglu(L, F=12) == INVALID          # not a multiple of 8
    assert _swiglu(L, ld=13816) == INVALID      # row stride shorter than a row
    assert _swiglu(L, ld=13828) == INVALID      # row stride not a multiple of 8
    assert _swiglu(L, rows=1 << 40) == INVALID  # size overflow
    assert _swiglu(L, gate=A + 8) == MISALIGNED
    assert _swiglu(L, out=A + 0x100002) == MISALIGNED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure path")
def test_valid_call_without_gpu_fails_cleanly(L):
    # every argument is valid, so the call reaches the CUDA runtime, which
    # has no device here: it must report SBATTN_ERR_CUDA, not crash
    assert _forward(L) == CUDA
