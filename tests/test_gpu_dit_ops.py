"""GPU parity of the fused DiT-block elementwise steps (AdaLN modulation,
SwiGLU gating) through the C ABI against the fp64 oracle.  Inputs are drawn
by a seeded NumPy generator and rounded to bf16; the oracle runs on exactly
those values.  Tolerance: bf16 output rounding (half an ulp, 2^-9 relative)
plus fp32 arithmetic -> 4e-3 * max(1, |ref|), and at least 99.9 % of the
elements equal to the rounded fp64 value."""

import numpy as np
import pytest
import torch

import block_sparse_attention_qk_b200 as sb
from oracle import sbattn_oracle as orc

from .parity import check_prologue, f64, to_bf16_tensor

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bf16(rng, shape, loc=0.0, scale=1.0):
    return orc.round_to_bf16(rng.normal(loc, scale, size=shape))


# C = 5120 (40 heads x 128: rows fill every lane 20 times), 1152 (partial
# lanes), 6144 (largest supported), 8 (one vector); N spans ragged counts
@pytest.mark.parametrize("B,N,C", [(2, 257, 5120), (1, 64, 1152), (3, 5, 6144), (2, 3, 8)])
def test_adaln_matches_oracle(B, N, C):
    rng = np.random.default_rng(1000 + C + N)
    x = _bf16(rng, (B, N, C), 0.3, 1.5)
    shift = _bf16(rng, (B, C), 0.0, 0.5)
    scale = _bf16(rng, (B, C), 0.0, 0.3)
    out = sb.adaln_modulate(to_bf16_tensor(x, DEV), to_bf16_tensor(shift, DEV), to_bf16_tensor(scale, DEV))
    torch.cuda.synchronize()
    check_prologue(f64(out), orc.adaln_modulate(x, shift, scale), "adaln")


def test_adaln_constant_rows_and_in_place():
    rng = np.random.default_rng(7)
    B, N, C = 2, 40, 5120
    x = _bf16(rng, (B, N, C))
    x[0, 3, :] = 3.25       # constant rows normalise to 0: output = shift
    x[1, 7, :] = -0.5
    shift = _bf16(rng, (B, C), 0.0, 0.5)
    scale = _bf16(rng, (B, C), 0.0, 0.3)
    xt = to_bf16_tensor(x, DEV)
    out = sb.adaln_modulate(xt, to_bf16_tensor(shift, DEV), to_bf16_tensor(scale, DEV), out=xt)
    torch.cuda.synchronize()
    got = f64(out)
    check_prologue(got, orc.adaln_modulate(x, shift, scale), "adaln in place")
    np.testing.assert_array_equal(got[0, 3], shift[0])
    np.testing.assert_array_equal(got[1, 7], shift[1])


def test_adaln_full_size_sampled_rows():
    # the 5 s layer's hidden states: [1, 124992, 5120] bf16 (1.28 GB)
    B, N, C = 1, 124992, 5120
    g = torch.Generator(device=DEV).manual_seed(5)
    x = (torch.randn((B, N, C), generator=g, device=DEV) * 1.5 + 0.3).to(torch.bfloat16)
    shift = (torch.randn((B, C), generator=g, device=DEV) * 0.5).to(torch.bfloat16)
    scale = (torch.randn((B, C), generator=g, device=DEV) * 0.3).to(torch.bfloat16)
    out = sb.adaln_modulate(x, shift, scale)
    torch.cuda.synchronize()
    rows = torch.from_numpy(np.random.default_rng(6).choice(N, 48, replace=False)).to(DEV)
    xs = f64(x[:, rows])
    check_prologue(f64(out[:, rows]), orc.adaln_modulate(xs, f64(shift), f64(scale)), "adaln full size")


@pytest.mark.parametrize("rows,F", [(333, 1000), (77, 13824), (1, 8)])
def test_swiglu_matches_oracle(rows, F):
    rng = np.random.default_rng(2000 + rows + F)
    gate = _bf16(rng, (rows, F), 0.0, 2.0)
    up = _bf16(rng, (rows, F))
    out = sb.swiglu(to_bf16_tensor(gate, DEV), to_bf16_tensor(up, DEV))
    torch.cuda.synchronize()
    check_prologue(f64(out), orc.swiglu(gate, up), "swiglu")


def test_swiglu_fused_projection_layout_and_limits():
    rng = np.random.default_rng(9)
    rows, F = 129, 2048
    h = _bf16(rng, (rows, 2 * F), 0.0, 2.0)
    h[:5, :F] = orc.round_to_bf16(np.linspace(-100.0, 100.0, 5 * F)).reshape(5, F)  # saturating gates
    out = sb.swiglu(to_bf16_tensor(h, DEV))
    torch.cuda.synchronize()
    got, ref = f64(out), orc.swiglu(h[:, :F], h[:, F:])
    check_prologue(got[5:], ref[5:], "swiglu fused layout")
    # saturating gates: within the bound; below about -87 the fp32 exp of -gate
    # overflows and the kernel returns 0 where the fp64 value is ~1e-37 or less
    err = np.abs(got[:5] - ref[:5])
    assert np.all(err <= 4e-3 * np.maximum(1.0, np.abs(ref[:5])))


def test_swiglu_full_size_sampled_rows():
    # the 5 s layer's MLP activations, reading F = 13824 (the pages give no MLP width)
    rows, F = 124992, 13824
    g = torch.Generator(device=DEV).manual_seed(8)
    gate = (torch.randn((rows, F), generator=g, device=DEV) * 2.0).to(torch.bfloat16)
    up = torch.randn((rows, F), generator=g, device=DEV).to(torch.bfloat16)
    out = sb.swiglu(gate, up)
    torch.cuda.synchronize()
    r = torch.from_numpy(np.random.default_rng(10).choice(rows, 32, replace=False)).to(DEV)
    check_prologue(f64(out[r]), orc.swiglu(f64(gate[r]), f64(up[r])), "swiglu full size")
