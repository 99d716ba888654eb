"""CPU checks of the seeded input generator (the one module both sides share,
holding no arithmetic of the method) and of the binding's argument checks,
which reject bad tensors before the library is called."""

import pytest
import torch

import block_sparse_attention_qk_b200 as sb
from block_sparse_attention_qk_b200.inputs import WORKLOADS, custom_workload, make_inputs
from oracle import sbattn_oracle as orc


def test_workload_sizes_match_the_configs():
    # the configs' token and block counts and the kept-block budgets they quote
    expect = {"tiny": (256, 4, 2), "dense": (16128, 252, 252), "5s": (124992, 1953, 489),
              "5s_aggr": (124992, 1953, 391), "10s": (245952, 3843, 961), "portrait": (124992, 1953, 489)}
    for name, (N, nblk, K) in expect.items():
        wl = WORKLOADS[name]
        assert (wl.N, wl.nblk, orc.keep_count(wl.nblk, wl.sparsity)) == (N, nblk, K), name
    assert orc.keep_count(1953, 0.5) == 977 and orc.keep_count(1953, 0.9) == 196


def test_inputs_are_seeded_bf16_and_shaped():
    wl = WORKLOADS["tiny"]
    a, b = make_inputs(wl), make_inputs(wl)
    for key in ("q", "k", "v", "w_q", "w_k"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key]), key
    assert a["q"].shape == (wl.B, wl.N, wl.H, wl.d) and a["w_q"].shape == (wl.d,)
    c = make_inputs(wl, seed=wl.seed + 1)
    assert not torch.equal(a["q"], c["q"])


def test_inputs_share_the_block_offset():
    # Q, K and V of one (block, head) share the offset u: their block means correlate
    wl = custom_workload("t", B=1, H=2, T=2, Hh=8, W=16, sparsity=0.5, seed=5)
    x = make_inputs(wl)
    qb = x["q"].float().reshape(1, -1, 64, 2, 128).mean(2)
    kb = x["k"].float().reshape(1, -1, 64, 2, 128).mean(2)
    corr = torch.nn.functional.cosine_similarity(qb.flatten(0, 2), kb.flatten(0, 2), dim=-1)
    assert corr.mean() > 0.9


def test_binding_rejects_host_and_wrong_dtype_tensors():
    q = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sb.forward(q, q, q, torch.zeros(1, 1, 1, 1, dtype=torch.int32), torch.ones(1, 1, 1, dtype=torch.int32))
    with pytest.raises(TypeError):
        sb.adaln_modulate(q.float(), q, q)
    with pytest.raises(TypeError):
        sb.swiglu(torch.zeros(4, 16))
