"""Seeded synthetic workloads.

This module only draws random tensors: it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Shapes follow the video DiT attention layer described on the pages: one
attention layer of the MiniMax-H3 video model at 1344x768, 24 FPS, 5 s and
10 s (xiaodao.ai "MiniMax-H3 的 6.24 倍…", section "先把近两倍的免费收益拿走";
chat-gpts.plus "MiniMax-H3 在 8×H200 上基准测试…", section "事件核心：发生了什么").
The pages do not print the latent grid, head count or head size; the grids
below are the stand-in for that workload: 40 heads of size 128 over a
T x 48 x 84 latent grid (T = 31 for 5 s, 61 for 10 s) and its 84 x 48 portrait
transpose.

Value recipe (identical for every workload):
  u  ~ N(0, 1), one d-vector per (batch, 64-token block, head), shared by Q, K
       and V of that block;
  x  = N(0, 1) + 0.5 * u  for each of Q, K, V, rounded to bfloat16 (RNE);
  w_q, w_k ~ N(1, 0.1) per channel, rounded to bfloat16.
The shared per-block offset gives the pooled block scores a real ranking, as
in a video where a block's tokens are correlated.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch

BLOCK = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    Hh: int
    W: int
    sparsity: float
    seed: int
    d: int = 128
    dims: tuple = (32, 48, 48)
    theta: float = 10000.0
    eps: float = 1e-6

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.W

    @property
    def nblk(self) -> int:
        return -(-self.N // BLOCK)

    def with_sparsity(self, s: float) -> "Workload":
        return replace(self, sparsity=s)


WORKLOADS = {
    # 2 x 8 x 16 grid, 4 blocks, keep 2 of 4 (diagonal included)
    "tiny": Workload("tiny", B=1, H=2, T=2, Hh=8, W=16, sparsity=0.5, seed=0),
    # sparsity 0 keeps every block: must equal dense attention
    "dense": Workload("dense", B=1, H=8, T=4, Hh=48, W=84, sparsity=0.0, seed=1),
    # 5 s at 1344x768: N = 124992 tokens, 1953 blocks
    "5s": Workload("5s", B=1, H=40, T=31, Hh=48, W=84, sparsity=0.75, seed=2),
    "5s_aggr": Workload("5s_aggr", B=1, H=40, T=31, Hh=48, W=84, sparsity=0.8, seed=2),
    # 10 s at 1344x768: N = 245952 tokens, 3843 blocks
    "10s": Workload("10s", B=1, H=40, T=61, Hh=48, W=84, sparsity=0.75, seed=3),
    # 768x1344 portrait grid
    "portrait": Workload("portrait", B=1, H=40, T=31, Hh=84, W=48, sparsity=0.75, seed=4),
}


def make_inputs(wl: Workload, device="cpu", seed: int | None = None) -> dict:
    """Draw q, k, v [B, N, H, d] and w_q, w_k [d], all bfloat16, on `device`.

    The draw order is fixed (u, q-noise, k-noise, v-noise, w_q, w_k) and uses a
    generator on `device`, so the same (workload, seed, device) always gives
    the same tensors.  CPU and CUDA generators give different streams: tests
    that compare the two sides draw once and copy.
    """
    seed = wl.seed if seed is None else seed
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    B, N, H, d, nblk = wl.B, wl.N, wl.H, wl.d, wl.nblk
    u = torch.randn((B, nblk, H, d), generator=g, device=device, dtype=torch.float32)
    u_tok = u.repeat_interleave(BLOCK, dim=1)[:, :N]
    out = {}
    for name in ("q", "k", "v"):
        x = torch.randn((B, N, H, d), generator=g, device=device, dtype=torch.float32)
        x.add_(u_tok, alpha=0.5)
        out[name] = x.to(torch.bfloat16)
        del x
    del u_tok
    for name in ("w_q", "w_k"):
        w = 1.0 + 0.1 * torch.randn((d,), generator=g, device=device, dtype=torch.float32)
        out[name] = w.to(torch.bfloat16)
    return out


def custom_workload(name="custom", *, B=1, H=2, T=1, Hh=4, W=16, sparsity=0.5, seed=0, **kw) -> Workload:
    """A workload of any grid, for edge-case tests."""
    return Workload(name, B=B, H=H, T=T, Hh=Hh, W=W, sparsity=sparsity, seed=seed, **kw)
