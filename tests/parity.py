"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (all bf16 results against float64):
  prologue   |gpu - ref| <= 4e-3 * max(1, |ref|) element-wise, and at least
             99.9 % of the elements equal to ref rounded to bf16.  (A flat
             4e-3 absolute bound is below half a bf16 ulp once |ref| >= 2,
             where the spacing is 2^-6; scaling by max(1, |ref|) keeps the
             bound at about half an ulp everywhere.)
  selection  kept sets equal the oracle's except in near-tie rows: the
             oracle's (K-1)-th and K-th largest off-diagonal scores a, b with
             |a - b| <= 1e-5 * max(|a|, |b|, |q_bar_i| * max_j |k_bar_j|);
             every block in the difference must score within that tolerance of
             the boundary; and at least 99.9 % of all keep/drop decisions agree.
  attention  max |gpu - ref| <= 1e-2 and mean |gpu - ref| <= 1e-3.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import sbattn_oracle as orc

PROLOGUE_REL = 4e-3
NEAR_TIE_REL = 1e-5
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_ABS = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def to_bf16_tensor(x: np.ndarray, device) -> torch.Tensor:
    """Exact bf16 tensor of values that are already bf16-representable."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32).to(torch.bfloat16).to(device)


def check_prologue(gpu: np.ndarray, ref: np.ndarray, what="prologue"):
    err = np.abs(gpu - ref)
    bound = PROLOGUE_REL * np.maximum(1.0, np.abs(ref))
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"{what}: error reaches {worst:.3f} of the bound (max abs err {err.max():.3e})"
    exact = float(np.mean(gpu == orc.round_to_bf16(ref)))
    assert exact >= 0.999, f"{what}: only {exact:.5f} of elements equal the rounded fp64 value"
    return {"max_abs": float(err.max()), "exact_frac": exact, "worst_vs_bound": worst}


def check_kept_structure(idx: np.ndarray, cnt: np.ndarray, nblk: int, K=None):
    """Sorted, unique, in range, diagonal present, -1 past the count."""
    B, H, nb, cap = idx.shape
    assert nb == nblk
    if K is not None:
        assert np.all(cnt == K), "kept count differs from the budget"
    diag = np.arange(nblk)[None, None, :, None]
    for b in range(B):
        for h in range(H):
            for i in range(nblk):
                c = int(cnt[b, h, i])
                row = idx[b, h, i]
                assert 1 <= c <= cap
                kept = row[:c]
                assert np.all(np.diff(kept) > 0), "kept list not strictly ascending"
                assert kept[0] >= 0 and kept[-1] < nblk
                assert i in kept, "diagonal block missing"
                assert np.all(row[c:] == -1)
    del diag


def check_selection(gpu_idx, gpu_cnt, ref_idx, ref_scores, q_bar, k_bar, tol_rel=NEAR_TIE_REL):
    """Compare kept sets row by row under the near-tie rule; returns stats."""
    B, H, nblk, K = ref_idx.shape
    n_rows = n_diff = 0
    disagree = 0
    for b in range(B):
        for h in range(H):
            kmax = np.max(np.linalg.norm(k_bar[b, h], axis=-1))
            for i in range(nblk):
                n_rows += 1
                g = set(gpu_idx[b, h, i, :gpu_cnt[b, h, i]].tolist())
                r = set(ref_idx[b, h, i].tolist())
                if g == r:
                    continue
                n_diff += 1
                sym = g ^ r
                disagree += len(sym)
                row = ref_scores[b, h, i].astype(np.float32).astype(np.float64)
                off = np.sort(np.delete(row, i))[::-1]
                cs = np.linalg.norm(q_bar[b, h, i]) * kmax
                a_ = off[K - 2] if K >= 2 else np.inf
                b_ = off[K - 1] if K - 1 < len(off) else -np.inf
                tol = tol_rel * max(abs(a_), abs(b_), cs)
                assert abs(a_ - b_) <= tol, f"row {(b, h, i)} differs but is no near tie: gap {abs(a_ - b_):.3e} > {tol:.3e}"
                for j in sym:
                    assert abs(row[j] - a_) <= tol or abs(row[j] - b_) <= tol, f"block {j} of row {(b, h, i)} far from the boundary"
    agree = 1.0 - disagree / float(B * H * nblk * nblk)
    assert agree >= 0.999, f"only {agree:.5f} of keep/drop decisions agree"
    return {"rows": n_rows, "rows_differing": n_diff, "decision_agreement": agree}


def check_attention(gpu: np.ndarray, ref: np.ndarray, what="attention"):
    err = np.abs(gpu - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= ATTN_MAX_ABS, f"{what}: max abs error {mx:.3e} > {ATTN_MAX_ABS}"
    assert mean <= ATTN_MEAN_ABS, f"{what}: mean abs error {mean:.3e} > {ATTN_MEAN_ABS}"
    return {"max_abs": mx, "mean_abs": mean}


def oracle_prologue(x: dict, wl):
    """fp64 prologue of the oracle and its bf16-rounded copy (the stored form)."""
    qr, kr = orc.qk_norm_rope(f64(x["q"]), f64(x["k"]), f64(x["w_q"]), f64(x["w_k"]), wl.T, wl.Hh, wl.W,
                              wl.dims, wl.theta, wl.eps)
    return qr, kr, orc.round_to_bf16(qr), orc.round_to_bf16(kr)
