"""Shared comparison helpers for the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

# Attention output tolerance on bf16 inputs/outputs with fp32 accumulation.
ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 1e-2
# Top-k sets must match exactly where the oracle's relative score gap at the k-th boundary
# exceeds this; closer rows may legitimately select differently under fp32 score rounding.
TOPK_GAP = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_attn_close(got: np.ndarray, want: np.ndarray, what: str = "attention") -> dict:
    diff = np.abs(got - want)
    max_abs = float(diff.max()) if diff.size else 0.0
    den = float(np.sqrt((want ** 2).sum()))
    rel = float(np.sqrt((diff ** 2).sum()) / den) if den > 0 else float(np.sqrt((diff ** 2).sum()))
    assert max_abs <= ATTN_MAX_ABS, f"{what}: max abs error {max_abs:.3e} > {ATTN_MAX_ABS}"
    assert rel <= ATTN_REL_L2, f"{what}: relative L2 error {rel:.3e} > {ATTN_REL_L2}"
    return {"max_abs": max_abs, "rel_l2": rel}


def gpu_sets(kv_idx: torch.Tensor, kv_cnt: torch.Tensor) -> list:
    """int32 [B, heads, nT, kcap] + counts -> nested lists of int64 arrays (in stored order)."""
    idx = kv_idx.cpu().numpy()
    cnt = kv_cnt.cpu().numpy()
    B, nh, nT = cnt.shape
    return [[[idx[b, h, i, :cnt[b, h, i]].astype(np.int64) for i in range(nT)] for h in range(nh)]
            for b in range(B)]


def check_topk_sets(got: list, want: list, S: np.ndarray, k: int, heads=None) -> dict:
    """Exact equality where the oracle's gap exceeds TOPK_GAP; elsewhere the GPU set must be a
    valid top-k (right size, ascending, and no dropped tile scoring clearly above a kept one)."""
    from oracle import select
    gaps = select.topk_gap(S, k)
    n_exact = n_close = 0
    B, nh, nT = S.shape[:3]
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                g = got[b][h][i]
                w = want[b][h][i]
                assert np.all(np.diff(g) > 0), "indices must be strictly ascending"
                assert len(g) == len(w)
                if gaps[b, h, i] > TOPK_GAP:
                    np.testing.assert_array_equal(g, w, err_msg=f"row {(b, h, i)}")
                    n_exact += 1
                else:
                    row = S[b, h, i]
                    scale = np.abs(row).max()
                    dropped = np.setdiff1d(np.arange(nT), g)
                    if dropped.size:
                        assert row[dropped].max() <= row[g].min() + TOPK_GAP * scale
                    n_close += 1
    return {"exact": n_exact, "near_tie": n_close}
