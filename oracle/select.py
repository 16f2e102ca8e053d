"""Oracle: tile-to-tile scores and KV tile selection (fp64 scores, integer sets).

Sources:
* ``fastvideo.attention.backends`` page, ``sla.get_block_map``: scores are the pooled queries times
  the transposed pooled keys (no softmax scale), ``topk = min(K, int(ratio * K))`` tiles are kept per
  query tile and the map is recorded both as a 0/1 block map and as an index list (LUT).
* ``bsa_attn`` page, ``BSAAttentionImpl.forward``: KV tiles are chosen per query block from the
  pruned queries with a cumulative threshold (``kv_cumulative_threshold``) and a floor
  (``min_kv_blocks``).

Readings taken where the pages are silent:
* Smooth-k (subtracting the sequence mean of K before pooling) is left out: it subtracts
  ``pq_i . mean(k)`` from every score of row ``i``, which changes neither the top-k set nor a
  softmax over the row. A CPU test pins that invariance.
* Top-k ties go to the lower KV tile index; kept indices are reported in ascending order.
* Mass mode: ``p = softmax(scale * S_i)`` over the row, with ``scale`` the attention softmax scale;
  tiles are taken in descending ``p`` (ties: lower index) until the running sum first reaches the
  threshold, the tile that reaches it included; at least ``min_k`` tiles are kept; if the running
  sum never reaches the threshold (rounding at threshold 1) every tile is kept. At a threshold of
  1 every tile is kept outright: every softmax probability is positive, so the exact running sum
  reaches 1 only with the last tile, while a rounded one can reach it earlier when the tail
  probabilities are too small to change it.
"""
from __future__ import annotations

import numpy as np


def tile_scores(pq: np.ndarray, pk: np.ndarray) -> np.ndarray:
    """``[B, heads, nT, D]`` x2 -> ``[B, heads, nT, nT]``: ``S[i, j] = pq_i . pk_j`` in fp64."""
    return np.matmul(pq.astype(np.float64), np.swapaxes(pk.astype(np.float64), -1, -2))


def _desc_order(row: np.ndarray) -> np.ndarray:
    """Indices of ``row`` by descending value, ties by ascending index."""
    idx = np.arange(row.shape[0])
    return np.lexsort((idx, -row))


def select_topk_row(row: np.ndarray, k: int) -> np.ndarray:
    k = min(int(k), row.shape[0])
    return np.sort(_desc_order(row)[:k])


def select_topk(S: np.ndarray, k: int) -> list:
    """Per row of ``S [..., nT, nT]``: the ascending indices of its ``k`` largest scores.

    Returns a nested list with the leading dims of ``S`` and an int64 array per query tile."""
    return _map_rows(S, lambda r: select_topk_row(r, k))


def topk_gap(S: np.ndarray, k: int) -> np.ndarray:
    """Relative gap at the k-th boundary per row: ``(S_(k) - S_(k+1)) / max_j |S_j|``.

    ``inf`` when every tile is kept. Rows whose gap is small may be selected differently by any
    implementation whose scores carry rounding error; parity on them is checked for validity."""
    nT = S.shape[-1]
    if k >= nT:
        return np.full(S.shape[:-1], np.inf)
    srt = -np.sort(-S, axis=-1)
    den = np.maximum(np.abs(S).max(axis=-1), np.finfo(np.float64).tiny)
    return (srt[..., k - 1] - srt[..., k]) / den


def softmax_row(x: np.ndarray) -> np.ndarray:
    z = x - x.max()
    e = np.exp(z)
    return e / e.sum()


def select_mass_row(row: np.ndarray, scale: float, tau: float, min_k: int) -> np.ndarray:
    nT = row.shape[0]
    p = softmax_row(scale * row.astype(np.float64))
    order = _desc_order(row.astype(np.float64))
    csum = np.cumsum(p[order])
    hit = np.nonzero(csum >= tau)[0]
    m = int(hit[0]) + 1 if hit.size and tau < 1.0 else nT
    m = max(m, min(int(min_k), nT))
    return np.sort(order[:m])


def select_mass(S: np.ndarray, scale: float, tau: float, min_k: int) -> list:
    """Per row: the smallest set of KV tiles, taken in descending softmax probability, whose mass
    reaches ``tau`` (at least ``min_k`` tiles). Ascending indices per query tile."""
    return _map_rows(S, lambda r: select_mass_row(r, scale, tau, min_k))


def mass_margins(row: np.ndarray, scale: float, tau: float, min_k: int) -> dict:
    """How decisively a row's mass selection is determined, for parity checks.

    ``cut_gap``: relative probability gap between the last kept and the first dropped tile;
    ``sum_margin``: how far the running sums just before and at the cut lie from ``tau`` (``inf``
    when the floor ``min_k``, not the threshold, fixes the count)."""
    nT = row.shape[0]
    p = softmax_row(scale * row.astype(np.float64))
    order = _desc_order(row.astype(np.float64))
    ps = p[order]
    csum = np.cumsum(ps)
    hit = np.nonzero(csum >= tau)[0] if tau < 1.0 else np.zeros(0, dtype=np.int64)
    m_tau = int(hit[0]) + 1 if hit.size else nT
    m = max(m_tau, min(int(min_k), nT))
    cut_gap = np.inf if m >= nT else (ps[m - 1] - ps[m]) / ps[0]
    if m > m_tau or not hit.size:
        sum_margin = np.inf if m > m_tau else abs(tau - csum[-1])
    else:
        before = csum[m - 2] if m >= 2 else 0.0
        sum_margin = min(tau - before, csum[m - 1] - tau)
    return {"count": m, "cut_gap": cut_gap, "sum_margin": sum_margin}


def sets_to_map(sets, nT: int) -> np.ndarray:
    """Nested per-row index lists -> 0/1 block map ``[..., nT, nT]`` (uint8)."""
    if isinstance(sets, np.ndarray):
        row = np.zeros(nT, dtype=np.uint8)
        row[sets.astype(np.int64)] = 1
        return row
    return np.stack([sets_to_map(s, nT) for s in sets])


def map_to_sets(mask: np.ndarray) -> list:
    """0/1 block map ``[..., nT, nT]`` -> nested per-row ascending index lists."""
    return _map_rows(mask, lambda r: np.nonzero(r)[0].astype(np.int64))


def _map_rows(S: np.ndarray, fn) -> list:
    if S.ndim == 1:
        return fn(S)
    return [_map_rows(S[i], fn) for i in range(S.shape[0])]
