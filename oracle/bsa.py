"""Oracle: query pruning and reconstruction of bidirectional sparse attention (fp64).

Source: ``bsa_attn`` page (FastVideo API docs), ``BSAAttentionImpl.forward``: the tile-ordered
sequence is viewed as blocks of ``block_size`` tokens (the length must be an exact multiple), the
queries of each block are pruned, KV blocks are selected from the pruned queries, attention runs
for the kept queries only, and the pruned positions are filled back in before the output is
returned in tile order. ``BSAAttentionImpl.__init__`` fixes the contract: no grouped-query
attention, no causal mask, softmax scale 1/sqrt(D).

The pages name the pruning and reconstruction helpers but do not print their bodies. Readings
taken here (the workload definition prunes by a cosine threshold):
* a query row of a block is pruned iff its cosine similarity to the mean of all rows of the block
  exceeds the threshold; a cosine with a zero-norm operand counts as 0;
* if every row of a block would be pruned, the row with the lowest cosine (lowest index on ties)
  is kept;
* a pruned row takes the output of the kept row of the same block and head that it is most
  cosine-similar to (lowest index on ties);
* KV selection pools the queries over the kept rows of the block only.

The page's forward passes ``attn_metadata.query_keep_ratio`` to the pruning helper, which returns a
``keep_size``: a fixed count of kept rows per block. Readings for that mode:
* ``keep_size = max(1, floor(ratio * 64))`` (computed in fp64);
* the kept rows are the ``keep_size`` rows least similar to the block mean (lowest cosine first,
  lowest index on ties) — the rows the threshold mode would keep last-pruned; pruned rows copy
  their most similar kept row exactly as in the threshold mode.
"""
from __future__ import annotations

import numpy as np

TILE_ELEMS = 64


def _cos(a: np.ndarray, b: np.ndarray) -> float:
    na = float(np.sqrt(np.dot(a, a)))
    nb = float(np.sqrt(np.dot(b, b)))
    if na == 0.0 or nb == 0.0:
        return 0.0
    return float(np.dot(a, b)) / (na * nb)


def prune_block(rows: np.ndarray, thresh: float):
    """One block ``[n, D]`` -> ``(keep bool[n], src int[n], cos_to_mean float[n])``.

    ``src[i] == i`` for kept rows; for pruned rows it names the kept row whose output they copy."""
    rows = rows.astype(np.float64)
    n = rows.shape[0]
    mu = rows.sum(axis=0) / n
    cmean = np.array([_cos(rows[i], mu) for i in range(n)])
    keep = ~(cmean > thresh)
    if not keep.any():
        keep[int(np.argmin(cmean))] = True
    kept = np.nonzero(keep)[0]
    src = np.arange(n)
    for i in range(n):
        if keep[i]:
            continue
        best_j, best_c = -1, -np.inf
        for j in kept:
            c = _cos(rows[i], rows[j])
            if c > best_c:
                best_j, best_c = int(j), c
        src[i] = best_j
    return keep, src, cmean


def keep_size_for_ratio(ratio: float, n: int = TILE_ELEMS) -> int:
    """Kept rows per block of ``n`` for a keep ratio in (0, 1]."""
    return max(1, min(n, int(np.floor(ratio * n))))


def _sources(rows: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """For each pruned row, the kept row it is most cosine-similar to (lowest index on ties)."""
    kept = np.nonzero(keep)[0]
    src = np.arange(rows.shape[0])
    for i in range(rows.shape[0]):
        if keep[i]:
            continue
        best_j, best_c = -1, -np.inf
        for j in kept:
            c = _cos(rows[i], rows[j])
            if c > best_c:
                best_j, best_c = int(j), c
        src[i] = best_j
    return src


def prune_block_ratio(rows: np.ndarray, ratio: float):
    """Ratio mode for one block ``[n, D]`` -> ``(keep bool[n], src int[n], cos_to_mean float[n])``:
    the ``keep_size_for_ratio(ratio, n)`` rows with the lowest cosine to the block mean are kept."""
    rows = rows.astype(np.float64)
    n = rows.shape[0]
    mu = rows.sum(axis=0) / n
    cmean = np.array([_cos(rows[i], mu) for i in range(n)])
    order = sorted(range(n), key=lambda i: (cmean[i], i))  # least similar first
    keep = np.zeros(n, dtype=bool)
    keep[order[:keep_size_for_ratio(ratio, n)]] = True
    return keep, _sources(rows, keep), cmean


def prune_queries_ratio(qt: np.ndarray, ratio: float):
    """Ratio mode over tile-ordered queries ``[B, 64*nT, heads, D]``; outputs as prune_queries."""
    B, Lp, nh, D = qt.shape
    nT = Lp // TILE_ELEMS
    keep = np.zeros((B, nh, nT, TILE_ELEMS), dtype=bool)
    src = np.zeros((B, nh, nT, TILE_ELEMS), dtype=np.int64)
    cosm = np.zeros((B, nh, nT, TILE_ELEMS), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                rows = qt[b, TILE_ELEMS * i:TILE_ELEMS * (i + 1), h, :]
                keep[b, h, i], src[b, h, i], cosm[b, h, i] = prune_block_ratio(rows, ratio)
    return keep, src, cosm


def prune_queries(qt: np.ndarray, thresh: float):
    """Tile-ordered queries ``[B, 64*nT, heads, D]`` (no pad rows) ->
    ``keep [B, heads, nT, 64]`` bool, ``src [B, heads, nT, 64]`` int, ``cos [B, heads, nT, 64]``."""
    B, Lp, nh, D = qt.shape
    nT = Lp // TILE_ELEMS
    keep = np.zeros((B, nh, nT, TILE_ELEMS), dtype=bool)
    src = np.zeros((B, nh, nT, TILE_ELEMS), dtype=np.int64)
    cosm = np.zeros((B, nh, nT, TILE_ELEMS), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                rows = qt[b, TILE_ELEMS * i:TILE_ELEMS * (i + 1), h, :]
                keep[b, h, i], src[b, h, i], cosm[b, h, i] = prune_block(rows, thresh)
    return keep, src, cosm


def pooled_kept_queries(qt: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """Mean of each block's kept query rows: ``[B, heads, nT, D]`` fp64."""
    B, Lp, nh, D = qt.shape
    nT = Lp // TILE_ELEMS
    out = np.zeros((B, nh, nT, D), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                rows = qt[b, TILE_ELEMS * i:TILE_ELEMS * (i + 1), h, :].astype(np.float64)
                kk = keep[b, h, i]
                out[b, h, i] = rows[kk].sum(axis=0) / int(kk.sum())
    return out
