"""Oracle: softmax attention restricted to kept (query tile, key tile) pairs (fp64).

Sources:
* ``bsa_attn`` page (FastVideo API docs), ``BSAAttentionImpl.__init__`` and ``forward``:
  bidirectional (no causal mask), one KV head per query head, softmax scale 1/sqrt(D), tensors
  ``[B, L, heads, D]`` in tile order, attention computed block-sparsely over kept block pairs.
* ``fastvideo.attention.backends`` page, ``sla.get_block_map``: the kept pairs are given per query
  block as a 0/1 block map or as the list of kept key-block indices.
* ``video_sparse_attn_h3`` page, ``tile()``: pad positions of the tile buffer hold zeros.

What is computed, for every valid query row ``r`` of query tile ``i``: one softmax over the union
of the valid keys of all key tiles kept for ``i``, ``o_r = sum_c softmax_c(scale * q_r . k_c) v_c``.
Readings taken where the pages are silent: pad keys get zero weight, pad query rows output zero,
and a query tile that keeps no key tile outputs zero. The softmax is evaluated in two passes (row
maximum, then exponentials and their sum) in fp64.
"""
from __future__ import annotations

import numpy as np

TILE_ELEMS = 64


def _key_rows(sets_i, vc, E: int = TILE_ELEMS) -> np.ndarray:
    parts = [E * int(j) + np.arange(int(vc[int(j)])) for j in sets_i]
    if not parts:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate(parts)


def attend_rows(q_rows: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray, scale: float):
    """Dense softmax attention of ``q_rows [m, D]`` over ``k_rows, v_rows [n, D]`` (fp64).

    Returns ``(out [m, D], weight_sum [m])``; the weights are normalised, so ``weight_sum`` is 1 up
    to rounding."""
    q = q_rows.astype(np.float64)
    k = k_rows.astype(np.float64)
    v = v_rows.astype(np.float64)
    logits = scale * (q @ k.T)
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    den = e.sum(axis=1, keepdims=True)
    w = e / den
    return w @ v, w.sum(axis=1)


def block_sparse_attention(qt, kt, vt, vc, sets, scale: float, keep=None, src=None,
                           q_tiles=None, return_wsum: bool = False, tile_elems: int = TILE_ELEMS):
    """Block-sparse attention on padded tile-ordered ``[B, E*nT, heads, D]`` tensors (``E`` =
    ``tile_elems``: 64, or 128 for the packed sequences' large tile).

    ``sets[b][h][i]``: kept key tiles of query tile ``i``. ``keep``/``src`` (``[B, heads, nT, 64]``)
    switch on the pruned-query variant: only kept rows attend, pruned rows copy ``src``'s output.
    ``q_tiles``: optional list of ``(b, h, i)`` to compute (other rows stay 0), for sampled checks.
    Returns fp64 ``[B, 64*nT, heads, D]`` (and the per-row weight sums if asked)."""
    B, Lp, nh, D = qt.shape
    E = int(tile_elems)
    nT = Lp // E
    out = np.zeros((B, Lp, nh, D), dtype=np.float64)
    wsum = np.zeros((B, Lp, nh), dtype=np.float64)
    todo = q_tiles if q_tiles is not None else [(b, h, i) for b in range(B) for h in range(nh)
                                                 for i in range(nT)]
    for (b, h, i) in todo:
        rows_k = _key_rows(sets[b][h][i], vc, E)
        n_q = int(vc[i])
        base = E * i
        if rows_k.size == 0:
            continue
        if keep is None:
            o, ws = attend_rows(qt[b, base:base + n_q, h], kt[b, rows_k, h], vt[b, rows_k, h], scale)
            out[b, base:base + n_q, h] = o
            wsum[b, base:base + n_q, h] = ws
        else:
            kk = np.nonzero(keep[b, h, i][:n_q])[0]
            o, ws = attend_rows(qt[b, base + kk, h], kt[b, rows_k, h], vt[b, rows_k, h], scale)
            blk = np.zeros((n_q, D), dtype=np.float64)
            wb = np.zeros(n_q, dtype=np.float64)
            blk[kk] = o
            wb[kk] = ws
            s = np.asarray(src[b, h, i][:n_q], dtype=np.int64)
            out[b, base:base + n_q, h] = blk[s]
            wsum[b, base:base + n_q, h] = wb[s]
    if return_wsum:
        return out, wsum
    return out
