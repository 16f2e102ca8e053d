"""Oracle: the whole hot path chained the way the method runs it (fp64).

Stage order, as the ``bsa_attn`` page (``preprocess_qkv`` -> ``forward`` -> ``postprocess_output``)
and the ``sla`` page (``get_block_map`` before the sparse attention) lay it out:
  1. scatter Q, K, V from raster order into the padded tile order;
  2. coarse stage: mean-pool Q and K per tile, score tile pairs, keep a set of key tiles per query
     tile (top-k, cumulative mass, a caller's fixed block mask, or the pruned-query variant);
  3. fine stage: softmax attention over the kept pairs;
  4. gather the output back to raster order.
"""
from __future__ import annotations

import numpy as np

from . import attention, bsa, pool, select, tiling


def as_f64(x) -> np.ndarray:
    """Exact upcast of a bf16/fp32 torch tensor or numpy array to a float64 numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def coarse_select(qt, kt, vc, mode: str, *, k: int = 0, scale: float = 1.0, tau: float = 0.9,
                  min_k: int = 1, cos_thresh: float = 0.95, mask=None, keep_ratio=None) -> dict:
    """Stage 2 on tile-ordered tensors. Returns a dict with ``sets`` and the intermediates.

    In ``"bsa"`` mode a ``keep_ratio`` selects the ratio form of the query pruning (a fixed count
    of kept rows per block) instead of the cosine threshold."""
    res: dict = {}
    if mode == "mask":
        res["sets"] = select.map_to_sets(np.asarray(mask))
        return res
    pk = pool.tile_mean_pool(kt, vc)
    res["pk"] = pk
    if mode == "bsa":
        if keep_ratio is not None:
            keep, src, cosm = bsa.prune_queries_ratio(qt, keep_ratio)
        else:
            keep, src, cosm = bsa.prune_queries(qt, cos_thresh)
        pq = bsa.pooled_kept_queries(qt, keep)
        res.update(keep=keep, src=src, cos=cosm)
    else:
        pq = pool.tile_mean_pool(qt, vc)
    res["pq"] = pq
    S = select.tile_scores(pq, pk)
    res["S"] = S
    if mode == "topk":
        res["sets"] = select.select_topk(S, k)
    elif mode in ("mass", "bsa"):
        res["sets"] = select.select_mass(S, scale, tau, min_k)
    else:
        raise ValueError(mode)
    return res


def forward(q, k, v, T: int, H: int, W: int, mode: str, *, scale: float, topk: int = 0,
            tau: float = 0.9, min_k: int = 1, cos_thresh: float = 0.95, mask=None,
            q_tiles=None, keep_ratio=None) -> dict:
    """Raster ``[B, L, heads, D]`` Q, K, V -> raster output plus every intermediate (fp64)."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    vc = tiling.variable_block_sizes(T, H, W)
    qt = tiling.tile_scatter(q, T, H, W)
    kt = tiling.tile_scatter(k, T, H, W)
    vt = tiling.tile_scatter(v, T, H, W)
    res = coarse_select(qt, kt, vc, mode, k=topk, scale=scale, tau=tau, min_k=min_k,
                        cos_thresh=cos_thresh, mask=mask, keep_ratio=keep_ratio)
    ot = attention.block_sparse_attention(qt, kt, vt, vc, res["sets"], scale,
                                          keep=res.get("keep"), src=res.get("src"),
                                          q_tiles=q_tiles)
    res.update(vc=vc, qt=qt, kt=kt, vt=vt, ot=ot, o=tiling.tile_gather(ot, T, H, W))
    return res
