"""Oracle: mean pooling of each 64-token tile (fp64).

Source: ``fastvideo.attention.backends`` page, ``sla.mean_pool`` (one mean per block along the
sequence) as used by ``sla.get_block_map`` for both queries and keys.

Reading taken where the pages are silent: a partial tile is averaged over its valid tokens only
(divide by the tile's valid count, not by 64); pad rows never enter the mean.
"""
from __future__ import annotations

import numpy as np

TILE_ELEMS = 64


def tile_mean_pool(y: np.ndarray, vc: np.ndarray, tile_elems: int = TILE_ELEMS) -> np.ndarray:
    """Padded tile order ``[B, E*nT, heads, D]`` -> pooled ``[B, heads, nT, D]`` (fp64); ``E`` =
    ``tile_elems`` rows per tile (64, or 128 for the packed sequences' large tile)."""
    B, Lp, nh, D = y.shape
    E = int(tile_elems)
    nT = Lp // E
    assert nT * E == Lp and len(vc) == nT
    out = np.zeros((B, nh, nT, D), dtype=np.float64)
    for i in range(nT):
        n = int(vc[i])
        rows = y[:, E * i:E * i + n].astype(np.float64)  # [B, n, heads, D]
        out[:, :, i, :] = rows.sum(axis=1) / n
    return out
