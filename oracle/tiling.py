"""Oracle: 3D tile geometry, tile scatter and untile (fp64 / integer, plain loops).

Sources:
* ``bsa_attn`` page (FastVideo API docs), ``get_tile_partition_indices``: tiles are visited
  t-tile, then h-tile, then w-tile (outermost to innermost); inside a tile, tokens keep raster
  (t, h, w) order; a partial edge tile contributes only the tokens that exist.
* ``bsa_attn`` page, ``get_reverse_tile_partition_indices``: the inverse map is the argsort of
  the forward map.
* ``fastvideo.attention.backends`` page, ``video_sparse_attn.construct_variable_block_sizes``:
  the number of valid tokens per tile; the last tile along a dimension holds
  ``dim - (n - 1) * tile`` tokens along it.
* ``video_sparse_attn_h3`` page, ``tile()``: rows are scattered into a padded tile buffer whose
  pad positions stay zero.

Reading taken where the pages are silent: inside the padded buffer, tile ``i`` owns rows
``[64 i, 64 i + 64)``; its valid tokens fill slots ``0 .. vc_i - 1`` in the in-tile raster order
above and the remaining slots are zero.
"""
from __future__ import annotations

import math

import numpy as np

TILE = (4, 4, 4)
TILE_ELEMS = 64


def tile_counts(T: int, H: int, W: int, tile=TILE) -> tuple[int, int, int]:
    return (math.ceil(T / tile[0]), math.ceil(H / tile[1]), math.ceil(W / tile[2]))


def tile_partition_indices(T: int, H: int, W: int, tile=TILE) -> np.ndarray:
    """Raster token ids listed in tile-contiguous order (length T*H*W).

    Visit every tile in (t-tile, h-tile, w-tile) order and, inside it, every existing token in raster
    order; concatenate."""
    ts, hs, ws = tile
    order: list[int] = []
    for a in range(math.ceil(T / ts)):
        for b in range(math.ceil(H / hs)):
            for c in range(math.ceil(W / ws)):
                for t in range(a * ts, min(a * ts + ts, T)):
                    for h in range(b * hs, min(b * hs + hs, H)):
                        for w in range(c * ws, min(c * ws + ws, W)):
                            order.append((t * H + h) * W + w)
    return np.asarray(order, dtype=np.int64)


def reverse_tile_partition_indices(T: int, H: int, W: int, tile=TILE) -> np.ndarray:
    """Position of each raster token in the tile-contiguous order: argsort of the forward map."""
    return np.argsort(tile_partition_indices(T, H, W, tile), kind="stable")


def variable_block_sizes(T: int, H: int, W: int, tile=TILE) -> np.ndarray:
    """Valid (non-pad) token count of every tile, flattened in (t-tile, h-tile, w-tile) order."""

    def sizes(n_len: int, edge: int) -> list[int]:
        n = math.ceil(n_len / edge)
        out = [edge] * n
        rem = n_len - (n - 1) * edge
        out[-1] = rem if rem > 0 else edge
        return out

    st, sh, sw = sizes(T, tile[0]), sizes(H, tile[1]), sizes(W, tile[2])
    return np.asarray([x * y * z for x in st for y in sh for z in sw], dtype=np.int64)


def padded_positions(T: int, H: int, W: int, tile=TILE) -> np.ndarray:
    """Row of the padded tile buffer that each raster token lands in (length T*H*W).

    Tile ``i`` owns rows ``64 i ..``; its tokens take the slots in the order of
    ``tile_partition_indices``."""
    order = tile_partition_indices(T, H, W, tile)
    vc = variable_block_sizes(T, H, W, tile)
    pos = np.empty(T * H * W, dtype=np.int64)
    k = 0
    for i, n in enumerate(vc):
        for s in range(int(n)):
            pos[order[k]] = TILE_ELEMS * i + s
            k += 1
    assert k == T * H * W
    return pos


def padded_length(T: int, H: int, W: int, tile=TILE) -> int:
    a, b, c = tile_counts(T, H, W, tile)
    return TILE_ELEMS * a * b * c


def tile_scatter(x: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    """Raster ``[B, L, heads, D]`` -> padded tile order ``[B, 64*nT, heads, D]``; pads are zero."""
    B, L, nh, D = x.shape
    assert L == T * H * W
    y = np.zeros((B, padded_length(T, H, W), nh, D), dtype=x.dtype)
    y[:, padded_positions(T, H, W)] = x
    return y


def tile_gather(y: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    """Padded tile order ``[B, 64*nT, heads, D]`` -> raster ``[B, L, heads, D]`` (pads dropped)."""
    return y[:, padded_positions(T, H, W)].copy()


def valid_slot_mask(T: int, H: int, W: int) -> np.ndarray:
    """Boolean ``[64*nT]``: True where a padded row holds a real token."""
    vc = variable_block_sizes(T, H, W)
    m = np.zeros(TILE_ELEMS * len(vc), dtype=bool)
    for i, n in enumerate(vc):
        m[TILE_ELEMS * i:TILE_ELEMS * i + int(n)] = True
    return m
