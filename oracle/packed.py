"""Oracle: packed multi-region sequences with tiles of 64 or 128 tokens (fp64 / integer, plain loops).

Sources:
* ``video_sparse_attn_h3`` page (FastVideo API docs), ``build()``: a packed sequence is listed in
  packed order; an integer is a dense segment's row count (segments without rows are dropped), a
  ``(t, h, w)`` triple is the latent shape of a video region, which the patch size must divide
  (positive multiples only) and which becomes a token grid of ``(t/pt, h/ph, w/pw)``; at least one
  region is required; the last region is the generated video and follows ``VSA_sparsity``, every
  earlier one is a reference video that keeps ``ref_keep_rate`` of its tiles (required when there
  are reference regions); compete mode (``exempt=False``) allows the generated region only; a
  sparsity of zero or below keeps every region dense; the tile size must be one of the tile-shape
  table's sizes; the metadata records ``num_prefix_tiles``, ``num_video_tiles``,
  ``video_tile_spans`` and one sparsity per span.
* ``video_sparse_attn_h3`` page, ``tile()``: every packed row goes to one slot of a padded buffer
  of ``n_tiles * tile_elems`` rows whose pad positions stay zero; tile 64 and tile 128 exist.
* ``bsa_attn`` page, ``get_tile_partition_indices``, and the ``video_sparse_attn`` section's
  ``construct_variable_block_sizes``: how one video region is cut into tiles and how many valid
  tokens each tile holds.
* ``fastvideo.attention.backends`` page, ``sla.get_block_map``: ``min(K, int(ratio * K))`` tiles of
  a candidate set of ``K`` are kept, by pooled score.

Readings taken where the pages are silent (the helper bodies are not printed):
* P1 buffer order: the dense segments' tiles come first (they are the ``num_prefix_tiles``), each
  dense segment cut into consecutive runs of ``tile_elems`` rows with a partial last run, segments
  in packed order; the video regions' tiles follow in packed order, each region tiled exactly as a
  single video. Valid tokens fill the first ``vc`` slots of a tile.
* P2 tile shapes: 64 tokens as ``(4, 4, 4)``; 128 tokens as ``(4, 4, 8)`` (the table's entries are
  not printed; every function takes the shape as an argument).
* P3 selection, exempt mode: every query tile keeps every prefix tile; a prefix query tile keeps
  every tile; a video query tile keeps, separately inside each region ``r``, the
  ``min(n_r, int(keep_r * n_r))`` tiles of that region with the highest scores, ``keep_r = 1 -
  sparsity_r`` (ties: lower index). Compete mode: every query tile keeps the
  ``min(n, int(keep * n))`` highest-scoring tiles among all ``n`` tiles. A dense layer keeps every
  tile for every query tile.
* P4 attention over the buffer is the single-video one: one softmax over the valid keys of the kept
  tiles; pad query rows output zero.
"""
from __future__ import annotations

import math

import numpy as np

from . import tiling

TILE_SHAPES = {64: (4, 4, 4), 128: (4, 4, 8)}


def token_segments(packed_segments, patch) -> list:
    """Latent segments -> token segments (dense row counts and ``(T, H, W)`` token grids).

    Raises ``ValueError`` for a region not divisible by the patch and when no region is left."""
    out = []
    for seg in packed_segments:
        if isinstance(seg, tuple):
            if any(int(v) <= 0 or int(v) % int(p) for v, p in zip(seg, patch)):
                raise ValueError(f"region {seg} is not a positive multiple of patch {tuple(patch)}")
            out.append(tuple(int(v) // int(p) for v, p in zip(seg, patch)))
        elif int(seg) > 0:
            out.append(int(seg))
    if not any(isinstance(s, tuple) for s in out):
        raise ValueError("a packed sequence needs at least one video region")
    return out


def span_keep_rates(n_regions: int, sparsity: float, ref_keep_rate, exempt: bool) -> list:
    """Keep rate of every region (reference regions first, the generated one last)."""
    if n_regions > 1:
        if ref_keep_rate is None:
            raise ValueError("reference-video regions need ref_keep_rate")
        if not exempt:
            raise ValueError("compete mode supports the generated-video region only")
    if float(sparsity) <= 0.0:
        return [1.0] * n_regions
    refs = [] if n_regions == 1 else [float(ref_keep_rate)] * (n_regions - 1)
    return refs + [1.0 - float(sparsity)]


def packed_geometry(segs, tile_shape) -> dict:
    """Tile geometry of a packed sequence of token segments (reading P1).

    Returns ``slot_row`` (``[n_tiles * E]``: the packed row held by each buffer slot, -1 for a
    pad), ``vc`` (valid tokens per tile), ``n_prefix`` (dense tiles), ``spans`` (``[start, end)``
    tile range of every region, in packed order), ``rows`` (packed length) and ``E``."""
    E = int(np.prod(tile_shape))
    starts = []
    off = 0
    for s in segs:
        starts.append(off)
        off += s if isinstance(s, int) else s[0] * s[1] * s[2]
    tiles = []  # per tile: list of packed rows in slot order
    for s, st in zip(segs, starts):
        if isinstance(s, int):
            for a in range(0, s, E):
                tiles.append([st + r for r in range(a, min(a + E, s))])
    n_prefix = len(tiles)
    spans = []
    for s, st in zip(segs, starts):
        if isinstance(s, tuple):
            T, H, W = s
            order = tiling.tile_partition_indices(T, H, W, tile_shape)
            vcs = tiling.variable_block_sizes(T, H, W, tile_shape)
            first = len(tiles)
            k = 0
            for n in vcs:
                tiles.append([st + int(order[k + j]) for j in range(int(n))])
                k += int(n)
            spans.append((first, len(tiles)))
    slot_row = np.full(len(tiles) * E, -1, dtype=np.int64)
    vc = np.zeros(len(tiles), dtype=np.int64)
    for i, rows in enumerate(tiles):
        vc[i] = len(rows)
        slot_row[E * i:E * i + len(rows)] = rows
    return {"slot_row": slot_row, "vc": vc, "n_prefix": n_prefix, "spans": spans, "rows": off, "E": E}


def scatter(x: np.ndarray, geo: dict) -> np.ndarray:
    """Packed ``[B, rows, heads, D]`` -> padded buffer ``[B, n_tiles * E, heads, D]``, pads zero."""
    B, L, nh, D = x.shape
    assert L == geo["rows"]
    sr = geo["slot_row"]
    y = np.zeros((B, sr.shape[0], nh, D), dtype=x.dtype)
    for slot in range(sr.shape[0]):
        if sr[slot] >= 0:
            y[:, slot] = x[:, sr[slot]]
    return y


def gather(y: np.ndarray, geo: dict) -> np.ndarray:
    """Padded buffer -> packed rows (pads dropped)."""
    B, _, nh, D = y.shape
    x = np.zeros((B, geo["rows"], nh, D), dtype=y.dtype)
    sr = geo["slot_row"]
    for slot in range(sr.shape[0]):
        if sr[slot] >= 0:
            x[:, sr[slot]] = y[:, slot]
    return x


def select(S: np.ndarray, geo: dict, keep_rates, exempt: bool = True, dense: bool = False) -> list:
    """Kept key tiles per query tile of ``S [B, heads, nT, nT]`` (reading P3): nested lists of
    ascending int64 arrays."""
    nT = S.shape[-1]
    n_prefix = geo["n_prefix"]
    spans = geo["spans"]

    def top(row, lo, hi, rate):
        n = hi - lo
        k = min(n, int(rate * n))
        order = sorted(range(lo, hi), key=lambda j: (-row[j], j))
        return order[:k]

    def row_sets(row, i):
        if dense:
            return np.arange(nT, dtype=np.int64)
        if not exempt:
            return np.asarray(sorted(top(row, 0, nT, keep_rates[-1])), dtype=np.int64)
        if i < n_prefix:
            return np.arange(nT, dtype=np.int64)
        kept = list(range(n_prefix))
        for (lo, hi), rate in zip(spans, keep_rates):
            kept += top(row, lo, hi, rate)
        return np.asarray(sorted(kept), dtype=np.int64)

    return [[[row_sets(S[b, h, i].astype(np.float64), i) for i in range(nT)]
             for h in range(S.shape[1])] for b in range(S.shape[0])]


def tile_count_check(segs, tile_shape) -> int:
    """Number of tiles by counting alone (for cross-checks): dense runs plus region tile grids."""
    E = int(np.prod(tile_shape))
    n = 0
    for s in segs:
        if isinstance(s, int):
            n += math.ceil(s / E)
        else:
            a, b, c = tiling.tile_counts(*s, tile_shape)
            n += a * b * c
    return n
