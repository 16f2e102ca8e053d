"""CPU pins of the oracle's tile geometry, scatter and gather.

Each check uses a formulation other than the oracle's nested loops: a closed form for divisible
grids, a sort by tile key for ragged ones, hand-worked golden fixtures, and invariants.
"""
import os

import numpy as np
import pytest

from oracle import tiling

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [list(map(int, ln.split())) for ln in f if ln.strip() and not ln.startswith("#")]


def test_golden_tiny_tile_order():
    rows = _read_rows("tiny_4x8x8_tile_order.txt")
    want = np.concatenate([np.asarray(r) for r in rows])
    np.testing.assert_array_equal(tiling.tile_partition_indices(4, 8, 8), want)


@pytest.mark.parametrize("grid", [(4, 8, 8), (8, 4, 12), (16, 32, 56), (4, 4, 4)])
def test_closed_form_divisible(grid):
    T, H, W = grid
    nh, nw = H // 4, W // 4
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    tile = ((t // 4) * nh + h // 4) * nw + w // 4
    slot = (t % 4) * 16 + (h % 4) * 4 + (w % 4)
    np.testing.assert_array_equal(tiling.padded_positions(T, H, W), (64 * tile + slot).reshape(-1))
    assert tiling.padded_length(T, H, W) == T * H * W


@pytest.mark.parametrize("grid", [(1, 1, 1), (3, 5, 7), (5, 4, 9), (21, 30, 52), (6, 9, 2)])
def test_partition_matches_sort_by_tile_key(grid):
    T, H, W = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    keys = [x.reshape(-1) for x in (w, h, t, w // 4, h // 4, t // 4)]  # lexsort: last key primary
    want = np.lexsort(keys)
    np.testing.assert_array_equal(tiling.tile_partition_indices(T, H, W), want)


@pytest.mark.parametrize("grid", [(3, 5, 7), (21, 30, 52), (4, 8, 8)])
def test_reverse_is_inverse(grid):
    fwd = tiling.tile_partition_indices(*grid)
    rev = tiling.reverse_tile_partition_indices(*grid)
    np.testing.assert_array_equal(rev[fwd], np.arange(len(fwd)))
    np.testing.assert_array_equal(fwd[rev], np.arange(len(fwd)))


@pytest.mark.parametrize("grid", [(1, 1, 1), (3, 5, 7), (5, 4, 9), (21, 30, 52), (16, 32, 56)])
def test_valid_counts_by_counting(grid):
    T, H, W = grid
    nt, nh, nw = tiling.tile_counts(T, H, W)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    tid = ((t // 4) * nh + h // 4) * nw + w // 4
    want = np.bincount(tid.reshape(-1), minlength=nt * nh * nw)
    vc = tiling.variable_block_sizes(T, H, W)
    np.testing.assert_array_equal(vc, want)
    assert vc.sum() == T * H * W


def test_golden_ragged_valid_counts():
    vc = tiling.variable_block_sizes(21, 30, 52)
    assert len(vc) == 624
    rows = _read_rows("ragged_21x30x52_valid_counts.txt")
    vals, counts = np.unique(vc, return_counts=True)
    assert {int(a): int(b) for a, b in zip(vals, counts)} == {r[0]: r[1] for r in rows}
    assert vc.min() == 8


@pytest.mark.parametrize("grid", [(3, 5, 7), (5, 4, 9), (4, 8, 8), (9, 6, 10)])
def test_scatter_gather_roundtrip_and_zero_pads(grid):
    T, H, W = grid
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, T * H * W, 3, 8)) + 5.0  # no zeros among valid rows
    y = tiling.tile_scatter(x, T, H, W)
    assert y.shape == (2, tiling.padded_length(T, H, W), 3, 8)
    np.testing.assert_array_equal(tiling.tile_gather(y, T, H, W), x)
    valid = tiling.valid_slot_mask(T, H, W)
    assert np.all(y[:, ~valid] == 0.0)
    assert np.all(y[:, valid] != 0.0)
    assert valid.sum() == T * H * W
    # every raster token lands in the tile that contains it, in in-tile raster order
    pos = tiling.padded_positions(T, H, W)
    assert len(np.unique(pos)) == len(pos)
    nt, nh, nw = tiling.tile_counts(T, H, W)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    tid = (((t // 4) * nh + h // 4) * nw + w // 4).reshape(-1)
    np.testing.assert_array_equal(pos // 64, tid)
    for i in range(nt * nh * nw):
        members = np.nonzero(tid == i)[0]  # ascending raster ids = in-tile raster order
        np.testing.assert_array_equal(pos[members] % 64, np.arange(len(members)))
