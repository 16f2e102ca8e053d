"""Pins of the oracle's BSA ratio mode (a fixed count of kept query rows per 64-row block).

FastVideo API docs, bsa_attn page, BSAAttentionImpl.forward: the query pruning helper takes
``query_keep_ratio`` and returns a ``keep_size``. Reading: ``keep_size = max(1, floor(64 * ratio))``
rows per block, the rows least similar to the block mean (lowest cosine, lowest index on ties);
pruned rows copy their most similar kept row, as in the threshold mode.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import bsa


def _fan(n: int = 64, delta: float = 0.02, seed: int = 5) -> tuple[np.ndarray, np.ndarray]:
    """2-D rows at angles (i - (n-1)/2) * delta with magnitudes symmetric about the middle row: the
    block mean points along +x, so each row's cosine to it is cos(angle) in closed form."""
    rng = np.random.default_rng(seed)
    half = rng.uniform(0.5, 2.0, size=n // 2)
    mag = np.concatenate([half, half[::-1]])
    ang = (np.arange(n) - (n - 1) / 2) * delta
    return np.stack([mag * np.cos(ang), mag * np.sin(ang)], axis=1), ang


@pytest.mark.parametrize("ratio,size", [(1.0, 64), (0.5, 32), (0.25, 16), (0.3, 19), (0.2, 12),
                                        (1e-3, 1), (0.0156, 1), (1 / 64, 1), (0.99, 63)])
def test_keep_size(ratio, size):
    assert bsa.keep_size_for_ratio(ratio) == size


def test_fan_keeps_the_widest_angles_and_copies_the_nearest_kept_row():
    rows, ang = _fan()
    keep, src, cm = bsa.prune_block_ratio(rows, 0.25)  # 16 rows: 8 at each end of the fan
    np.testing.assert_allclose(cm, np.cos(ang), atol=1e-12)
    want = np.zeros(64, dtype=bool)
    want[:8] = True
    want[56:] = True
    np.testing.assert_array_equal(keep, want)
    for i in range(64):
        if want[i]:
            assert src[i] == i
        else:
            assert src[i] == (7 if i < 32 else 56)  # the kept row at the nearest angle


def test_ratio_one_keeps_every_row():
    rows = np.random.default_rng(1).normal(size=(64, 16))
    keep, src, _ = bsa.prune_block_ratio(rows, 1.0)
    assert keep.all()
    np.testing.assert_array_equal(src, np.arange(64))


def test_identical_rows_keep_the_lowest_indices():
    rows = np.tile(np.random.default_rng(2).normal(size=(1, 16)), (64, 1))
    keep, src, _ = bsa.prune_block_ratio(rows, 0.125)
    np.testing.assert_array_equal(np.nonzero(keep)[0], np.arange(8))
    assert (src[8:] == 0).all()  # every kept row is equally similar: the lowest index wins


def test_random_blocks_keep_exactly_keep_size_least_similar_rows():
    rng = np.random.default_rng(3)
    for ratio in (0.1, 0.4, 0.77):
        rows = rng.normal(size=(64, 24)) + rng.normal(size=(1, 24))
        keep, src, cm = bsa.prune_block_ratio(rows, ratio)
        assert keep.sum() == bsa.keep_size_for_ratio(ratio)
        assert cm[keep].max() <= cm[~keep].min()
        # a pruned row's source is a kept row at least as similar as every other kept row
        nrm = np.linalg.norm(rows, axis=1)
        kept = np.nonzero(keep)[0]
        for i in np.nonzero(~keep)[0]:
            c = rows[kept] @ rows[i] / (nrm[kept] * nrm[i])
            assert keep[src[i]]
            assert np.isclose(c[list(kept).index(src[i])], c.max())


def test_ratio_mode_over_tiles_matches_per_block_calls():
    rng = np.random.default_rng(4)
    qt = rng.normal(size=(2, 64 * 3, 2, 8))
    keep, src, cm = bsa.prune_queries_ratio(qt, 0.5)
    for b in range(2):
        for h in range(2):
            for i in range(3):
                k1, s1, c1 = bsa.prune_block_ratio(qt[b, 64 * i:64 * (i + 1), h], 0.5)
                np.testing.assert_array_equal(keep[b, h, i], k1)
                np.testing.assert_array_equal(src[b, h, i], s1)


def test_pipeline_ratio_one_is_mass_selection_over_all_rows():
    """Keep ratio 1 keeps every query row, so the BSA chain (pooled kept queries, mass selection,
    attention with every row its own source) reduces to plain mass selection and attention."""
    from oracle import pipeline

    rng = np.random.default_rng(7)
    T, H, W = 4, 8, 8  # no pads: the ratio mode needs L == 64 * nT
    q, k, v = (rng.normal(size=(1, T * H * W, 2, 16)) for _ in range(3))
    bsa_res = pipeline.forward(q, k, v, T, H, W, "bsa", scale=0.25, tau=0.8, keep_ratio=1.0)
    mass_res = pipeline.forward(q, k, v, T, H, W, "mass", scale=0.25, tau=0.8)
    assert bsa_res["keep"].all()
    np.testing.assert_allclose(bsa_res["pq"], mass_res["pq"], rtol=1e-12, atol=1e-12)
    for b in range(1):
        for h in range(2):
            for i in range(len(mass_res["sets"][b][h])):
                np.testing.assert_array_equal(bsa_res["sets"][b][h][i], mass_res["sets"][b][h][i])
    np.testing.assert_allclose(bsa_res["o"], mass_res["o"], rtol=1e-12, atol=1e-12)
