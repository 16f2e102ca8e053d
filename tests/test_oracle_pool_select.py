"""CPU pins of the oracle's tile pooling and KV tile selection.

Pooling is checked against sums accumulated per raster token with no use of the tile buffer;
selection against brute-force enumeration of subsets, closed-form special cases and invariances.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle import pool, select, tiling


@pytest.mark.parametrize("grid", [(3, 5, 7), (5, 4, 9), (4, 8, 8)])
def test_pool_matches_per_token_accumulation(grid):
    T, H, W = grid
    rng = np.random.default_rng(1)
    B, nh, D = 2, 3, 5
    x = rng.standard_normal((B, T * H * W, nh, D))
    y = tiling.tile_scatter(x, T, H, W)
    got = pool.tile_mean_pool(y, tiling.variable_block_sizes(T, H, W))
    nt, nhh, nw = tiling.tile_counts(T, H, W)
    acc = np.zeros((B, nh, nt * nhh * nw, D))
    cnt = np.zeros(nt * nhh * nw)
    for t in range(T):
        for h in range(H):
            for w in range(W):
                tid = ((t // 4) * nhh + h // 4) * nw + w // 4
                acc[:, :, tid] += x[:, (t * H + h) * W + w]
                cnt[tid] += 1
    np.testing.assert_allclose(got, acc / cnt[None, None, :, None], rtol=1e-13, atol=1e-13)


def test_pool_constant_tile():
    T, H, W = 5, 4, 9
    x = np.full((1, T * H * W, 1, 4), 3.25)
    got = pool.tile_mean_pool(tiling.tile_scatter(x, T, H, W), tiling.variable_block_sizes(T, H, W))
    assert np.all(got == 3.25)


def test_topk_bruteforce_subsets():
    rng = np.random.default_rng(2)
    for nT in (1, 3, 5, 8):
        for k in range(1, nT + 1):
            row = rng.standard_normal(nT)
            best = max(itertools.combinations(range(nT), k), key=lambda c: row[list(c)].sum())
            np.testing.assert_array_equal(select.select_topk_row(row, k), np.array(sorted(best)))


def test_topk_special_cases():
    rng = np.random.default_rng(3)
    S = rng.standard_normal((2, 3, 7, 7))
    for b in range(2):
        for h in range(3):
            for i in range(7):
                np.testing.assert_array_equal(select.select_topk(S, 7)[b][h][i], np.arange(7))
                np.testing.assert_array_equal(select.select_topk(S, 99)[b][h][i], np.arange(7))
                assert select.select_topk(S, 1)[b][h][i].tolist() == [int(np.argmax(S[b, h, i]))]


def test_topk_ties_go_to_lower_index():
    row = np.array([1.0, 5.0, 3.0, 5.0, 3.0, 3.0])
    assert select.select_topk_row(row, 1).tolist() == [1]
    assert select.select_topk_row(row, 3).tolist() == [1, 2, 3]
    assert select.select_topk_row(row, 4).tolist() == [1, 2, 3, 4]


def test_scores_are_pooled_dot_products():
    rng = np.random.default_rng(4)
    pq, pk = rng.standard_normal((1, 2, 6, 9)), rng.standard_normal((1, 2, 6, 9))
    S = select.tile_scores(pq, pk)
    want = torch.einsum("bhid,bhjd->bhij", torch.from_numpy(pq), torch.from_numpy(pk)).numpy()
    np.testing.assert_allclose(S, want, rtol=1e-12, atol=1e-12)


def test_smooth_k_shift_changes_no_selection():
    """Subtracting the sequence mean of K (smooth-k) shifts each score row by a constant."""
    rng = np.random.default_rng(5)
    T, H, W, D = 8, 8, 12, 16
    q = rng.standard_normal((1, T * H * W, 2, D)) + rng.standard_normal((1, 1, 2, D))
    k = rng.standard_normal((1, T * H * W, 2, D)) + 3.0
    vc = tiling.variable_block_sizes(T, H, W)
    pq = pool.tile_mean_pool(tiling.tile_scatter(q, T, H, W), vc)
    pk = pool.tile_mean_pool(tiling.tile_scatter(k, T, H, W), vc)
    pk_s = pool.tile_mean_pool(tiling.tile_scatter(k - k.mean(axis=1, keepdims=True), T, H, W), vc)
    S, S_s = select.tile_scores(pq, pk), select.tile_scores(pq, pk_s)
    for kk in (1, 5, 11):
        a, b = select.select_topk(S, kk), select.select_topk(S_s, kk)
        for h in range(2):
            for i in range(len(vc)):
                np.testing.assert_array_equal(a[0][h][i], b[0][h][i])
    a, b = select.select_mass(S, 0.25, 0.9, 1), select.select_mass(S_s, 0.25, 0.9, 1)
    for h in range(2):
        for i in range(len(vc)):
            np.testing.assert_array_equal(a[0][h][i], b[0][h][i])


def test_mass_bruteforce_minimal_subset():
    rng = np.random.default_rng(6)
    for nT in (2, 4, 7, 8):
        for tau in (0.3, 0.6, 0.9, 0.99):
            row = rng.standard_normal(nT) * 2.0
            p = torch.softmax(torch.from_numpy(0.7 * row), dim=0).numpy()
            best = None
            for m in range(1, nT + 1):
                cands = [c for c in itertools.combinations(range(nT), m) if p[list(c)].sum() >= tau]
                if cands:
                    best = max(cands, key=lambda c: p[list(c)].sum())
                    break
            np.testing.assert_array_equal(select.select_mass_row(row, 0.7, tau, 1),
                                          np.array(sorted(best)))


def test_mass_special_cases():
    rng = np.random.default_rng(7)
    row = rng.standard_normal(9)
    assert select.select_mass_row(row, 0.5, 1.0, 1).tolist() == list(range(9))
    assert select.select_mass_row(row, 0.5, 1e-9, 1).tolist() == [int(np.argmax(row))]
    assert len(select.select_mass_row(row, 0.5, 1e-9, 4)) == 4
    np.testing.assert_array_equal(select.select_mass_row(row, 0.5, 1e-9, 4),
                                  select.select_topk_row(row, 4))
    assert len(select.select_mass_row(row, 0.5, 1e-9, 50)) == 9
    # a uniform row needs ceil(tau * n) tiles
    assert len(select.select_mass_row(np.zeros(10), 1.0, 0.55, 1)) == 6


def test_topk_gap_and_margins():
    row = np.array([4.0, 1.0, 3.0, 2.0])
    g = select.topk_gap(row[None], 2)
    np.testing.assert_allclose(g, [(3.0 - 2.0) / 4.0])
    assert np.isinf(select.topk_gap(row[None], 4)).all()
    m = select.mass_margins(np.zeros(10), 1.0, 0.55, 1)
    assert m["count"] == 6
    np.testing.assert_allclose(m["sum_margin"], 0.05, atol=1e-12)


def test_mass_one_keeps_every_tile_even_when_the_tail_rounds_away():
    # Scores spread so far that the tail probabilities (e^-60, e^-120 relative to the largest) are
    # below fp64's resolution of 1: the rounded running sum reaches 1.0 before them, but each of
    # them is positive, so the exact sum reaches 1 only with the last tile.
    row = np.array([0.0, -60.0, 10.0, -120.0, 5.0])
    assert np.cumsum(select.softmax_row(row)[[2, 4, 0, 1, 3]])[2] >= 1.0  # rounding reaches 1
    np.testing.assert_array_equal(select.select_mass_row(row, 1.0, 1.0, 1), np.arange(5))
    m = select.mass_margins(row, 1.0, 1.0, 1)
    assert m["count"] == 5 and np.isinf(m["cut_gap"])


def test_mass_margins_hand_worked_row():
    # Logits log(p) with p = (0.05, 0.45, 0.15, 0.35) at scale 1: the softmax gives p back. Ranked:
    # 0.45 (tile 1), 0.35 (tile 3), 0.15 (tile 2), 0.05 (tile 0); running sums .45, .80, .95, 1.
    row = np.log(np.array([0.05, 0.45, 0.15, 0.35]))
    # tau = 0.65: the sum first reaches it at the second tile, so tiles {1, 3} are kept; the cut
    # lies between p = 0.35 and p = 0.15, a gap of 0.2 relative to the largest p 0.45 (the gaps
    # one place earlier or later would be 0.1 / 0.45); the sums on either side of the cut are
    # 0.45 and 0.80, at distances 0.20 and 0.15 from tau.
    np.testing.assert_array_equal(select.select_mass_row(row, 1.0, 0.65, 1), [1, 3])
    m = select.mass_margins(row, 1.0, 0.65, 1)
    assert m["count"] == 2
    np.testing.assert_allclose(m["cut_gap"], 0.2 / 0.45, rtol=1e-12)
    np.testing.assert_allclose(m["sum_margin"], 0.15, rtol=1e-9)
    # a floor of 3 tiles moves the cut to between 0.15 and 0.05 and makes the sum irrelevant
    m = select.mass_margins(row, 1.0, 0.65, 3)
    assert m["count"] == 3
    np.testing.assert_allclose(m["cut_gap"], 0.1 / 0.45, rtol=1e-12)
    assert np.isinf(m["sum_margin"])
    # tau = 0.97 needs every tile: no cut at all
    m = select.mass_margins(row, 1.0, 0.97, 1)
    assert m["count"] == 4 and np.isinf(m["cut_gap"])
    # two equal probabilities at the cut: a zero gap flags the row as undecidable
    tie = np.log(np.array([0.3, 0.3, 0.4]))
    m = select.mass_margins(tie, 1.0, 0.5, 1)
    assert m["count"] == 2 and m["cut_gap"] == 0.0


def test_map_set_roundtrip():
    rng = np.random.default_rng(8)
    mask = (rng.random((2, 3, 5, 5)) < 0.4).astype(np.uint8)
    sets = select.map_to_sets(mask)
    np.testing.assert_array_equal(select.sets_to_map(sets, 5), mask)
