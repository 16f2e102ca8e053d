"""Pins of the packed multi-region oracle (video_sparse_attn_h3 page, build() and tile()).

The geometry is checked against two hand-worked fixtures (tests/golden/packed_*.txt), the
single-video tiling it must reduce to, and counting; selection against hand-worked rows, the plain
top-k it reduces to, and brute-force properties; pooling and attention with 128-token tiles
against means and masked softmax attention computed over the packed rows by torch in fp64.
"""
import os

import numpy as np
import pytest
import torch

from oracle import attention, packed, pool, select, tiling

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_fixture(name):
    out = {"tiles": {}}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == "tile":
            rows = []
            for tok in parts[3:]:
                if "-" in tok:
                    a, b = tok.split("-")
                    rows += list(range(int(a), int(b) + 1))
                else:
                    rows.append(int(tok))
            out["tiles"][int(parts[1])] = rows
        else:
            out[parts[0]] = [int(v) for v in parts[1:]]
    return out


def check_against_fixture(geo, fx):
    E = geo["E"]
    assert geo["rows"] == fx["rows"][0]
    assert geo["n_prefix"] == fx["n_prefix"][0]
    assert [tuple(s) for s in geo["spans"]] == [tuple(fx["spans"][i:i + 2])
                                                for i in range(0, len(fx["spans"]), 2)]
    assert geo["vc"].tolist() == fx["vc"]
    for t, rows in fx["tiles"].items():
        assert geo["slot_row"][E * t:E * t + len(rows)].tolist() == rows
        assert (geo["slot_row"][E * t + len(rows):E * (t + 1)] == -1).all()


def test_geometry_mixed_tile64_fixture():
    segs = packed.token_segments([5, (8, 4, 8), 70], (2, 1, 2))
    assert segs == [5, (4, 4, 4), 70]
    geo = packed.packed_geometry(segs, packed.TILE_SHAPES[64])
    check_against_fixture(geo, read_fixture("packed_mixed_tile64.txt"))


def test_geometry_tile128_fixture():
    segs = packed.token_segments([130, (5, 4, 9)], (1, 1, 1))
    geo = packed.packed_geometry(segs, packed.TILE_SHAPES[128])
    check_against_fixture(geo, read_fixture("packed_tile128.txt"))


@pytest.mark.parametrize("grid", [(4, 8, 8), (5, 6, 7), (21, 30, 52)])
def test_single_region_reduces_to_single_video_tiling(grid):
    geo = packed.packed_geometry([grid], tiling.TILE)
    T, H, W = grid
    pos = tiling.padded_positions(T, H, W)
    slot_row = np.full(tiling.padded_length(T, H, W), -1)
    slot_row[pos] = np.arange(T * H * W)
    assert np.array_equal(geo["slot_row"], slot_row)
    assert np.array_equal(geo["vc"], tiling.variable_block_sizes(T, H, W))
    assert geo["n_prefix"] == 0 and geo["spans"] == [(0, len(geo["vc"]))]


@pytest.mark.parametrize("E", [64, 128])
def test_geometry_is_a_bijection_and_counts_agree(E):
    segs = [3, (5, 9, 6), 200, (2, 3, 17), 64, (4, 4, 8)]
    geo = packed.packed_geometry(segs, packed.TILE_SHAPES[E])
    sr = geo["slot_row"]
    assert len(geo["vc"]) == packed.tile_count_check(segs, packed.TILE_SHAPES[E])
    assert sorted(sr[sr >= 0].tolist()) == list(range(geo["rows"]))
    assert geo["vc"].sum() == geo["rows"]
    for t in range(len(geo["vc"])):  # valid slots first, then pads
        blk = sr[E * t:E * (t + 1)]
        assert (blk[:geo["vc"][t]] >= 0).all() and (blk[geo["vc"][t]:] == -1).all()
    # dense tiles first: 1 + 4 (200 rows at 64) or 1 + 2 (at 128) plus one for the 64-row segment
    assert geo["n_prefix"] == (1 + 4 + 1 if E == 64 else 1 + 2 + 1)
    assert len(geo["spans"]) == 3 and geo["spans"][0][0] == geo["n_prefix"]
    assert geo["spans"][-1][1] == len(geo["vc"])


def test_scatter_gather_round_trip_and_zero_pads():
    rng = np.random.default_rng(3)
    segs = [7, (3, 5, 6), 70]
    for E in (64, 128):
        geo = packed.packed_geometry(segs, packed.TILE_SHAPES[E])
        x = rng.standard_normal((2, geo["rows"], 3, 8))
        y = packed.scatter(x, geo)
        pads = geo["slot_row"] < 0
        assert (y[:, pads] == 0).all()
        assert np.array_equal(packed.gather(y, geo), x)


def test_token_segments_and_keep_rates_contract():
    with pytest.raises(ValueError):
        packed.token_segments([(5, 4, 9)], (2, 1, 1))  # 5 is not a multiple of 2
    with pytest.raises(ValueError):
        packed.token_segments([(0, 4, 8)], (1, 1, 1))
    with pytest.raises(ValueError):
        packed.token_segments([10, 0], (1, 1, 1))  # no region
    assert packed.token_segments([0, 12, (2, 2, 2)], (1, 1, 1)) == [12, (2, 2, 2)]
    with pytest.raises(ValueError):
        packed.span_keep_rates(2, 0.9, None, True)
    with pytest.raises(ValueError):
        packed.span_keep_rates(2, 0.9, 0.5, False)
    assert packed.span_keep_rates(3, 0.875, 0.25, True) == [0.25, 0.25, 0.125]
    assert packed.span_keep_rates(3, 0.0, 0.25, True) == [1.0, 1.0, 1.0]
    assert packed.span_keep_rates(1, 0.75, None, False) == [0.25]


def test_select_hand_worked_row():
    # One prefix tile (0); region A = tiles 1..4 at keep 0.5 (int(2.0) = 2 tiles); region B =
    # tiles 5..7 at keep 0.4 (int(1.2) = 1 tile). Scores: A's best two are tiles 3 (0.9) and 1 (0.5,
    # tied with tile 4 -> the lower index wins); B's best is tile 6.
    row = np.array([-5.0, 0.5, 0.1, 0.9, 0.5, 0.2, 0.7, 0.3])
    S = row[None, None, None, :].repeat(8, axis=2)
    geo = {"n_prefix": 1, "spans": [(1, 5), (5, 8)]}
    sets = packed.select(S, geo, [0.5, 0.4], exempt=True)
    assert sets[0][0][0].tolist() == list(range(8))  # a prefix query tile keeps everything
    assert sets[0][0][3].tolist() == [0, 1, 3, 6]
    # compete: one top-k over all 8 tiles at the last keep rate: int(0.4 * 8) = 3 tiles
    assert packed.select(S, geo, [0.5, 0.4], exempt=False)[0][0][2].tolist() == [1, 3, 6]
    assert packed.select(S, geo, [0.5, 0.4], dense=True)[0][0][5].tolist() == list(range(8))


def test_select_single_region_reduces_to_topk():
    rng = np.random.default_rng(5)
    S = rng.standard_normal((2, 3, 40, 40))
    geo = {"n_prefix": 0, "spans": [(0, 40)]}
    sets = packed.select(S, geo, [0.3])
    ref = select.select_topk(S, int(0.3 * 40))
    for b in range(2):
        for h in range(3):
            for i in range(40):
                assert np.array_equal(sets[b][h][i], ref[b][h][i])


def test_select_multi_region_properties():
    rng = np.random.default_rng(11)
    geo = packed.packed_geometry([30, (4, 8, 8), 10, (8, 8, 8), (4, 4, 12)], packed.TILE_SHAPES[64])
    nT = len(geo["vc"])
    S = np.round(rng.standard_normal((1, 2, nT, nT)), 1)  # rounded: many ties
    rates = [0.3, 0.3, 0.6]
    sets = packed.select(S, geo, rates)
    npre = geo["n_prefix"]
    for h in range(2):
        for i in range(nT):
            kept = set(sets[0][h][i].tolist())
            if i < npre:
                assert kept == set(range(nT))
                continue
            assert set(range(npre)) <= kept
            for (lo, hi), r in zip(geo["spans"], rates):
                ks = [j for j in range(lo, hi) if j in kept]
                drop = [j for j in range(lo, hi) if j not in kept]
                assert len(ks) == min(hi - lo, int(r * (hi - lo)))
                row = S[0, h, i]
                for a in ks:  # every kept tile outranks every dropped one of its region
                    for d in drop:
                        assert row[a] > row[d] or (row[a] == row[d] and a < d)


def masked_reference(x_q, x_k, x_v, allowed, scale):
    """Softmax attention over packed rows with a boolean [rows, rows] mask, torch fp64."""
    q = torch.from_numpy(x_q).double()
    k = torch.from_numpy(x_k).double()
    v = torch.from_numpy(x_v).double()
    m = torch.from_numpy(allowed)
    out = torch.zeros_like(q)
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            rows = m.any(dim=1)
            o = torch.nn.functional.scaled_dot_product_attention(
                q[b, :, h][None], k[b, :, h][None], v[b, :, h][None], attn_mask=m[None], scale=scale)
            out[b, rows, h] = o[0][rows]
    return out.numpy()


@pytest.mark.parametrize("E", [64, 128])
def test_packed_attention_matches_masked_softmax(E):
    rng = np.random.default_rng(17 + E)
    segs = [20, (4, 6, 9), 90, (2, 4, 8)]
    geo = packed.packed_geometry(segs, packed.TILE_SHAPES[E])
    nT = len(geo["vc"])
    B, nh, D = 1, 2, 16
    xq, xk, xv = (rng.standard_normal((B, geo["rows"], nh, D)) for _ in range(3))
    scale = D ** -0.5
    qt, kt, vt = (packed.scatter(t, geo) for t in (xq, xk, xv))
    pq = pool.tile_mean_pool(qt, geo["vc"], E)
    pk = pool.tile_mean_pool(kt, geo["vc"], E)
    sets = packed.select(select.tile_scores(pq, pk), geo, [0.5, 0.5])
    out = packed.gather(attention.block_sparse_attention(qt, kt, vt, geo["vc"], sets, scale,
                                                         tile_elems=E), geo)
    tile_of = np.empty(geo["rows"], dtype=np.int64)
    sr = geo["slot_row"]
    tile_of[sr[sr >= 0]] = np.nonzero(sr >= 0)[0] // E
    for h in range(nh):
        allowed = np.zeros((geo["rows"], geo["rows"]), dtype=bool)
        for r in range(geo["rows"]):
            allowed[r] = np.isin(tile_of, sets[0][h][tile_of[r]])
        ref = masked_reference(xq[:, :, h:h + 1], xk[:, :, h:h + 1], xv[:, :, h:h + 1], allowed, scale)
        np.testing.assert_allclose(out[:, :, h:h + 1], ref, rtol=1e-10, atol=1e-12)
    assert nT == len(geo["vc"])


def test_pool_tile128_is_the_mean_of_each_tiles_rows():
    rng = np.random.default_rng(2)
    fx = read_fixture("packed_tile128.txt")
    geo = packed.packed_geometry([130, (5, 4, 9)], packed.TILE_SHAPES[128])
    x = rng.standard_normal((2, geo["rows"], 3, 8))
    pooled = pool.tile_mean_pool(packed.scatter(x, geo), geo["vc"], 128)
    for t, rows in fx["tiles"].items():
        np.testing.assert_allclose(pooled[:, :, t], x[:, rows].mean(axis=1), rtol=1e-12)
