"""GPU parity of the packed multi-region path (include/tile3d_packed.h) with the oracle
(oracle/packed.py): scatter / gather bit-exact, pooling to fp32 rounding, per-region selection
exact where the score gap is decisive, attention with the oracle's kept lists fed in directly
(tiles of 64 and 128 rows, dense prefix, two regions, ragged tiles, D = 64 and 128), and the whole
module end to end."""
import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import packed as P
from oracle import attention, packed, pool, select
from tests.helpers import TOPK_GAP, assert_attn_close, f64, gpu_sets

pytestmark = pytest.mark.gpu

SEQS = {
    "prefix_two_regions": [37, (6, 9, 10), 70, (5, 8, 13)],
    "one_region": [(7, 10, 9)],
    "text_then_video": [200, (8, 12, 16)],
}


def _x(B, rows, heads, D, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((B, rows, heads, D), generator=g) * scale).to(torch.bfloat16)


def _geos(seq, E):
    geo = P.PackedGeometry(seq, tile_size=E)
    ref = packed.packed_geometry(packed.token_segments(seq, (1, 1, 1)), packed.TILE_SHAPES[E])
    return geo, ref


@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("name", sorted(SEQS))
def test_scatter_gather_and_pool(name, E):
    geo, ref = _geos(SEQS[name], E)
    x = _x(2, geo.rows, 3, 64, seed=E + len(name))
    y = P.tile3d_scatter_packed(x.cuda(), geo)
    want = packed.scatter(x.view(torch.int16).numpy(), ref)
    np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy(), want)
    back = P.tile3d_gather_packed(y, geo)
    assert torch.equal(back.cpu().view(torch.int16), x.view(torch.int16))
    pooled = P.tile_pool_packed(y, geo)
    want_p = pool.tile_mean_pool(packed.scatter(f64(x), ref), ref["vc"], E)
    np.testing.assert_allclose(pooled.cpu().numpy(), want_p, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("E", [64, 128])
def test_fused_scatter_pool_equals_the_two_calls(E):
    geo, ref = _geos(SEQS["prefix_two_regions"], E)
    x = _x(2, geo.rows, 3, 128, seed=31 + E)
    y, pooled = P.tile3d_scatter_pool_packed(x.cuda(), geo)
    y2 = P.tile3d_scatter_packed(x.cuda(), geo)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    want_p = pool.tile_mean_pool(packed.scatter(f64(x), ref), ref["vc"], E)
    np.testing.assert_allclose(pooled.cpu().numpy(), want_p, rtol=1e-5, atol=1e-6)


def test_head_range_scatter_leaves_other_heads():
    geo, ref = _geos(SEQS["prefix_two_regions"], 128)
    x = _x(1, geo.rows, 4, 64, seed=9).cuda()
    y = torch.full((1, geo.buffer_rows, 4, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    P.tile3d_scatter_packed(x, geo, out=y, head0=1, heads=2)
    full = P.tile3d_scatter_packed(x, geo)
    assert torch.equal(y[:, :, 1:3], full[:, :, 1:3])
    assert bool((y[:, :, 0] == 7.0).all()) and bool((y[:, :, 3] == 7.0).all())


def _check_sets(got, want, S, geo_ref, rates, mode):
    """Equal where every boundary the row's selection crosses has a decisive gap; elsewhere a
    valid selection (right counts per region, nothing dropped clearly above something kept)."""
    B, nh, nT = S.shape[:3]
    n_exact = 0
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                g, w = got[b][h][i], want[b][h][i]
                assert np.all(np.diff(g) > 0)
                assert len(g) == len(w), (b, h, i)
                row = S[b, h, i]
                scale = np.abs(row).max()
                if mode == P.COMPETE:
                    groups = [(0, nT, len(w))]
                elif mode == P.DENSE or i < geo_ref["n_prefix"]:
                    groups = []
                    np.testing.assert_array_equal(g, w)
                else:
                    groups = [(lo, hi, min(hi - lo, int(r * (hi - lo))))
                              for (lo, hi), r in zip(geo_ref["spans"], rates)]
                decisive = True
                for lo, hi, k in groups:
                    if 0 < k < hi - lo:
                        srt = np.sort(row[lo:hi])[::-1]
                        decisive &= (srt[k - 1] - srt[k]) / scale > TOPK_GAP
                if decisive:
                    np.testing.assert_array_equal(g, w, err_msg=str((b, h, i)))
                    n_exact += 1
                else:
                    for lo, hi, k in groups:
                        ks = g[(g >= lo) & (g < hi)]
                        assert len(ks) == k
                        drop = np.setdiff1d(np.arange(lo, hi), ks)
                        if drop.size and ks.size:
                            assert row[drop].max() <= row[ks].min() + TOPK_GAP * scale
    return n_exact


@pytest.mark.parametrize("mode", ["exempt", "compete", "dense"])
@pytest.mark.parametrize("E", [64, 128])
def test_select_matches_oracle(E, mode):
    seq = SEQS["prefix_two_regions"] if mode != "compete" else SEQS["text_then_video"]
    geo, ref = _geos(seq, E)
    m = {"exempt": P.EXEMPT, "compete": P.COMPETE, "dense": P.DENSE}[mode]
    rates = [0.3, 0.25] if mode != "compete" else [0.2]
    g = torch.Generator().manual_seed(5 + E)
    B, nh, D = 2, 3, 64
    pq = torch.randn((B, nh, geo.n_tiles, D), generator=g)
    pk = torch.randn((B, nh, geo.n_tiles, D), generator=g)
    kv_idx, kv_cnt = P.tile_select_packed(pq.cuda(), pk.cuda(), geo, rates, m)
    S = select.tile_scores(pq.numpy(), pk.numpy())
    want = packed.select(S, ref, rates, exempt=(m != P.COMPETE), dense=(m == P.DENSE))
    n_exact = _check_sets(gpu_sets(kv_idx, kv_cnt), want, S, ref, rates, m)
    assert n_exact >= 0.8 * B * nh * geo.n_tiles


def _lists(sets, B, nh, nT):
    kmax = max(1, max(len(s) for bb in sets for hh in bb for s in hh))
    idx = np.full((B, nh, nT, kmax), -3, dtype=np.int32)
    cnt = np.zeros((B, nh, nT), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                idx[b, h, i, :len(sets[b][h][i])] = sets[b][h][i]
                cnt[b, h, i] = len(sets[b][h][i])
    return torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("name", ["prefix_two_regions", "one_region"])
def test_attention_with_oracle_lists(name, E, D):
    geo, ref = _geos(SEQS[name], E)
    B, nh = 1, 2
    q, k, v = (_x(B, geo.rows, nh, D, seed=s) for s in (11, 12, 13))
    qt, kt, vt = (packed.scatter(f64(t), ref) for t in (q, k, v))
    pq = pool.tile_mean_pool(qt, ref["vc"], E)
    pk = pool.tile_mean_pool(kt, ref["vc"], E)
    n_regions = len(ref["spans"])
    rates = packed.span_keep_rates(n_regions, 0.7, 0.4 if n_regions > 1 else None, True)
    sets = packed.select(select.tile_scores(pq, pk), ref, rates)
    # an empty list, to cover a query tile that keeps nothing
    sets[0][1][min(3, geo.n_tiles - 1)] = np.zeros(0, dtype=np.int64)
    kv_idx, kv_cnt = _lists(sets, B, nh, geo.n_tiles)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gq, gk, gv = (P.tile3d_scatter_packed(t.cuda(), geo) for t in (q, k, v))
    ot = P.block_sparse_attn_fwd_packed(gq, gk, gv, kv_idx, kv_cnt, geo, dev_status=status)
    want = attention.block_sparse_attention(qt, kt, vt, ref["vc"], sets, D ** -0.5, tile_elems=E)
    assert int(status.item()) == 0
    got = f64(ot)
    pads = ref["slot_row"] < 0
    assert (got[:, pads] == 0).all()
    assert_attn_close(got, want, f"packed {name} E={E} D={D}")


def test_attention_reports_out_of_range_tile_128():
    geo, ref = _geos(SEQS["one_region"], 128)
    q = _x(1, geo.rows, 1, 64, seed=3).cuda()
    qt = P.tile3d_scatter_packed(q, geo)
    kv_idx = torch.zeros((1, 1, geo.n_tiles, 2), dtype=torch.int32, device="cuda")
    kv_idx[0, 0, 0, 1] = geo.n_tiles  # out of range: skipped and reported
    kv_cnt = torch.ones((1, 1, geo.n_tiles), dtype=torch.int32, device="cuda")
    kv_cnt[0, 0, 0] = 2
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    P.block_sparse_attn_fwd_packed(qt, qt, qt, kv_idx, kv_cnt, geo, dev_status=status)
    assert int(status.item()) & 0x1


@pytest.mark.parametrize("E", [64, 128])
def test_module_end_to_end(E):
    seq = [90, (8, 12, 16), 40, (8, 16, 20)]
    mod = P.PackedTileSparseAttention(seq, heads=2, D=128, tile_size=E, sparsity=0.75,
                                      ref_keep_rate=0.5)
    geo, ref = mod.geo, packed.packed_geometry(packed.token_segments(seq, (1, 1, 1)),
                                                packed.TILE_SHAPES[E])
    q, k, v = (_x(1, geo.rows, 2, 128, seed=s) for s in (21, 22, 23))
    out = mod(q.cuda(), k.cuda(), v.cuda())
    assert int(mod.status.item()) == 0
    qt, kt, vt = (packed.scatter(f64(t), ref) for t in (q, k, v))
    pq, pk = (pool.tile_mean_pool(t, ref["vc"], E) for t in (qt, kt))
    S = select.tile_scores(pq, pk)
    want_sets = packed.select(S, ref, mod.keep_rates)
    got_sets = gpu_sets(mod.kv_idx, mod.kv_cnt)
    n_exact = _check_sets(got_sets, want_sets, S, ref, mod.keep_rates, P.EXEMPT)
    assert n_exact >= 0.8 * 2 * geo.n_tiles
    want = packed.gather(attention.block_sparse_attention(qt, kt, vt, ref["vc"], want_sets,
                                                          128 ** -0.5, tile_elems=E), ref)
    got = f64(out)
    # rows of query tiles whose kept set equals the oracle's must match its output
    tile_of = np.empty(geo.rows, dtype=np.int64)
    sr = ref["slot_row"]
    tile_of[sr[sr >= 0]] = np.nonzero(sr >= 0)[0] // E
    for h in range(2):
        same = np.array([np.array_equal(got_sets[0][h][i], want_sets[0][h][i])
                         for i in range(geo.n_tiles)])
        rows = same[tile_of]
        assert rows.mean() >= 0.8
        assert_attn_close(got[:, rows, h], want[:, rows, h], f"module E={E} head {h}")


@pytest.mark.parametrize("E", [64, 128])
def test_head_range_pool_and_attention(E):
    """A call on heads 1..2 of 4-head rows equals the full call on those heads and leaves the
    other heads of the output untouched."""
    geo, ref = _geos(SEQS["prefix_two_regions"], E)
    q, k, v = (_x(1, geo.rows, 4, 64, seed=s).cuda() for s in (41, 42, 43))
    qt, kt, vt = (P.tile3d_scatter_packed(t, geo) for t in (q, k, v))
    full_p = P.tile_pool_packed(qt, geo)
    part_p = P.tile_pool_packed(qt, geo, head0=1, heads=2)
    assert torch.equal(part_p, full_p[:, 1:3])
    y, pooled = P.tile3d_scatter_pool_packed(q, geo, head0=1, heads=2)
    np.testing.assert_allclose(pooled.cpu().numpy(), full_p[:, 1:3].cpu().numpy(),
                               rtol=1e-6, atol=1e-7)
    pk = P.tile_pool_packed(kt, geo)
    rates = packed.span_keep_rates(2, 0.6, 0.5, True)
    kv_idx, kv_cnt = P.tile_select_packed(full_p, pk, geo, rates)
    o_full = P.block_sparse_attn_fwd_packed(qt, kt, vt, kv_idx, kv_cnt, geo)
    o = torch.full_like(qt, 5.0)
    P.block_sparse_attn_fwd_packed(qt, kt, vt, kv_idx[:, 1:3].contiguous(),
                                   kv_cnt[:, 1:3].contiguous(), geo, out=o, head0=1, heads=2)
    assert torch.equal(o[:, :, 1:3], o_full[:, :, 1:3])
    assert bool((o[:, :, 0] == 5.0).all()) and bool((o[:, :, 3] == 5.0).all())


@pytest.mark.parametrize("kind", ["dense_layer", "compete"])
def test_module_dense_and_compete(kind):
    """The module in its other two selection modes against the oracle: a dense layer keeps every
    tile (output exact to the dense oracle); compete mode, one top-k over all tiles of a
    one-region sequence."""
    E = 64
    seq = [90, (8, 12, 16)]
    kw = {"dense_layer": True} if kind == "dense_layer" else {"exempt": False}
    mod = P.PackedTileSparseAttention(seq, heads=2, D=64, tile_size=E, sparsity=0.75, **kw)
    geo = mod.geo
    ref = packed.packed_geometry(packed.token_segments(seq, (1, 1, 1)), packed.TILE_SHAPES[E])
    q, k, v = (_x(1, geo.rows, 2, 64, seed=s) for s in (51, 52, 53))
    out = mod(q.cuda(), k.cuda(), v.cuda())
    assert int(mod.status.item()) == 0
    qt, kt, vt = (packed.scatter(f64(t), ref) for t in (q, k, v))
    pq, pk = (pool.tile_mean_pool(t, ref["vc"], E) for t in (qt, kt))
    S = select.tile_scores(pq, pk)
    want_sets = packed.select(S, ref, mod.keep_rates, exempt=(kind == "dense_layer"),
                              dense=(kind == "dense_layer"))
    got_sets = gpu_sets(mod.kv_idx, mod.kv_cnt)
    n_exact = _check_sets(got_sets, want_sets, S, ref, mod.keep_rates, mod.mode)
    assert n_exact >= 0.8 * 2 * geo.n_tiles
    if kind == "dense_layer":
        assert n_exact == 2 * geo.n_tiles
    want = packed.gather(attention.block_sparse_attention(qt, kt, vt, ref["vc"], want_sets,
                                                          64 ** -0.5, tile_elems=E), ref)
    got = f64(out)
    tile_of = np.empty(geo.rows, dtype=np.int64)
    sr = ref["slot_row"]
    tile_of[sr[sr >= 0]] = np.nonzero(sr >= 0)[0] // E
    for h in range(2):
        same = np.array([np.array_equal(got_sets[0][h][i], want_sets[0][h][i])
                         for i in range(geo.n_tiles)])
        rows = same[tile_of]
        assert_attn_close(got[:, rows, h], want[:, rows, h], f"module {kind} head {h}")
