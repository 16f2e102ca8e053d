"""Host side of the packed multi-region calls (include/tile3d_packed.h): the library's geometry
equals the oracle's on mixed sequences with 64- and 128-token tiles, list capacities follow the
selection reading, and bad arguments are rejected on the host (no GPU: nothing here is enqueued).
"""
import ctypes
import math

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from block_sparse_video_tile3d_b200 import _lib
from block_sparse_video_tile3d_b200._lib import lib
from block_sparse_video_tile3d_b200.packed import PackedGeometry, TILE_SHAPES, span_keep_rates
from oracle import packed as opacked

SEQS = [
    [5, (8, 4, 8), 70],
    [130, (5, 4, 9)],
    [(21, 30, 52)],
    [3, (5, 9, 6), 200, (2, 3, 17), 64, (4, 4, 8)],
    [(4, 4, 4), 1, (3, 3, 3), 129],
]


@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("seq", SEQS)
def test_geometry_matches_oracle(seq, E):
    geo = PackedGeometry(seq, tile_size=E, device="cpu")
    ref = opacked.packed_geometry(opacked.token_segments(seq, (1, 1, 1)), TILE_SHAPES[E])
    assert geo.rows == ref["rows"] and geo.n_prefix == ref["n_prefix"]
    assert geo.spans == [tuple(s) for s in ref["spans"]]
    assert geo.vc == ref["vc"].tolist()
    assert geo.slot_row_host == ref["slot_row"].tolist()


_segment = st.one_of(st.integers(1, 300),
                     st.tuples(st.integers(1, 12), st.integers(1, 12), st.integers(1, 12)))


@settings(max_examples=40, deadline=None, derandomize=True)
@given(seq=st.lists(_segment, min_size=1, max_size=6).filter(
    lambda q: any(isinstance(x, tuple) for x in q)), E=st.sampled_from([64, 128]))
def test_geometry_matches_oracle_on_random_sequences(seq, E):
    """Random mixes of dense runs and regions (ragged every way): the library's host geometry is
    the oracle's, slot for slot."""
    geo = PackedGeometry(seq, tile_size=E, device="cpu")
    ref = opacked.packed_geometry(opacked.token_segments(seq, (1, 1, 1)), TILE_SHAPES[E])
    assert geo.rows == ref["rows"] and geo.n_prefix == ref["n_prefix"]
    assert geo.spans == [tuple(s) for s in ref["spans"]]
    assert geo.vc == ref["vc"].tolist()
    assert geo.slot_row_host == ref["slot_row"].tolist()


def test_patch_division_and_contract():
    geo = PackedGeometry([5, (8, 4, 8), 70], patch=(2, 1, 2), device="cpu")
    assert geo.vc == [5, 64, 6, 64]
    with pytest.raises(ValueError):
        PackedGeometry([(5, 4, 9)], patch=(2, 1, 1), device="cpu")
    with pytest.raises(_lib.Tile3dError):
        PackedGeometry([10, 0], device="cpu")  # no region
    with pytest.raises(ValueError):
        PackedGeometry([(4, 4, 4)], tile_size=96, device="cpu")
    with pytest.raises(_lib.Tile3dError):
        PackedGeometry([(4, 4, 4)], tile_shape=(4, 4, 5), device="cpu")  # 80 tokens


def test_geometry_rejects_malformed_segments():
    lay = _lib.PackedLayout()
    bad = (_lib.Segment * 1)(_lib.Segment(3, 1, 1, 1))  # both a row count and a grid
    assert lib.t3d_packed_geometry(bad, 1, 4, 4, 4, ctypes.byref(lay), None, None, None) == 1
    assert b"neither" in lib.t3d_last_error_string()
    assert lib.t3d_packed_geometry(bad, 0, 4, 4, 4, ctypes.byref(lay), None, None, None) == 1
    ok = (_lib.Segment * 1)(_lib.Segment(0, 2, 2, 2))
    assert lib.t3d_packed_geometry(ok, 1, 4, 4, 4, None, None, None, None) == 1
    assert lib.t3d_packed_geometry(ok, 1, 4, 4, 4, ctypes.byref(lay), None, None, None) == 0
    assert (lay.n_tiles, lay.rows, lay.n_prefix, lay.n_regions) == (1, 8, 0, 1)


def _cap(n_tiles, mode, n_prefix, spans, rates):
    sp = (ctypes.c_int32 * len(spans))(*spans)
    rt = (ctypes.c_double * len(rates))(*rates)
    out = ctypes.c_int()
    st = lib.tile_select_packed_capacity(n_tiles, mode, n_prefix, len(rates), ctypes.cast(sp, ctypes.c_void_p),
                                         ctypes.cast(rt, ctypes.c_void_p), ctypes.byref(out))
    return st, out.value


def test_capacity_follows_the_selection_reading():
    E, C, Dn = _lib.T3D_PACKED_EXEMPT, _lib.T3D_PACKED_COMPETE, _lib.T3D_PACKED_DENSE
    # no prefix: the sum of int(rate * n) over regions
    assert _cap(30, E, 0, [0, 10, 10, 30], [0.25, 0.5]) == (0, 2 + 10)
    # a prefix row keeps every tile
    assert _cap(33, E, 3, [3, 13, 13, 33], [0.25, 0.5]) == (0, 33)
    assert _cap(33, C, 3, [3, 33], [0.125]) == (0, int(0.125 * 33))
    assert _cap(33, Dn, 3, [3, 33], [0.5]) == (0, 33)
    # malformed spans and rates, compete with references, unknown mode
    assert _cap(33, E, 3, [3, 13, 14, 33], [0.25, 0.5])[0] == 1
    assert _cap(33, E, 3, [0, 13, 13, 33], [0.25, 0.5])[0] == 1
    assert _cap(33, E, 3, [3, 13, 13, 33], [0.25, 1.5])[0] == 1
    assert _cap(33, C, 3, [3, 13, 13, 33], [0.25, 0.5])[0] == 1
    assert _cap(33, 7, 3, [3, 33], [0.5])[0] == 1


def test_keep_count_truncates_like_the_oracle():
    # the library computes min(n, int(rate * n)) in double, as the oracle and sla.get_block_map
    for n in (1, 7, 100, 448):
        for rate in (0.0, 0.1, 0.125, 1 / 3, 0.5, 0.9999, 1.0):
            st, cap = _cap(n, _lib.T3D_PACKED_EXEMPT, 0, [0, n], [rate])
            assert st == 0 and cap == max(1, min(n, int(rate * n)))


def test_span_keep_rates_matches_oracle():
    for args in [(3, 0.875, 0.25, True), (3, 0.0, 0.25, True), (1, 0.75, None, False), (1, 0.5, None, True)]:
        assert span_keep_rates(*args) == opacked.span_keep_rates(*args)
    for bad in [(2, 0.9, None, True), (2, 0.9, 0.5, False)]:
        with pytest.raises(ValueError):
            span_keep_rates(*bad)
        with pytest.raises(ValueError):
            opacked.span_keep_rates(*bad)


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation


def _packed(**kw):
    f = dict(B=1, heads=2, D=64, heads_total=0, head0=0, tile_elems=64, n_tiles=4, rows=200,
             slot_row=FAKE, vc=FAKE)
    f.update(kw)
    return _lib.Packed(**f)


def test_device_calls_validate_on_the_host():
    P = ctypes.c_void_p(FAKE)
    for kw, frag in [(dict(tile_elems=96), b"tile_elems"), (dict(D=96), b"D=96"),
                     (dict(slot_row=None), b"slot_row"), (dict(heads_total=2, head0=1), b"heads"),
                     (dict(n_tiles=0), b"n_tiles")]:
        p = _packed(**kw)
        assert lib.tile3d_scatter_packed(ctypes.byref(p), P, P, None) != 0
        assert frag in lib.t3d_last_error_string(), (kw, lib.t3d_last_error_string())
    p = _packed()
    scale = 1.0 / math.sqrt(64)
    ws = lib.block_sparse_attn_packed_workspace_size(ctypes.byref(p), 2)
    assert ws >= 256
    assert lib.block_sparse_attn_fwd_packed(ctypes.byref(p), P, P, P, P, P, P, 5, scale, P, ws, None,
                                            None) == 1  # kmax > n_tiles
    assert lib.block_sparse_attn_fwd_packed(ctypes.byref(p), P, P, P, P, P, P, 2, 0.2, P, ws, None,
                                            None) == 1  # scale
    assert lib.block_sparse_attn_fwd_packed(ctypes.byref(p), P, P, P, P, P, P, 2, scale, P, ws - 1,
                                            None, None) == 1  # workspace
    big = _packed(tile_elems=128, n_tiles=2049, rows=2049 * 128)
    wsb = lib.block_sparse_attn_packed_workspace_size(ctypes.byref(big), 2)
    assert lib.block_sparse_attn_fwd_packed(ctypes.byref(big), P, P, P, P, P, P, 2, scale, P, wsb,
                                            None, None) == 2  # 4098 units
    sp = (ctypes.c_int32 * 2)(0, 4)
    rt = (ctypes.c_double * 1)(0.5)
    need = lib.tile_select_packed_workspace_size(ctypes.byref(p))
    assert lib.tile_select_packed(ctypes.byref(p), P, P, _lib.T3D_PACKED_EXEMPT, 0, 1,
                                  ctypes.cast(sp, ctypes.c_void_p), ctypes.cast(rt, ctypes.c_void_p),
                                  1, P, P, P, need, None, None) == 1  # kmax 1 < capacity 2
    assert b"kmax" in lib.t3d_last_error_string()
