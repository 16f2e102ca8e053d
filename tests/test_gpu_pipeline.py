"""GPU parity of the whole hot path (scatter -> coarse selection -> block-sparse attention ->
gather) against the oracle run independently on the same seeded raster inputs."""
import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import TileSparseAttention, workloads
from oracle import attention, pipeline, pool, select, tiling
from tests.helpers import assert_attn_close, check_topk_sets, f64, gpu_sets

pytestmark = pytest.mark.gpu


def test_tiny_workload_end_to_end():
    w = workloads.WORKLOADS["tiny"]
    q, k, v = workloads.make_qkv(w)
    m = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode="topk", topk=w.k)
    out = m(q.cuda(), k.cuda(), v.cuda())
    ref = pipeline.forward(q, k, v, w.T, w.H, w.W, "topk", scale=w.scale, topk=w.k)
    stats = check_topk_sets(gpu_sets(m.kv_idx, m.kv_cnt), ref["sets"], ref["S"], w.k)
    assert stats["near_tie"] == 0
    assert_attn_close(f64(out), ref["o"])
    assert m.device_status() == 0


def test_ragged_topk_end_to_end():
    w = workloads.WORKLOADS["tiny"].with_(B=2, T=9, H=10, W=13, heads=3, D=128, k=7)
    q, k, v = workloads.make_qkv(w, seed=77)
    m = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode="topk", topk=w.k)
    out = m(q.cuda(), k.cuda(), v.cuda())
    ref = pipeline.forward(q, k, v, w.T, w.H, w.W, "topk", scale=w.scale, topk=w.k)
    got_sets = gpu_sets(m.kv_idx, m.kv_cnt)
    check_topk_sets(got_sets, ref["sets"], ref["S"], w.k)
    same = all(np.array_equal(a, b) for bb in range(w.B) for h in range(w.heads)
               for a, b in zip(got_sets[bb][h], ref["sets"][bb][h]))
    if same:
        assert_attn_close(f64(out), ref["o"])


def test_mask_mode_end_to_end_sliding():
    w = workloads.WORKLOADS["ragged_sliding"].with_(B=1, T=9, H=10, W=13, heads=2)
    q, k, v = workloads.make_qkv(w)
    mask = workloads.block_mask(w)
    m = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode="mask", mask=mask)
    out = m(q.cuda(), k.cuda(), v.cuda())
    ref = pipeline.forward(q, k, v, w.T, w.H, w.W, "mask", scale=w.scale, mask=mask.numpy())
    assert_attn_close(f64(out), ref["o"])


def _exact_rows(got_sets, ref_sets, B, heads, nT):
    return {(b, h, i) for b in range(B) for h in range(heads) for i in range(nT)
            if np.array_equal(got_sets[b][h][i], ref_sets[b][h][i])}


def test_bsa_end_to_end_structured():
    w = workloads.WORKLOADS["bsa"].with_(T=8, H=16, W=16, heads=2)
    q, k, v = workloads.make_qkv(w)
    q = workloads.make_structured_queries(w, q)
    m = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode="bsa", mass=w.mass,
                            min_k=w.min_kv, cos_thresh=w.cos_thresh)
    out = f64(m(q.cuda(), k.cuda(), v.cuda()))
    ref = pipeline.forward(q, k, v, w.T, w.H, w.W, "bsa", scale=w.scale, tau=w.mass,
                           min_k=w.min_kv, cos_thresh=w.cos_thresh)
    keep = m.keep.cpu().numpy().astype(bool)
    # tiles where pruning and selection agree exactly are compared element by element
    got_sets = gpu_sets(m.kv_idx, m.kv_cnt)
    rows = _exact_rows(got_sets, ref["sets"], w.B, w.heads, w.nT)
    assert len(rows) >= 0.8 * w.heads * w.nT
    n = 0
    for (b, h, i) in rows:
        if not np.array_equal(keep[b, h, i], ref["keep"][b, h, i]):
            continue
        assert_attn_close(out[b, :, h][ref_rows(w, i)], ref["o"][b, :, h][ref_rows(w, i)],
                          what=f"tile {(b, h, i)}")
        n += 1
    assert n >= 0.7 * w.heads * w.nT


def ref_rows(w, i):
    """Raster token ids of tile i (from the oracle's geometry)."""
    pos = tiling.padded_positions(w.T, w.H, w.W)
    return np.nonzero(pos // 64 == i)[0]


@pytest.mark.parametrize("name,heads_checked", [("small", [0, 7, 11]), ("large", [3, 39])])
def test_workload_topk_full_size(name, heads_checked):
    """Full-size GPU pipeline; the oracle reruns selected heads on single-head slices and checks
    the kept sets (exact where the score gap allows) and sampled output tiles."""
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.make_qkv(w)
    m = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode="topk", topk=w.k)
    out = f64(m(q.cuda(), k.cuda(), v.cuda()))
    assert m.device_status() == 0
    got_sets = gpu_sets(m.kv_idx, m.kv_cnt)
    vc = tiling.variable_block_sizes(w.T, w.H, w.W)
    pos = tiling.padded_positions(w.T, w.H, w.W)
    rng = np.random.default_rng(3)
    for h in heads_checked:
        sl = lambda x: f64(x[:, :, h:h + 1])  # noqa: E731
        qt, kt, vt = (tiling.tile_scatter(sl(x), w.T, w.H, w.W) for x in (q, k, v))
        S = select.tile_scores(pool.tile_mean_pool(qt, vc), pool.tile_mean_pool(kt, vc))
        sets = select.select_topk(S, w.k)
        stats = check_topk_sets([[got_sets[0][h]]], sets, S, w.k)
        assert stats["exact"] >= 0.3 * w.nT
        tiles = [int(t) for t in rng.choice(w.nT, 6, replace=False)] + [w.nT - 1]
        tiles = [i for i in tiles if np.array_equal(got_sets[0][h][i], sets[0][0][i])]
        want = attention.block_sparse_attention(qt, kt, vt, vc, sets, w.scale,
                                                q_tiles=[(0, 0, i) for i in tiles])
        got_t = np.zeros_like(want)
        got_t[:, pos, 0] = out[:, :, h]
        for i in tiles:
            rows = slice(64 * i, 64 * i + 64)
            assert_attn_close(got_t[0, rows, 0], want[0, rows, 0], what=f"{name} tile {(h, i)}")
