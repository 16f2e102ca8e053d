"""GPU parity of the BSA ratio mode: a fixed count ``max(1, floor(64 * keep_ratio))`` of kept query
rows per 64-row block (the rows least cosine-similar to the block mean), then the same source rows,
kept-query pooling, mass selection and attention as the threshold mode."""
import numpy as np
import pytest

from block_sparse_video_tile3d_b200 import (TileSparseAttention, tile3d_scatter,
                                            tile_prune_queries_ratio, workloads)
from oracle import bsa, pipeline, tiling
from tests.helpers import assert_attn_close, f64, gpu_sets

pytestmark = pytest.mark.gpu

# The kernel ranks fp32 cosines of bf16 rows; the oracle ranks fp64 ones. Rows whose oracle cosine
# lies within this distance of the keep boundary may fall on either side.
COS_TIE = 1e-4


def _queries(structured: bool, heads: int = 3):
    w = workloads.WORKLOADS["bsa"].with_(T=8, H=8, W=12, heads=heads)
    q, k, v = workloads.make_qkv(w)
    if structured:
        q = workloads.make_structured_queries(w, q)
    return w, q, k, v


def _check_block(rows, keep_g, src_g, pq_g, keep_o, cos_o, ks):
    """One block: exact count, the kept set is a least-similar set up to COS_TIE, decided rows
    agree with the oracle, sources name the most similar kept row, pooled query of the kept rows."""
    assert keep_g.sum() == ks
    if ks < 64:
        assert cos_o[keep_g].max() <= cos_o[~keep_g].min() + COS_TIE
    order = np.sort(cos_o)
    thr = 0.5 * (order[ks - 1] + order[ks]) if ks < 64 else np.inf
    decided = np.abs(cos_o - thr) > COS_TIE
    np.testing.assert_array_equal(keep_g[decided], keep_o[decided])
    kept = np.nonzero(keep_g)[0]
    np.testing.assert_array_equal(src_g[keep_g], kept)
    nrm = np.linalg.norm(rows, axis=1)
    for r in np.nonzero(~keep_g)[0]:
        c = rows[kept] @ rows[r] / (nrm[kept] * nrm[r])
        best = c.max()
        assert keep_g[src_g[r]]
        assert c[list(kept).index(src_g[r])] >= best - COS_TIE
    np.testing.assert_allclose(pq_g, rows[kept].mean(axis=0), rtol=1e-5, atol=2e-6)
    return int(decided.sum())


@pytest.mark.parametrize("structured", [False, True])
@pytest.mark.parametrize("ratio", [0.25, 0.3, 0.5, 0.01, 1.0])
def test_ratio_prune_matches_oracle(structured, ratio):
    w, q, _, _ = _queries(structured)
    qt = tile3d_scatter(q.cuda(), w.T, w.H, w.W)
    keep, src, pqk = tile_prune_queries_ratio(qt, w.T, w.H, w.W, ratio)
    keep, src, pqk = keep.cpu().numpy().astype(bool), src.cpu().numpy(), f64(pqk)
    r32 = float(np.float32(ratio))  # the C ABI takes the ratio as fp32
    ks = bsa.keep_size_for_ratio(r32)
    oqt = tiling.tile_scatter(f64(q), w.T, w.H, w.W)
    okeep, _, ocos = bsa.prune_queries_ratio(oqt, r32)
    decided = 0
    for h in range(w.heads):
        for i in range(w.nT):
            rows = oqt[0, 64 * i:64 * i + 64, h]
            decided += _check_block(rows, keep[0, h, i], src[0, h, i], pqk[0, h, i],
                                    okeep[0, h, i], ocos[0, h, i], ks)
    # unstructured rows have well-separated cosines: almost every decision is checked exactly
    if not structured:
        assert decided >= 0.95 * w.heads * w.nT * 64


def test_ratio_one_keeps_every_row_and_pools_the_block():
    w, q, _, _ = _queries(True, heads=2)
    qt = tile3d_scatter(q.cuda(), w.T, w.H, w.W)
    keep, src, pqk = tile_prune_queries_ratio(qt, w.T, w.H, w.W, 1.0)
    assert bool(keep.all())
    np.testing.assert_array_equal(src.cpu().numpy(),
                                  np.broadcast_to(np.arange(64), src.shape))
    oqt = tiling.tile_scatter(f64(q), w.T, w.H, w.W)
    want = oqt[0].reshape(w.nT, 64, w.heads, w.D).mean(axis=1).transpose(1, 0, 2)
    np.testing.assert_allclose(f64(pqk)[0], want, rtol=1e-5, atol=2e-6)


def test_ratio_rejects_out_of_range():
    w, q, _, _ = _queries(False, heads=1)
    qt = tile3d_scatter(q.cuda(), w.T, w.H, w.W)
    for bad in (0.0, 1.25, -0.1):
        with pytest.raises(RuntimeError):
            tile_prune_queries_ratio(qt, w.T, w.H, w.W, bad)


@pytest.mark.parametrize("ratio", [0.25, 0.5])
def test_bsa_ratio_end_to_end(ratio):
    w = workloads.WORKLOADS["bsa"].with_(T=8, H=16, W=16, heads=2)
    q, k, v = workloads.make_qkv(w)
    q = workloads.make_structured_queries(w, q)
    m = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode="bsa", mass=w.mass,
                            min_k=w.min_kv, keep_ratio=ratio)
    out = f64(m(q.cuda(), k.cuda(), v.cuda()))
    assert m.device_status() == 0
    ref = pipeline.forward(q, k, v, w.T, w.H, w.W, "bsa", scale=w.scale, tau=w.mass,
                           min_k=w.min_kv, keep_ratio=float(np.float32(ratio)))
    keep = m.keep.cpu().numpy().astype(bool)
    ks = bsa.keep_size_for_ratio(float(np.float32(ratio)))
    assert (keep.sum(axis=-1) == ks).all()
    got_sets = gpu_sets(m.kv_idx, m.kv_cnt)
    pos = tiling.padded_positions(w.T, w.H, w.W)
    n = 0
    for b in range(w.B):
        for h in range(w.heads):
            for i in range(w.nT):
                if not (np.array_equal(got_sets[b][h][i], ref["sets"][b][h][i])
                        and np.array_equal(keep[b, h, i], ref["keep"][b, h, i])):
                    continue
                rows = np.nonzero(pos // 64 == i)[0]
                assert_attn_close(out[b, rows, h], ref["o"][b, rows, h], what=f"tile {(b, h, i)}")
                n += 1
    assert n >= 0.7 * w.B * w.heads * w.nT
