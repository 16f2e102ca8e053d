"""CPU pins of the oracle's block-sparse attention, BSA pruning and the chained pipeline.

The references here are torch's own ``scaled_dot_product_attention`` and ``cosine_similarity``
in fp64 on the CPU (library routines independent of the oracle's numpy code), pure-Python
scalar loops on tiny inputs, and closed-form special cases.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention, bsa, pipeline, select, tiling


def _sdpa(q, k, v, scale, mask=None):
    """q [m, D], k/v [n, D] fp64 numpy -> torch SDPA output (optionally with a boolean mask)."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(a))[None, None] for a in (q, k, v))
    am = None if mask is None else torch.from_numpy(mask)[None, None]
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("grid", [(4, 8, 8), (5, 6, 7)])
def test_full_selection_is_dense_attention(grid):
    """k = nT (every key tile kept) reproduces dense softmax attention over the raster sequence,
    pads included in the geometry (ragged grid)."""
    T, H, W = grid
    rng = np.random.default_rng(10)
    B, nh, D = 1, 2, 16
    q, k, v = (rng.standard_normal((B, T * H * W, nh, D)) for _ in range(3))
    nT = len(tiling.variable_block_sizes(T, H, W))
    scale = 1.0 / math.sqrt(D)
    res = pipeline.forward(q, k, v, T, H, W, "topk", scale=scale, topk=nT)
    for h in range(nh):
        want = _sdpa(q[0, :, h], k[0, :, h], v[0, :, h], scale)
        np.testing.assert_allclose(res["o"][0, :, h], want, rtol=1e-10, atol=1e-12)


def test_block_sparse_equals_masked_dense():
    """Attention over kept tile pairs equals dense attention with the tile-pair mask expanded to
    tokens (raster order, boolean attention mask)."""
    T, H, W = 6, 5, 9
    rng = np.random.default_rng(11)
    B, nh, D = 2, 2, 8
    q, k, v = (rng.standard_normal((B, T * H * W, nh, D)) for _ in range(3))
    nT = len(tiling.variable_block_sizes(T, H, W))
    mask = (rng.random((B, nh, nT, nT)) < 0.3).astype(np.uint8)
    for i in range(nT):
        mask[:, :, i, i] = 1
    scale = 0.3
    res = pipeline.forward(q, k, v, T, H, W, "mask", scale=scale, mask=mask)
    pos = tiling.padded_positions(T, H, W)
    tid = pos // 64
    for b in range(B):
        for h in range(nh):
            tok_mask = mask[b, h][tid][:, tid].astype(bool)
            want = _sdpa(q[b, :, h], k[b, :, h], v[b, :, h], scale, tok_mask)
            np.testing.assert_allclose(res["o"][b, :, h], want, rtol=1e-10, atol=1e-12)


def test_scalar_loops_tiny():
    """Pure-Python loops for a few rows of the tiny workload shape."""
    T, H, W, D = 4, 8, 8, 4
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((1, T * H * W, 1, D)) for _ in range(3))
    sets = [[[np.array([0, 2]), np.array([1]), np.array([1, 2, 3]), np.array([3])]]]
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v))
    out = attention.block_sparse_attention(qt, kt, vt, vc, sets, 0.5)
    for (i, r) in [(0, 0), (0, 63), (2, 17), (3, 40)]:
        keys = [64 * j + c for j in sets[0][0][i] for c in range(64)]
        logits = [0.5 * sum(qt[0, 64 * i + r, 0, d] * kt[0, n, 0, d] for d in range(D)) for n in keys]
        mx = max(logits)
        ws = [math.exp(x - mx) for x in logits]
        s = sum(ws)
        for d in range(D):
            want = sum(w * vt[0, n, 0, d] for w, n in zip(ws, keys)) / s
            assert abs(out[0, 64 * i + r, 0, d] - want) < 1e-12


def test_convexity_and_weight_sums():
    T, H, W = 5, 4, 9
    rng = np.random.default_rng(13)
    q, k, v = (rng.standard_normal((1, T * H * W, 2, 8)) * 3 for _ in range(3))
    vc = tiling.variable_block_sizes(T, H, W)
    nT = len(vc)
    qt, kt, vt = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v))
    mask = (rng.random((1, 2, nT, nT)) < 0.5).astype(np.uint8)
    mask[..., 0] = 1
    sets = select.map_to_sets(mask)
    out, ws = attention.block_sparse_attention(qt, kt, vt, vc, sets, 0.35, return_wsum=True)
    valid = tiling.valid_slot_mask(T, H, W)
    np.testing.assert_allclose(ws[0, valid], 1.0, atol=1e-12)
    assert np.all(out[0, ~valid] == 0.0)
    for h in range(2):
        for i in range(nT):
            keys = np.concatenate([64 * j + np.arange(vc[j]) for j in sets[0][h][i]])
            lo, hi = vt[0, keys, h].min(axis=0), vt[0, keys, h].max(axis=0)
            o = out[0, 64 * i:64 * i + vc[i], h]
            assert np.all(o >= lo - 1e-12) and np.all(o <= hi + 1e-12)


def test_identical_keys_give_mean_of_values():
    T, H, W = 4, 4, 8
    rng = np.random.default_rng(14)
    q = rng.standard_normal((1, T * H * W, 1, 8))
    k = np.ones((1, T * H * W, 1, 8))
    v = rng.standard_normal((1, T * H * W, 1, 8))
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v))
    sets = [[[np.array([1]), np.array([1])]]]
    out = attention.block_sparse_attention(qt, kt, vt, vc, sets, 0.125)
    want = vt[0, 64:128, 0].mean(axis=0)
    np.testing.assert_allclose(out[0, :128, 0], np.broadcast_to(want, (128, 8)), rtol=1e-12)


def test_empty_set_gives_zero_rows():
    T, H, W = 4, 4, 8
    rng = np.random.default_rng(15)
    q, k, v = (rng.standard_normal((1, T * H * W, 1, 4)) for _ in range(3))
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v))
    sets = [[[np.zeros(0, dtype=np.int64), np.array([0])]]]
    out = attention.block_sparse_attention(qt, kt, vt, vc, sets, 0.5)
    assert np.all(out[0, :64] == 0.0) and np.all(out[0, 64:] != 0.0)


# ---------------------------------------------------------------------------------- BSA variant

def test_prune_cosine_against_torch():
    rng = np.random.default_rng(16)
    base = rng.standard_normal(32)
    rows = np.where(rng.random((64, 1)) < 0.5, base + 0.05 * rng.standard_normal((64, 32)),
                    rng.standard_normal((64, 32)))
    keep, src, cosm = bsa.prune_block(rows, 0.8)
    rt = torch.from_numpy(rows)
    cm = F.cosine_similarity(rt, rt.mean(dim=0, keepdim=True), dim=1, eps=0).numpy()
    np.testing.assert_allclose(cosm, cm, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(keep, ~(cm > 0.8))
    gram = F.cosine_similarity(rt[:, None, :], rt[None, :, :], dim=2, eps=0).numpy()
    kept = np.nonzero(keep)[0]
    for i in range(64):
        if keep[i]:
            assert src[i] == i
        else:
            assert src[i] == kept[int(np.argmax(gram[i, kept]))]
            assert keep[src[i]]


def test_prune_identical_rows_keep_one():
    rows = np.tile(np.arange(1.0, 9.0), (64, 1))
    keep, src, _ = bsa.prune_block(rows, 0.95)
    assert keep.sum() == 1 and keep[0]
    assert np.all(src == 0)


def test_prune_threshold_above_one_keeps_all_and_matches_mass_path():
    T, H, W = 4, 8, 8
    rng = np.random.default_rng(17)
    q, k, v = (rng.standard_normal((1, T * H * W, 2, 16)) for _ in range(3))
    a = pipeline.forward(q, k, v, T, H, W, "bsa", scale=0.25, tau=0.7, min_k=1, cos_thresh=1.5)
    b = pipeline.forward(q, k, v, T, H, W, "mass", scale=0.25, tau=0.7, min_k=1)
    assert a["keep"].all()
    np.testing.assert_array_equal(a["src"], np.broadcast_to(np.arange(64), a["src"].shape))
    np.testing.assert_allclose(a["o"], b["o"], rtol=1e-13, atol=1e-13)


def test_bsa_pruned_rows_copy_source_outputs():
    T, H, W = 4, 8, 8
    rng = np.random.default_rng(18)
    base = rng.standard_normal((1, 1, 2, 16))
    q = base + 0.02 * rng.standard_normal((1, T * H * W, 2, 16))
    q[:, ::3] = rng.standard_normal(q[:, ::3].shape)
    k, v = (rng.standard_normal((1, T * H * W, 2, 16)) for _ in range(2))
    r = pipeline.forward(q, k, v, T, H, W, "bsa", scale=0.25, tau=0.9, min_k=1, cos_thresh=0.9)
    keep, src, ot = r["keep"], r["src"], r["ot"]
    assert (~keep).sum() > 0
    for h in range(2):
        for i in range(4):
            for s in range(64):
                np.testing.assert_array_equal(ot[0, 64 * i + s, h], ot[0, 64 * i + src[0, h, i, s], h])
    # kept rows equal dense attention of that row over the kept key tiles
    vc = r["vc"]
    for h in range(2):
        for i in range(4):
            rows = 64 * i + np.nonzero(keep[0, h, i])[0]
            keys = np.concatenate([64 * j + np.arange(vc[j]) for j in r["sets"][0][h][i]])
            want = _sdpa(r["qt"][0, rows, h], r["kt"][0, keys, h], r["vt"][0, keys, h], 0.25)
            np.testing.assert_allclose(ot[0, rows, h], want, rtol=1e-10, atol=1e-12)
    # KV selection uses queries pooled over kept rows only
    for h in range(2):
        for i in range(4):
            rows = 64 * i + np.nonzero(keep[0, h, i])[0]
            np.testing.assert_allclose(r["pq"][0, h, i], r["qt"][0, rows, h].mean(axis=0), rtol=1e-12)
