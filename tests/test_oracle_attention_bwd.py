"""CPU pins of the oracle's backward pass of block-sparse attention (gradients of the output with
respect to Q, K and V for a given output gradient).

The references are torch autograd through ``scaled_dot_product_attention`` in fp64 on the CPU (a
library routine independent of the oracle's numpy code, dense and with a boolean token mask),
central finite differences of the oracle's pinned forward, and two identities of softmax attention.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention, attention_bwd, bsa, tiling


def _problem(T, H, W, B=1, nh=2, D=8, seed=0, density=0.4):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, T * H * W, nh, D)) for _ in range(3))
    nT = len(tiling.variable_block_sizes(T, H, W))
    mask = rng.random((B, nh, nT, nT)) < density
    for i in range(nT):
        mask[:, :, i, i] = True
    sets = [[[np.nonzero(mask[b, h, i])[0] for i in range(nT)] for h in range(nh)]
            for b in range(B)]
    return rng, q, k, v, mask, sets


def _autograd_raster(q, k, v, do, scale, tok_mask=None):
    """Gradients of sum(do * SDPA(q, k, v)) for one (batch, head) in raster order, fp64."""
    qt, kt, vt = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    am = None if tok_mask is None else torch.from_numpy(tok_mask)[None, None]
    o = F.scaled_dot_product_attention(qt[None, None], kt[None, None], vt[None, None],
                                       attn_mask=am, scale=scale)[0, 0]
    (o * torch.from_numpy(do)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def _oracle_raster(q, k, v, do, T, H, W, sets, scale, keep=None, src=None):
    """The oracle's gradients, computed in tile order and returned in raster order."""
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt, dot = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v, do))
    g = attention_bwd.block_sparse_attention_bwd(qt, kt, vt, vc, sets, scale, dot, keep, src)
    return tuple(tiling.tile_gather(x, T, H, W) for x in g)


@pytest.mark.parametrize("grid", [(4, 8, 8), (5, 6, 7)])
def test_all_tiles_kept_is_dense_autograd(grid):
    """Every key tile kept: the gradients of dense softmax attention (ragged grid included)."""
    T, H, W = grid
    rng, q, k, v, _, _ = _problem(T, H, W, seed=1)
    nT = len(tiling.variable_block_sizes(T, H, W))
    sets = [[[np.arange(nT) for _ in range(nT)] for _ in range(q.shape[2])]]
    do = rng.standard_normal(q.shape)
    scale = 1.0 / math.sqrt(q.shape[3])
    dq, dk, dv = _oracle_raster(q, k, v, do, T, H, W, sets, scale)
    for h in range(q.shape[2]):
        want = _autograd_raster(q[0, :, h], k[0, :, h], v[0, :, h], do[0, :, h], scale)
        for got, w in zip((dq, dk, dv), want):
            np.testing.assert_allclose(got[0, :, h], w, rtol=1e-9, atol=1e-11)


def test_block_sparse_is_masked_autograd():
    """Kept tile pairs: the gradients of dense attention with the tile mask expanded to tokens."""
    T, H, W = 6, 5, 9
    rng, q, k, v, mask, sets = _problem(T, H, W, B=2, seed=2)
    do = rng.standard_normal(q.shape)
    scale = 0.3
    dq, dk, dv = _oracle_raster(q, k, v, do, T, H, W, sets, scale)
    tid = tiling.padded_positions(T, H, W) // 64
    for b in range(2):
        for h in range(2):
            tok = mask[b, h][tid][:, tid]
            want = _autograd_raster(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, tok)
            for got, w in zip((dq, dk, dv), want):
                np.testing.assert_allclose(got[b, :, h], w, rtol=1e-9, atol=1e-11)


def test_finite_differences_tiny():
    """Central differences of sum(dO * forward) agree with the oracle's gradients entry by entry."""
    T, H, W = 3, 5, 6  # two tiles, one of them partial
    rng, q, k, v, _, sets = _problem(T, H, W, nh=1, D=4, seed=3, density=0.5)
    do = rng.standard_normal(q.shape)
    scale = 0.7
    vc = tiling.variable_block_sizes(T, H, W)

    def loss(qq, kk, vv):
        qt, kt, vt = (tiling.tile_scatter(a, T, H, W) for a in (qq, kk, vv))
        o = tiling.tile_gather(attention.block_sparse_attention(qt, kt, vt, vc, sets, scale),
                               T, H, W)
        return float((o * do).sum())

    grads = _oracle_raster(q, k, v, do, T, H, W, sets, scale)
    eps = 1e-6
    for which, g in enumerate(grads):
        for _ in range(12):
            idx = (0, int(rng.integers(q.shape[1])), 0, int(rng.integers(q.shape[3])))
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += eps
            up = loss(*args)
            args[which][idx] -= 2 * eps
            down = loss(*args)
            assert abs((up - down) / (2 * eps) - g[idx]) < 1e-7 * (1.0 + abs(g[idx]))


def test_softmax_identities():
    """Per query row the score gradients sum to zero, so the key gradients of all keys add up to 0;
    the weights sum to one, so the value gradients add up to the sum of the output gradients."""
    T, H, W = 4, 8, 12
    rng, q, k, v, _, _ = _problem(T, H, W, seed=4)
    nT = len(tiling.variable_block_sizes(T, H, W))
    sets = [[[np.arange(nT) for _ in range(nT)] for _ in range(2)]]
    do = rng.standard_normal(q.shape)
    _, dk, dv = _oracle_raster(q, k, v, do, T, H, W, sets, 0.4)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-10)
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), rtol=1e-10, atol=1e-10)


def test_pad_rows_and_keys_get_no_gradient():
    """On a ragged grid the tile-ordered gradients are zero at every pad slot."""
    T, H, W = 5, 6, 7
    rng, q, k, v, _, sets = _problem(T, H, W, seed=5)
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v))
    dot = rng.standard_normal(qt.shape)  # nonzero even at pad slots
    g = attention_bwd.block_sparse_attention_bwd(qt, kt, vt, vc, sets, 0.5, dot)
    pad = np.ones(qt.shape[1], dtype=bool)
    pad[tiling.padded_positions(T, H, W)] = False
    assert pad.any()
    for x in g:
        assert np.all(x[:, pad] == 0.0)


def test_pruned_rows_route_their_gradient_to_the_source_row():
    """Pruned-query variant: torch autograd through 'attend the kept rows, then copy each pruned
    row from its source' gives the oracle's gradients (pruned rows' q gets none)."""
    T, H, W = 4, 4, 8  # two full tiles
    rng = np.random.default_rng(6)
    nh, D = 2, 8
    base = rng.standard_normal((1, T * H * W, nh, D))
    q = base + 0.02 * rng.standard_normal(base.shape)  # near-duplicate rows: pruning finds some
    q[:, ::3] = rng.standard_normal(q[:, ::3].shape)
    k, v = (rng.standard_normal(q.shape) for _ in range(2))
    do = rng.standard_normal(q.shape)
    qt, kt, vt, dot = (tiling.tile_scatter(a, T, H, W) for a in (q, k, v, do))
    keep, src, _ = bsa.prune_queries_ratio(qt, 0.5)
    vc = tiling.variable_block_sizes(T, H, W)
    nT = len(vc)
    sets = [[[np.arange(nT) for _ in range(nT)] for _ in range(nh)]]
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = attention_bwd.block_sparse_attention_bwd(qt, kt, vt, vc, sets, scale, dot,
                                                         keep, src)
    for h in range(nh):
        qq, kk, vv = (torch.tensor(a[0, :, h], requires_grad=True) for a in (qt, kt, vt))
        rows = []
        for i in range(nT):
            blk = slice(64 * i, 64 * i + 64)
            kept = np.nonzero(keep[0, h, i])[0]
            o_kept = F.scaled_dot_product_attention(qq[blk][kept][None, None], kk[None, None],
                                                    vv[None, None], scale=scale)[0, 0]
            pos = np.full(64, -1)
            pos[kept] = np.arange(len(kept))
            rows.append(o_kept[torch.from_numpy(pos[src[0, h, i]])])
        out = torch.cat(rows)
        (out * torch.from_numpy(dot[0, :, h])).sum().backward()
        np.testing.assert_allclose(dq[0, :, h], qq.grad.numpy(), rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(dk[0, :, h], kk.grad.numpy(), rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(dv[0, :, h], vv.grad.numpy(), rtol=1e-9, atol=1e-11)
        pruned = ~keep[0, h].reshape(-1)
        assert pruned.any()
        assert np.all(dq[0, pruned, h] == 0.0)
