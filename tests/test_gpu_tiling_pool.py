"""GPU parity: tile scatter / gather (bit-exact) and tile pooling (fp32 vs the fp64 oracle)."""
import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import tile3d_gather, tile3d_scatter, tile_pool, workloads
from oracle import pool, tiling
from tests.helpers import f64

pytestmark = pytest.mark.gpu

GRIDS = [  # (B, T, H, W, heads, D)
    (1, 4, 8, 8, 2, 64),      # tiny workload shape
    (2, 5, 6, 7, 3, 64),      # ragged in every dimension, several tiles
    (1, 9, 10, 13, 2, 128),   # ragged, D = 128
    (1, 1, 1, 1, 1, 64),      # a single token
    (1, 16, 32, 56, 12, 128),  # small video-DiT layer, full size
    (2, 21, 30, 52, 24, 128),  # ragged stress layer, full size
]


def _rand_bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * 2 + 0.5).to(torch.bfloat16)


@pytest.mark.parametrize("B,T,H,W,heads,D", GRIDS)
def test_scatter_gather_bit_exact(B, T, H, W, heads, D):
    x = _rand_bf16((B, T * H * W, heads, D), seed=T * 131 + W)
    xd = x.cuda()
    y = tile3d_scatter(xd, T, H, W)
    want = tiling.tile_scatter(x.view(torch.int16).numpy(), T, H, W)  # exact: raw bf16 bits
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy(), want)
    back = tile3d_gather(y, T, H, W)
    assert torch.equal(back.cpu().view(torch.int16), x.view(torch.int16))


def test_scatter_overwrites_stale_pads():
    B, T, H, W, heads, D = 1, 5, 6, 7, 2, 64
    x = _rand_bf16((B, T * H * W, heads, D), seed=3).cuda()
    Lp = tiling.padded_length(T, H, W)
    y = torch.full((B, Lp, heads, D), 7.0, dtype=torch.bfloat16, device="cuda")
    tile3d_scatter(x, T, H, W, out=y)
    valid = torch.from_numpy(tiling.valid_slot_mask(T, H, W))
    assert torch.all(y.cpu()[:, ~valid] == 0)


@pytest.mark.parametrize("B,T,H,W,heads,D", GRIDS)
def test_pool_matches_oracle(B, T, H, W, heads, D):
    x = _rand_bf16((B, T * H * W, heads, D), seed=T * 7 + H)
    y = tile3d_scatter(x.cuda(), T, H, W)
    got = f64(tile_pool(y, T, H, W))
    vc = tiling.variable_block_sizes(T, H, W)
    hs = range(heads) if heads <= 3 else [0, heads - 1]
    for h in hs:
        want = pool.tile_mean_pool(tiling.tile_scatter(f64(x[:, :, h:h + 1]), T, H, W), vc)
        np.testing.assert_allclose(got[:, h:h + 1], want, rtol=1e-5, atol=2e-6)


def test_pool_workload_offsets_small():
    w = workloads.WORKLOADS["small"]
    q, _, _ = workloads.make_qkv(w)
    y = tile3d_scatter(q.cuda(), w.T, w.H, w.W)
    got = f64(tile_pool(y, w.T, w.H, w.W))
    vc = tiling.variable_block_sizes(w.T, w.H, w.W)
    want = pool.tile_mean_pool(tiling.tile_scatter(f64(q[:, :, 5:6]), w.T, w.H, w.W), vc)
    np.testing.assert_allclose(got[:, 5:6], want, rtol=1e-5, atol=2e-6)


@pytest.mark.parametrize("B,T,H,W,heads,D", GRIDS)
def test_scatter_pool_fused_matches(B, T, H, W, heads, D):
    from block_sparse_video_tile3d_b200 import tile3d_scatter_pool
    x = _rand_bf16((B, T * H * W, heads, D), seed=T * 5 + W)
    xd = x.cuda()
    y, pooled = tile3d_scatter_pool(xd, T, H, W)
    want = tiling.tile_scatter(x.view(torch.int16).numpy(), T, H, W)
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy(), want)
    vc = tiling.variable_block_sizes(T, H, W)
    got = f64(pooled)
    hs = range(heads) if heads <= 3 else [0, heads - 1]
    for h in hs:
        ref = pool.tile_mean_pool(tiling.tile_scatter(f64(x[:, :, h:h + 1]), T, H, W), vc)
        np.testing.assert_allclose(got[:, h:h + 1], ref, rtol=1e-5, atol=2e-6)
