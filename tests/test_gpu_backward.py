"""GPU parity of the backward pass (block_sparse_attn_bwd) with the oracle's gradients
(oracle/attention_bwd.py): ragged grids at D = 64 and 128, uneven and empty lists, key tiles that
no query tile keeps, pruned queries (BSA), a head range of full-width rows, and one head of the
full-size small layer. The forward's log-sum-exp comes from block_sparse_attn_fwd_lse.

Tolerance (the workload definition fixes none for gradients): the kernels round P, dS and the
effective dO to bf16 (relative error 2^-9) as MMA operands and the gradients to bf16; dS sums to
zero over a row's keys, so dK sums terms that largely cancel and its error relative to its own size
can exceed the forward's. Gradients are compared with max-abs error at most 1e-2 of the largest
reference magnitude and relative L2 error at most 1e-2 (measured on the ragged grids: 4e-3 and
2.4e-3, about what rounding each gradient to bf16 alone gives)."""
import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import (block_sparse_attn_bwd, block_sparse_attn_fwd,
                                            block_sparse_attn_fwd_lse, tile3d_scatter, workloads)
from oracle import attention, attention_bwd, bsa, select, tiling
from tests.helpers import f64

pytestmark = pytest.mark.gpu

BWD_MAX_ABS_REL = 1e-2  # of the largest reference magnitude
BWD_REL_L2 = 1e-2


def assert_grad_close(got, want, what):
    diff = np.abs(got - want)
    scale = max(float(np.abs(want).max()), 1e-30)
    rel = float(np.sqrt((diff ** 2).sum()) / max(np.sqrt((want ** 2).sum()), 1e-30))
    assert diff.max() <= BWD_MAX_ABS_REL * scale, f"{what}: max abs {diff.max():.3e} vs {scale:.3e}"
    assert rel <= BWD_REL_L2, f"{what}: relative L2 {rel:.3e}"
    return rel


def _qkv(B, T, H, W, heads, D, seed):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn((B, T * H * W, heads, D), generator=g).to(torch.bfloat16)
                 for _ in range(4))


def _lists(sets, B, heads, nT, kmax):
    idx = np.zeros((B, heads, nT, kmax), dtype=np.int32)
    cnt = np.zeros((B, heads, nT), dtype=np.int32)
    for b in range(B):
        for h in range(heads):
            for i in range(nT):
                s = np.asarray(sets[b][h][i], dtype=np.int32)
                idx[b, h, i, :len(s)] = s
                cnt[b, h, i] = len(s)
    return torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


def _run(q, k, v, do, T, H, W, sets, keep=None, src=None):
    B, L, heads, D = q.shape
    nT = len(tiling.variable_block_sizes(T, H, W))
    kmax = max(1, max(len(s) for bb in sets for hh in bb for s in hh))
    kv_idx, kv_cnt = _lists(sets, B, heads, nT, kmax)
    qt, kt, vt, dot = (tile3d_scatter(x.cuda(), T, H, W) for x in (q, k, v, do))
    kp = None if keep is None else torch.from_numpy(keep.astype(np.uint8)).cuda()
    sp = None if src is None else torch.from_numpy(src.astype(np.uint8)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = block_sparse_attn_fwd_lse(qt, kt, vt, kv_idx, kv_cnt, T, H, W, keep=kp, src_row=sp,
                                       dev_status=status)
    # the forward with the log-sum-exp is the plain forward, bit for bit
    o_plain = block_sparse_attn_fwd(qt, kt, vt, kv_idx, kv_cnt, T, H, W, keep=kp, src_row=sp)
    assert torch.equal(o, o_plain)
    dq, dk, dv = block_sparse_attn_bwd(qt, kt, vt, o, dot, lse, kv_idx, kv_cnt, T, H, W, keep=kp,
                                       src_row=sp, dev_status=status)
    assert int(status.item()) == 0
    return f64(dq), f64(dk), f64(dv), f64(lse)


def _oracle(q, k, v, do, T, H, W, sets, keep=None, src=None):
    D = q.shape[-1]
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt, dot = (tiling.tile_scatter(f64(x), T, H, W) for x in (q, k, v, do))
    return attention_bwd.block_sparse_attention_bwd(qt, kt, vt, vc, sets, 1.0 / np.sqrt(D), dot,
                                                    keep=keep, src=src)


def _random_sets(B, heads, nT, density, seed, empty_rows=()):
    rng = np.random.default_rng(seed)
    m = rng.random((B, heads, nT, nT)) < density
    m[:, :, np.arange(nT), np.arange(nT)] = True
    for (b, h, i) in empty_rows:
        m[b, h, i] = False
    return select.map_to_sets(m.astype(np.uint8))


@pytest.mark.parametrize("D", [64, 128])
def test_backward_ragged_random_sets(D):
    B, T, H, W, heads = 2, 9, 10, 13, 2
    q, k, v, do = _qkv(B, T, H, W, heads, D, seed=40 + D)
    sets = _random_sets(B, heads, 36, 0.3, seed=41, empty_rows=[(0, 1, 5), (1, 0, 35)])
    got = _run(q, k, v, do, T, H, W, sets)
    want = _oracle(q, k, v, do, T, H, W, sets)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got[:3], want):
        assert_grad_close(g_, w_, name)
    pad = ~tiling.valid_slot_mask(T, H, W)
    for g_ in got[:3]:
        assert np.all(g_[:, pad] == 0.0)
    # an empty query tile gets zero dq; the lse of its rows is -inf
    assert np.all(got[0][0, 64 * 5:64 * 6, 1] == 0.0)
    assert np.all(np.isneginf(got[3][0, 1, 64 * 5:64 * 6]))


def test_backward_key_tiles_nobody_keeps():
    B, T, H, W, heads, D = 1, 8, 8, 8, 2, 128
    q, k, v, do = _qkv(B, T, H, W, heads, D, seed=50)
    sets = [[[np.array([0, 2]) for _ in range(8)] for _ in range(heads)]]  # only tiles 0 and 2
    got = _run(q, k, v, do, T, H, W, sets)
    want = _oracle(q, k, v, do, T, H, W, sets)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got[:3], want):
        assert_grad_close(g_, w_, name)
    unused = [t for t in range(8) if t not in (0, 2)]
    for t in unused:
        assert np.all(got[1][0, 64 * t:64 * t + 64] == 0) and np.all(got[2][0, 64 * t:64 * t + 64] == 0)


def test_backward_pruned_queries():
    w = workloads.WORKLOADS["bsa"].with_(T=8, H=8, W=12, heads=2)
    q, k, v = workloads.make_qkv(w)
    q = workloads.make_structured_queries(w, q)
    do = _qkv(w.B, w.T, w.H, w.W, w.heads, w.D, seed=51)[0]
    oqt = tiling.tile_scatter(f64(q), w.T, w.H, w.W)
    keep, src, _ = bsa.prune_queries(oqt, w.cos_thresh)
    assert (~keep).sum() > 50
    sets = _random_sets(1, w.heads, w.nT, 0.4, seed=52)
    got = _run(q, k, v, do, w.T, w.H, w.W, sets, keep=keep, src=src)
    want = _oracle(q, k, v, do, w.T, w.H, w.W, sets, keep=keep, src=src)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got[:3], want):
        assert_grad_close(g_, w_, name)
    # pruned rows get no query gradient
    B, Lp = 1, 64 * w.nT
    pruned = np.zeros((B, Lp, w.heads), dtype=bool)
    for h in range(w.heads):
        pruned[0, :, h] = ~keep[0, h].reshape(-1)
    assert np.all(got[0][pruned] == 0.0)


def test_backward_matches_torch_autograd_dense():
    """Every tile kept: the oracle is pinned to torch autograd through SDPA; the GPU must agree with
    the same reference (through the oracle) on a ragged grid."""
    B, T, H, W, heads, D = 1, 5, 6, 7, 2, 128
    q, k, v, do = _qkv(B, T, H, W, heads, D, seed=53)
    nT = len(tiling.variable_block_sizes(T, H, W))
    sets = [[[np.arange(nT) for _ in range(nT)] for _ in range(heads)]]
    got = _run(q, k, v, do, T, H, W, sets)
    want = _oracle(q, k, v, do, T, H, W, sets)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got[:3], want):
        assert_grad_close(g_, w_, name)


def test_backward_small_layer_one_head():
    """The full-size small layer (12 heads, 448 tiles, 56 kept per query tile); head 7 checked
    against the oracle on a single-head slice."""
    w = workloads.WORKLOADS["small"]
    q, k, v = workloads.make_qkv(w)
    do = _qkv(w.B, w.T, w.H, w.W, w.heads, w.D, seed=54)[0]
    rng = np.random.default_rng(55)
    sets = [[[np.sort(rng.choice(w.nT, w.k, replace=False)) for _ in range(w.nT)]
             for _ in range(w.heads)]]
    dq, dk, dv, _ = _run(q, k, v, do, w.T, w.H, w.W, sets)
    h = 7
    sl = lambda x: x[:, :, h:h + 1]  # noqa: E731
    want = _oracle(sl(q), sl(k), sl(v), sl(do), w.T, w.H, w.W, [[sets[0][h]]])
    for name, g_, w_ in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        assert_grad_close(g_[:, :, h:h + 1], w_, name)
