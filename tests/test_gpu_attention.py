"""GPU parity of block_sparse_attn_fwd with the oracle's kept sets fed in directly, plus edge
cases: ragged tiles, D = 64 and 128, empty and unordered lists, out-of-range indices, the
pruned-query variant, and the full-size workloads on sampled query tiles."""
import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import block_sparse_attn_fwd, tile3d_scatter, workloads
from block_sparse_video_tile3d_b200._lib import (T3D_DEV_INDEX_RANGE, T3D_DEV_OVERFLOW,
                                                  T3D_DEV_TIMEOUT, check, lib)
from oracle import attention, bsa, select, tiling
from tests.helpers import assert_attn_close, f64

pytestmark = pytest.mark.gpu


def _qkv(B, T, H, W, heads, D, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return tuple((torch.randn((B, T * H * W, heads, D), generator=g) * scale).to(torch.bfloat16)
                 for _ in range(3))


def _lists(sets, B, heads, nT, kmax, order="asc", fill=-7):
    idx = np.full((B, heads, nT, kmax), fill, dtype=np.int32)
    cnt = np.zeros((B, heads, nT), dtype=np.int32)
    for b in range(B):
        for h in range(heads):
            for i in range(nT):
                s = np.asarray(sets[b][h][i], dtype=np.int32)
                if order == "desc":
                    s = s[::-1]
                elif order == "shuffle":
                    s = np.random.default_rng(b * 1000 + h * 100 + i).permutation(s)
                idx[b, h, i, :len(s)] = s
                cnt[b, h, i] = len(s)
    return torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


def _run(q, k, v, T, H, W, sets, kmax=None, order="asc", keep=None, src=None):
    B, L, heads, D = q.shape
    nT = len(tiling.variable_block_sizes(T, H, W))
    kmax = kmax or max(1, max(len(s) for bb in sets for hh in bb for s in hh))
    kv_idx, kv_cnt = _lists(sets, B, heads, nT, kmax, order)
    qt, kt, vt = (tile3d_scatter(x.cuda(), T, H, W) for x in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kp = None if keep is None else torch.from_numpy(keep.astype(np.uint8)).cuda()
    sp = None if src is None else torch.from_numpy(src.astype(np.uint8)).cuda()
    ot = block_sparse_attn_fwd(qt, kt, vt, kv_idx, kv_cnt, T, H, W, keep=kp, src_row=sp,
                               dev_status=status)
    return f64(ot), int(status.item())


def _oracle(q, k, v, T, H, W, sets, keep=None, src=None):
    D = q.shape[-1]
    vc = tiling.variable_block_sizes(T, H, W)
    qt, kt, vt = (tiling.tile_scatter(f64(x), T, H, W) for x in (q, k, v))
    return attention.block_sparse_attention(qt, kt, vt, vc, sets, 1.0 / np.sqrt(D), keep=keep,
                                            src=src)


def _random_sets(B, heads, nT, density, seed, diag=True):
    rng = np.random.default_rng(seed)
    m = rng.random((B, heads, nT, nT)) < density
    if diag:
        m[:, :, np.arange(nT), np.arange(nT)] = True
    return select.map_to_sets(m.astype(np.uint8))


@pytest.mark.parametrize("B,T,H,W,heads,D,density", [
    (1, 4, 8, 8, 2, 64, 0.5),
    (2, 9, 10, 13, 2, 128, 0.3),
    (1, 9, 10, 13, 3, 64, 0.3),
    (1, 5, 6, 7, 2, 128, 1.0),  # dense limit on a ragged grid
    (1, 1, 1, 1, 1, 64, 1.0),   # one token
])
def test_attention_random_sets(B, T, H, W, heads, D, density):
    q, k, v = _qkv(B, T, H, W, heads, D, seed=T * 17 + D)
    nT = len(tiling.variable_block_sizes(T, H, W))
    sets = _random_sets(B, heads, nT, density, seed=nT)
    got, st = _run(q, k, v, T, H, W, sets)
    want = _oracle(q, k, v, T, H, W, sets)
    assert st == 0
    assert_attn_close(got, want)
    pad = ~tiling.valid_slot_mask(T, H, W)
    assert np.all(got[:, pad] == 0.0)


@pytest.mark.parametrize("order", ["desc", "shuffle"])
def test_attention_list_order_irrelevant(order):
    B, T, H, W, heads, D = 1, 9, 10, 13, 2, 128
    q, k, v = _qkv(B, T, H, W, heads, D, seed=3)
    sets = _random_sets(B, heads, 36, 0.4, seed=4)
    got, _ = _run(q, k, v, T, H, W, sets, order=order)
    assert_attn_close(got, _oracle(q, k, v, T, H, W, sets))


def test_attention_empty_rows_and_large_magnitudes():
    B, T, H, W, heads, D = 1, 8, 8, 8, 2, 128
    q, k, _ = _qkv(B, T, H, W, heads, D, seed=5, scale=4.0)  # logits of std ~16: peaky softmax
    _, _, v = _qkv(B, T, H, W, heads, D, seed=6)
    sets = _random_sets(B, heads, 8, 0.5, seed=6)
    sets[0][0][3] = np.zeros(0, dtype=np.int64)
    sets[0][1][7] = np.zeros(0, dtype=np.int64)
    got, _ = _run(q, k, v, T, H, W, sets)
    want = _oracle(q, k, v, T, H, W, sets)
    assert np.all(got[0, 64 * 3:64 * 4, 0] == 0.0) and np.all(got[0, 64 * 7:, 1] == 0.0)
    assert_attn_close(got, want)


@pytest.mark.parametrize("D", [64, 128])
def test_attention_out_of_range_index_is_skipped_and_reported(D):
    B, T, H, W, heads = 1, 8, 8, 8, 1
    q, k, v = _qkv(B, T, H, W, heads, D, seed=7)
    sets = _random_sets(B, heads, 8, 0.5, seed=8)
    kv_idx, kv_cnt = _lists(sets, B, heads, 8, 8)
    idx = kv_idx.cpu()
    row = next(i for i in range(8) if len(sets[0][0][i]) < 8)
    idx[0, 0, row, int(kv_cnt[0, 0, row])] = 99  # append an out-of-range index to that row
    kv_cnt[0, 0, row] += 1
    qt, kt, vt = (tile3d_scatter(x.cuda(), T, H, W) for x in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ot = block_sparse_attn_fwd(qt, kt, vt, idx.cuda(), kv_cnt, T, H, W, dev_status=status)
    assert int(status.item()) & T3D_DEV_INDEX_RANGE
    assert_attn_close(f64(ot), _oracle(q, k, v, T, H, W, sets))


def test_attention_list_counts_outside_capacity():
    """kv_cnt above kmax reads the first kmax entries (T3D_DEV_OVERFLOW); a negative kv_cnt reads as
    an empty list (T3D_DEV_INDEX_RANGE, zero output rows)."""
    B, T, H, W, heads, D = 1, 8, 8, 8, 2, 128
    q, k, v = _qkv(B, T, H, W, heads, D, seed=12)
    sets = _random_sets(B, heads, 8, 0.6, seed=13)
    kmax = 8
    kv_idx, kv_cnt = _lists(sets, B, heads, 8, kmax)
    row = next(i for i in range(8) if len(sets[0][0][i]) >= 3)
    cnt = kv_cnt.cpu()
    cnt[0, 0, row] = kmax + 3          # claims more entries than a row holds
    cnt[0, 1, 5] = -4                  # a negative count
    want_sets = [[list(sets[0][0]), list(sets[0][1])]]
    want_sets[0][0][row] = np.asarray(kv_idx[0, 0, row].cpu().numpy(), dtype=np.int64)
    want_sets[0][1][5] = np.zeros(0, dtype=np.int64)
    # the row's kmax entries: its own list followed by fill values, which are out of range and
    # skipped (so the range bit is expected too)
    want_sets[0][0][row] = want_sets[0][0][row][(want_sets[0][0][row] >= 0)
                                                & (want_sets[0][0][row] < 8)]
    qt, kt, vt = (tile3d_scatter(x.cuda(), T, H, W) for x in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ot = block_sparse_attn_fwd(qt, kt, vt, kv_idx, cnt.cuda(), T, H, W, dev_status=status)
    st = int(status.item())
    assert st & T3D_DEV_OVERFLOW and st & T3D_DEV_INDEX_RANGE
    got = f64(ot)
    assert np.all(got[0, 64 * 5:64 * 6, 1] == 0.0)
    assert_attn_close(got, _oracle(q, k, v, T, H, W, want_sets))


def test_attention_uneven_lists_balanced_queue():
    """Units of very different lengths (every tile kept for one query tile in five, one to three
    for the rest) over more units than SMs: the dynamic unit queue must cover every unit once."""
    B, T, H, W, heads, D = 1, 9, 10, 13, 8, 128
    nT = 36
    q, k, v = _qkv(B, T, H, W, heads, D, seed=14)
    rng = np.random.default_rng(15)
    sets = [[[np.arange(nT) if (h * nT + i) % 5 == 0 else
              np.sort(rng.choice(nT, int(rng.integers(1, 4)), replace=False))
              for i in range(nT)] for h in range(heads)]]
    got, st = _run(q, k, v, T, H, W, sets)
    assert st == 0
    assert_attn_close(got, _oracle(q, k, v, T, H, W, sets))


def test_attention_repeated_calls_share_workspace():
    """The queue counter in the workspace is reset by every call: two calls with one workspace
    give the same output, bit for bit."""
    B, T, H, W, heads, D = 1, 9, 10, 13, 6, 64
    q, k, v = _qkv(B, T, H, W, heads, D, seed=16)
    sets = _random_sets(B, heads, 36, 0.3, seed=17)
    kv_idx, kv_cnt = _lists(sets, B, heads, 36, 36)
    qt, kt, vt = (tile3d_scatter(x.cuda(), T, H, W) for x in (q, k, v))
    ws = torch.full((256,), 0x7f, dtype=torch.uint8, device="cuda")  # not zero on entry
    o1 = block_sparse_attn_fwd(qt, kt, vt, kv_idx, kv_cnt, T, H, W, workspace=ws)
    o2 = block_sparse_attn_fwd(qt, kt, vt, kv_idx, kv_cnt, T, H, W, workspace=ws)
    assert torch.equal(o1, o2)
    assert_attn_close(f64(o1), _oracle(q, k, v, T, H, W, sets))


def test_attention_bounded_wait_gives_up_cleanly():
    """With the pipeline wait limit cut to 200 clock cycles the first wait that is not already
    satisfied gives up: the kernel must record T3D_DEV_TIMEOUT, let its copies and MMAs in flight
    finish, free its tensor memory and return; the next call at the normal limit must be exact."""
    B, T, H, W, heads, D = 1, 8, 8, 8, 2, 128
    q, k, v = _qkv(B, T, H, W, heads, D, seed=18)
    sets = _random_sets(B, heads, 8, 0.5, seed=19)
    try:
        check(lib.t3d_testing_set_wait_cycles(200))
        _, st = _run(q, k, v, T, H, W, sets)
    finally:
        check(lib.t3d_testing_set_wait_cycles(0))
    torch.cuda.synchronize()  # the context is still usable
    assert st & T3D_DEV_TIMEOUT
    got, st2 = _run(q, k, v, T, H, W, sets)
    assert st2 == 0
    assert_attn_close(got, _oracle(q, k, v, T, H, W, sets))


def test_attention_pruned_queries():
    w = workloads.WORKLOADS["bsa"].with_(T=8, H=8, W=12, heads=2)
    q, k, v = workloads.make_qkv(w)
    q = workloads.make_structured_queries(w, q)
    oqt = tiling.tile_scatter(f64(q), w.T, w.H, w.W)
    keep, src, _ = bsa.prune_queries(oqt, w.cos_thresh)
    assert (~keep).sum() > 50
    sets = _random_sets(1, w.heads, w.nT, 0.5, seed=9)
    got, _ = _run(q, k, v, w.T, w.H, w.W, sets, keep=keep, src=src)
    want = _oracle(q, k, v, w.T, w.H, w.W, sets, keep=keep, src=src)
    assert_attn_close(got, want)


def _sampled_check(q, k, v, T, H, W, sets_fn, samples, seed):
    """Full-size GPU run; the oracle recomputes the sampled (batch, head, query tile) triples on
    single-head slices."""
    B, L, heads, D = q.shape
    nT = len(tiling.variable_block_sizes(T, H, W))
    sets = sets_fn()
    got, st = _run(q, k, v, T, H, W, sets)
    assert st == 0
    rng = np.random.default_rng(seed)
    picks = [(int(rng.integers(B)), int(rng.integers(heads)), int(rng.integers(nT)))
             for _ in range(samples)] + [(B - 1, heads - 1, nT - 1), (0, 0, 0)]
    vc = tiling.variable_block_sizes(T, H, W)
    by_head = {}
    for b, h, i in picks:
        by_head.setdefault((b, h), []).append(i)
    for (b, h), tiles in by_head.items():
        sl = lambda x: f64(x[b:b + 1, :, h:h + 1])  # noqa: E731
        qt, kt, vt = (tiling.tile_scatter(sl(x), T, H, W) for x in (q, k, v))
        sub = [[sets[b][h]]]
        want = attention.block_sparse_attention(qt, kt, vt, vc, sub, 1.0 / np.sqrt(D),
                                                q_tiles=[(0, 0, i) for i in tiles])
        for i in tiles:
            rows = slice(64 * i, 64 * i + 64)
            assert_attn_close(got[b, rows, h], want[0, rows, 0], what=f"tile {(b, h, i)}")


def test_attention_small_full_size_sampled():
    w = workloads.WORKLOADS["small"]
    q, k, v = workloads.make_qkv(w)
    _sampled_check(q, k, v, w.T, w.H, w.W,
                   lambda: _random_sets(w.B, w.heads, w.nT, w.k / w.nT, seed=10), 24, seed=1)


@pytest.mark.parametrize("name", ["ragged_sliding", "ragged_random"])
def test_attention_ragged_masks_sampled(name):
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.make_qkv(w)
    mask = workloads.block_mask(w).numpy()
    _sampled_check(q, k, v, w.T, w.H, w.W, lambda: select.map_to_sets(mask), 24, seed=2)
