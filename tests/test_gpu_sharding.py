"""GPU: one layer shared out by head. Instances that each take a head range (head0, heads) of the
same full-width [B, L, heads_total, D] rows, writing into one output, must reproduce the
single-instance result bit for bit (every (batch, head) is independent, and each kernel's
arithmetic for a head does not depend on which other heads the call covers)."""
import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import TileSparseAttention, workloads
from block_sparse_video_tile3d_b200.sharding import head_partition
from oracle import pipeline
from tests.helpers import assert_attn_close, f64

pytestmark = pytest.mark.gpu


def _case(mode):
    if mode == "topk":
        w = workloads.WORKLOADS["tiny"].with_(B=2, T=9, H=10, W=13, heads=5, D=128, k=7)
        return w, dict(mode="topk", topk=w.k), None
    if mode == "bsa":
        w = workloads.WORKLOADS["bsa"].with_(T=8, H=8, W=12, heads=3)
        return w, dict(mode="bsa", mass=w.mass, min_k=w.min_kv, cos_thresh=w.cos_thresh), None
    w = workloads.WORKLOADS["ragged_sliding"].with_(B=1, T=9, H=10, W=13, heads=3)
    return w, dict(mode="mask"), workloads.block_mask(w)


@pytest.mark.parametrize("mode", ["topk", "bsa", "mask"])
@pytest.mark.parametrize("world", [2, 3])
def test_head_ranges_reassemble_bit_exactly(mode, world):
    w, kw, mask = _case(mode)
    q, k, v = workloads.make_qkv(w)
    if mode == "bsa":
        q = workloads.make_structured_queries(w, q)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    whole = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mask=mask, **kw)
    want = whole(qd, kd, vd)
    got = torch.full_like(want, float("nan"))
    for rank in range(world):
        h0, n = head_partition(w.heads, world, rank)
        if n == 0:
            continue
        part = TileSparseAttention(w.B, w.T, w.H, w.W, n, w.D, head0=h0, heads_total=w.heads,
                                   mask=None if mask is None else mask[:, h0:h0 + n], **kw)
        part(qd, kd, vd, out=got)
        assert part.device_status() == 0
    assert torch.equal(got, want)


def test_head_range_matches_the_oracle():
    """A middle head range on its own, against the oracle run on those heads."""
    w, kw, _ = _case("topk")
    q, k, v = workloads.make_qkv(w, seed=5)
    h0, n = 1, 3
    part = TileSparseAttention(w.B, w.T, w.H, w.W, n, w.D, head0=h0, heads_total=w.heads, **kw)
    out = torch.zeros((w.B, w.L, w.heads, w.D), dtype=torch.bfloat16, device="cuda")
    part(q.cuda(), k.cuda(), v.cuda(), out=out)
    got = f64(out)
    assert np.all(got[:, :, :h0] == 0) and np.all(got[:, :, h0 + n:] == 0)  # untouched heads
    hs = slice(h0, h0 + n)
    ref = pipeline.forward(q[:, :, hs], k[:, :, hs], v[:, :, hs], w.T, w.H, w.W, "topk",
                           scale=w.scale, topk=w.k)
    sets = [[[part.kv_idx[b, h, i, :int(part.kv_cnt[b, h, i])].cpu().numpy()
              for i in range(w.nT)] for h in range(n)] for b in range(w.B)]
    same = all(np.array_equal(np.sort(sets[b][h][i]), ref["sets"][b][h][i])
               for b in range(w.B) for h in range(n) for i in range(w.nT))
    if same:
        assert_attn_close(got[:, :, hs], ref["o"])
    else:  # a near tie selected differently: the oracle with the GPU's lists
        from oracle import attention
        ot = attention.block_sparse_attention(ref["qt"], ref["kt"], ref["vt"], ref["vc"], sets,
                                              w.scale)
        from oracle import tiling
        assert_attn_close(got[:, :, hs], tiling.tile_gather(ot, w.T, w.H, w.W))
