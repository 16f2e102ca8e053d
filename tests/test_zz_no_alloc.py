"""The allocation-free attention entry point, block_sparse_attn_fwd_noalloc, through the C ABI.

It exists for callers that cannot allocate device memory (a plugin whose host framework owns the
allocator, a runtime with a memory budget fixed at start-up, a loop that cannot afford cudaMalloc's
synchronisation): it runs the same attention kernel with its scratch in a fixed array inside the
library instead of a caller's workspace. Two calls in a row must match block_sparse_attn_fwd (the
entry point with a workspace) within the attention tolerance; the second call also shows that the
shared scratch is reset between calls. This file is collected last, and needs no other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from block_sparse_video_tile3d_b200 import block_sparse_attn_fwd, tile3d_scatter
from block_sparse_video_tile3d_b200._lib import Geom, check, lib
from tests.helpers import assert_attn_close, f64

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    B, T, H, W, heads, D = 2, 9, 10, 13, 3, 128  # ragged grid: 36 tiles, some of 8 tokens
    nT = 36
    gen = torch.Generator().manual_seed(31)
    q, k, v = (torch.randn((B, T * H * W, heads, D), generator=gen).to(torch.bfloat16).cuda()
               for _ in range(3))
    qt, kt, vt = (tile3d_scatter(x, T, H, W) for x in (q, k, v))
    rng = np.random.default_rng(32)
    kmax = 12
    idx = np.zeros((B, heads, nT, kmax), dtype=np.int32)
    cnt = rng.integers(0, kmax + 1, size=(B, heads, nT)).astype(np.int32)  # uneven, some empty
    for b in range(B):
        for h in range(heads):
            for i in range(nT):
                idx[b, h, i, :cnt[b, h, i]] = rng.choice(nT, cnt[b, h, i], replace=False)
    kv_idx, kv_cnt = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    want = block_sparse_attn_fwd(qt, kt, vt, kv_idx, kv_cnt, T, H, W)
    geom = Geom(B, T, H, W, heads, D)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(qt, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        check(lib.block_sparse_attn_fwd_noalloc(
            ctypes.byref(geom), _p(qt), _p(kt), _p(vt), _p(out), _p(kv_idx), _p(kv_cnt), kmax,
            None, None, 1.0 / math.sqrt(D), 0, heads, _p(status), stream))
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}"
        assert_attn_close(f64(out), f64(want), what=f"no-alloc call {call}")


def test_noalloc_rejects_like_the_workspace_entry_point():
    geom = Geom(1, 4, 8, 8, 2, 64)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation
    args = (fake, fake, fake, fake, fake, fake, 2, None, None)
    assert lib.block_sparse_attn_fwd_noalloc(ctypes.byref(geom), *args, 0.125, 1, 2, None,
                                             None) == 2  # causal: T3D_ERR_UNSUPPORTED
    assert lib.block_sparse_attn_fwd_noalloc(ctypes.byref(geom), *args, 0.2, 0, 2, None,
                                             None) == 1  # scale: T3D_ERR_INVALID
