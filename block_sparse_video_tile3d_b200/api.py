"""Python binding of the libtile3d C ABI: the same calls, on torch CUDA tensors.

PyTorch supplies device memory and the current CUDA stream; every step runs in the library's
CUDA kernels. Each function checks dtypes, shapes, devices and contiguity, passes raw pointers and
raises :class:`Tile3dError` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import functools
import math

import torch

from . import _lib
from ._lib import Geom, Tile3dError, check, lib

__all__ = [
    "Geom", "Tile3dError", "geometry", "tile3d_scatter", "tile3d_gather", "tile_pool",
    "tile3d_scatter_pool",
    "tile_select_topk", "tile_select_mass", "tile_select_workspace_size", "tile_prune_queries",
    "tile_prune_queries_ratio",
    "block_mask_to_index",
    "block_sparse_attn_fwd", "block_sparse_attn_workspace_size", "block_sparse_attn_fwd_lse",
    "block_sparse_attn_bwd", "block_sparse_attn_bwd_workspace_size", "TileSparseAttention",
]


def _geom(B, T, H, W, heads, D, heads_total=0, head0=0) -> Geom:
    return Geom(int(B), int(T), int(H), int(W), int(heads), int(D), int(heads_total), int(head0))


def _slice(nh: int, head0: int, heads):
    """(heads, heads_total, head0) of a call on heads head0 .. head0 + heads - 1 of rows of nh
    heads (every head when ``heads`` is None)."""
    head0 = int(head0)
    heads = nh - head0 if heads is None else int(heads)
    if head0 < 0 or heads < 1 or head0 + heads > nh:
        raise ValueError(f"heads {head0} .. {head0 + heads - 1} lie outside the {nh} heads of a row")
    return heads, nh, head0


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p | None:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, shape=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def geometry(T: int, H: int, W: int, B: int = 1, heads: int = 1, D: int = 64):
    """``(nT, Lp, vc)``: tile count, padded length and the per-tile valid counts (host ints)."""
    nT, Lp, vc = _geometry(int(T), int(H), int(W), int(B), int(heads), int(D))
    return nT, Lp, list(vc)


@functools.lru_cache(maxsize=64)
def _geometry(T, H, W, B, heads, D):
    g = _geom(B, T, H, W, heads, D)
    nT, Lp = ctypes.c_int(), ctypes.c_int()
    check(lib.tile3d_geometry(ctypes.byref(g), ctypes.byref(nT), ctypes.byref(Lp), None))
    vc = (ctypes.c_int32 * nT.value)()
    check(lib.tile3d_geometry(ctypes.byref(g), None, None, ctypes.cast(vc, ctypes.c_void_p)))
    return nT.value, Lp.value, tuple(vc)


def tile3d_scatter(x: torch.Tensor, T: int, H: int, W: int, out: torch.Tensor | None = None,
                   head0: int = 0, heads: int | None = None):
    """Raster ``[B, L, heads, D]`` bf16 -> padded tile order ``[B, Lp, heads, D]`` (zero pads).
    ``head0``/``heads`` restrict the call to those heads of each row (the rest of ``out`` is left
    as it is)."""
    B, L, nh, D = x.shape
    _need(x, "x", torch.bfloat16, (B, T * H * W, nh, D))
    _, Lp, _ = _geometry(int(T), int(H), int(W), B, nh, D)
    if out is None:
        out = torch.empty((B, Lp, nh, D), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", torch.bfloat16, (B, Lp, nh, D))
    hs = _slice(nh, head0, heads)
    g = _geom(B, T, H, W, hs[0], D, hs[1], hs[2])
    check(lib.tile3d_scatter(ctypes.byref(g), _ptr(x), _ptr(out), _stream()))
    return out


def tile3d_gather(y: torch.Tensor, T: int, H: int, W: int, out: torch.Tensor | None = None,
                  head0: int = 0, heads: int | None = None):
    """Padded tile order ``[B, Lp, heads, D]`` bf16 -> raster ``[B, L, heads, D]`` (the heads
    ``head0 .. head0 + heads - 1`` only, when given)."""
    B, Lp, nh, D = y.shape
    _, Lp2, _ = _geometry(int(T), int(H), int(W), B, nh, D)
    _need(y, "y", torch.bfloat16, (B, Lp2, nh, D))
    if out is None:
        out = torch.empty((B, T * H * W, nh, D), dtype=torch.bfloat16, device=y.device)
    _need(out, "out", torch.bfloat16, (B, T * H * W, nh, D))
    hs = _slice(nh, head0, heads)
    g = _geom(B, T, H, W, hs[0], D, hs[1], hs[2])
    check(lib.tile3d_gather(ctypes.byref(g), _ptr(y), _ptr(out), _stream()))
    return out


def tile_pool(y: torch.Tensor, T: int, H: int, W: int, out: torch.Tensor | None = None,
              head0: int = 0, heads: int | None = None):
    """Tile order ``[B, Lp, heads, D]`` bf16 -> per-tile mean ``[B, heads, nT, D]`` fp32 (of the
    heads ``head0 .. head0 + heads - 1`` when given)."""
    B, Lp, nh, D = y.shape
    nT, Lp2, _ = _geometry(int(T), int(H), int(W), B, nh, D)
    _need(y, "y", torch.bfloat16, (B, Lp2, nh, D))
    hs = _slice(nh, head0, heads)
    if out is None:
        out = torch.empty((B, hs[0], nT, D), dtype=torch.float32, device=y.device)
    _need(out, "out", torch.float32, (B, hs[0], nT, D))
    g = _geom(B, T, H, W, hs[0], D, hs[1], hs[2])
    check(lib.tile_pool(ctypes.byref(g), _ptr(y), _ptr(out), _stream()))
    return out


def tile3d_scatter_pool(x: torch.Tensor, T: int, H: int, W: int, out: torch.Tensor | None = None,
                        pooled: torch.Tensor | None = None, head0: int = 0,
                        heads: int | None = None):
    """Scatter and pool in one pass: returns ``(y [B, Lp, heads, D] bf16, pooled [B, heads, nT, D]
    fp32)``, the same as :func:`tile3d_scatter` then :func:`tile_pool`."""
    B, L, nh, D = x.shape
    _need(x, "x", torch.bfloat16, (B, T * H * W, nh, D))
    nT, Lp, _ = _geometry(int(T), int(H), int(W), B, nh, D)
    hs = _slice(nh, head0, heads)
    if out is None:
        out = torch.empty((B, Lp, nh, D), dtype=torch.bfloat16, device=x.device)
    if pooled is None:
        pooled = torch.empty((B, hs[0], nT, D), dtype=torch.float32, device=x.device)
    _need(out, "out", torch.bfloat16, (B, Lp, nh, D))
    _need(pooled, "pooled", torch.float32, (B, hs[0], nT, D))
    g = _geom(B, T, H, W, hs[0], D, hs[1], hs[2])
    check(lib.tile3d_scatter_pool(ctypes.byref(g), _ptr(x), _ptr(out), _ptr(pooled), _stream()))
    return out, pooled


def _sel_out(B, nh, nT, kcap, device, kv_idx, kv_cnt):
    if kv_idx is None:
        kv_idx = torch.empty((B, nh, nT, kcap), dtype=torch.int32, device=device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, nh, nT), dtype=torch.int32, device=device)
    _need(kv_idx, "kv_idx", torch.int32, (B, nh, nT, kcap))
    _need(kv_cnt, "kv_cnt", torch.int32, (B, nh, nT))
    return kv_idx, kv_cnt


def tile_select_workspace_size(B, T, H, W, heads, D) -> int:
    """Bytes of device workspace the selection calls need (the fp32 score rows)."""
    g = _geom(B, T, H, W, heads, D)
    return int(lib.tile_select_workspace_size(ctypes.byref(g)))


def _sel_workspace(g, device, workspace):
    need = int(lib.tile_select_workspace_size(ctypes.byref(g)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def tile_select_topk(pq, pk, T, H, W, k, kv_idx=None, kv_cnt=None, dev_status=None,
                     workspace=None):
    """Top-k key tiles per query tile from pooled ``[B, heads, nT, D]`` fp32 Q and K.
    Returns ``(kv_idx [B, heads, nT, min(k, nT)], kv_cnt [B, heads, nT])`` int32, ascending."""
    B, nh, nT, D = pq.shape
    _need(pq, "pq", torch.float32)
    _need(pk, "pk", torch.float32, pq.shape)
    kcap = min(int(k), nT)
    kv_idx, kv_cnt = _sel_out(B, nh, nT, kcap, pq.device, kv_idx, kv_cnt)
    g = _geom(B, T, H, W, nh, D)
    ws, ws_bytes = _sel_workspace(g, pq.device, workspace)
    check(lib.tile_select_topk(ctypes.byref(g), _ptr(pq), _ptr(pk), int(k), _ptr(kv_idx),
                               _ptr(kv_cnt), _ptr(ws), ws_bytes, _ptr(dev_status), _stream()))
    return kv_idx, kv_cnt


def tile_select_mass(pq, pk, T, H, W, scale, mass, min_k=1, kmax=None, kv_idx=None, kv_cnt=None,
                     dev_status=None, workspace=None):
    """Key tiles by cumulative softmax mass per query tile. Returns ``(kv_idx, kv_cnt)``."""
    B, nh, nT, D = pq.shape
    _need(pq, "pq", torch.float32)
    _need(pk, "pk", torch.float32, pq.shape)
    kmax = nT if kmax is None else int(kmax)
    kv_idx, kv_cnt = _sel_out(B, nh, nT, kmax, pq.device, kv_idx, kv_cnt)
    g = _geom(B, T, H, W, nh, D)
    ws, ws_bytes = _sel_workspace(g, pq.device, workspace)
    check(lib.tile_select_mass(ctypes.byref(g), _ptr(pq), _ptr(pk), float(scale), float(mass),
                               int(min_k), kmax, _ptr(kv_idx), _ptr(kv_cnt), _ptr(ws), ws_bytes,
                               _ptr(dev_status), _stream()))
    return kv_idx, kv_cnt


def tile_prune_queries(qt, T, H, W, cos_thresh, keep=None, src_row=None, pq_kept=None, head0=0,
                       heads=None):
    """BSA query pruning on tile-ordered ``[B, Lp, heads, D]`` bf16 queries (no pad tiles).
    Returns ``(keep u8 [B, heads, nT, 64], src_row u8 [B, heads, nT, 64], pq_kept f32)``."""
    B, Lp, nh_row, D = qt.shape
    nT, Lp2, _ = _geometry(int(T), int(H), int(W), B, nh_row, D)
    _need(qt, "q", torch.bfloat16, (B, Lp2, nh_row, D))
    nh, ht, h0 = _slice(nh_row, head0, heads)
    dev = qt.device
    keep = torch.empty((B, nh, nT, 64), dtype=torch.uint8, device=dev) if keep is None else keep
    src_row = torch.empty((B, nh, nT, 64), dtype=torch.uint8, device=dev) if src_row is None \
        else src_row
    pq_kept = torch.empty((B, nh, nT, D), dtype=torch.float32, device=dev) if pq_kept is None \
        else pq_kept
    _need(keep, "keep", torch.uint8, (B, nh, nT, 64))
    _need(src_row, "src_row", torch.uint8, (B, nh, nT, 64))
    _need(pq_kept, "pq_kept", torch.float32, (B, nh, nT, D))
    g = _geom(B, T, H, W, nh, D, ht, h0)
    check(lib.tile_prune_queries(ctypes.byref(g), _ptr(qt), float(cos_thresh), _ptr(keep),
                                 _ptr(src_row), _ptr(pq_kept), _stream()))
    return keep, src_row, pq_kept


def tile_prune_queries_ratio(qt, T, H, W, keep_ratio, keep=None, src_row=None, pq_kept=None,
                             head0=0, heads=None):
    """BSA query pruning keeping ``max(1, floor(64 * keep_ratio))`` rows per block (the rows least
    similar to the block mean). Same inputs and outputs as ``tile_prune_queries``."""
    B, Lp, nh_row, D = qt.shape
    nT, Lp2, _ = _geometry(int(T), int(H), int(W), B, nh_row, D)
    _need(qt, "q", torch.bfloat16, (B, Lp2, nh_row, D))
    nh, ht, h0 = _slice(nh_row, head0, heads)
    dev = qt.device
    keep = torch.empty((B, nh, nT, 64), dtype=torch.uint8, device=dev) if keep is None else keep
    src_row = torch.empty((B, nh, nT, 64), dtype=torch.uint8, device=dev) if src_row is None \
        else src_row
    pq_kept = torch.empty((B, nh, nT, D), dtype=torch.float32, device=dev) if pq_kept is None \
        else pq_kept
    _need(keep, "keep", torch.uint8, (B, nh, nT, 64))
    _need(src_row, "src_row", torch.uint8, (B, nh, nT, 64))
    _need(pq_kept, "pq_kept", torch.float32, (B, nh, nT, D))
    g = _geom(B, T, H, W, nh, D, ht, h0)
    check(lib.tile_prune_queries_ratio(ctypes.byref(g), _ptr(qt), float(keep_ratio), _ptr(keep),
                                       _ptr(src_row), _ptr(pq_kept), _stream()))
    return keep, src_row, pq_kept


def block_mask_to_index(mask, T, H, W, D, kmax=None, kv_idx=None, kv_cnt=None, dev_status=None):
    """uint8 block map ``[B, heads, nT, nT]`` -> ascending ``(kv_idx, kv_cnt)`` int32."""
    B, nh, nT, nT2 = mask.shape
    _need(mask, "mask", torch.uint8, (B, nh, nT, nT))
    kmax = nT if kmax is None else int(kmax)
    kv_idx, kv_cnt = _sel_out(B, nh, nT, kmax, mask.device, kv_idx, kv_cnt)
    g = _geom(B, T, H, W, nh, D)
    check(lib.block_mask_to_index(ctypes.byref(g), _ptr(mask), kmax, _ptr(kv_idx), _ptr(kv_cnt),
                                  _ptr(dev_status), _stream()))
    return kv_idx, kv_cnt


def block_sparse_attn_workspace_size(B, T, H, W, heads, D, kmax) -> int:
    g = _geom(B, T, H, W, heads, D)
    return int(lib.block_sparse_attn_workspace_size(ctypes.byref(g), int(kmax)))


def block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt, T, H, W, keep=None, src_row=None,
                          softmax_scale=None, causal=False, num_kv_heads=None, out=None,
                          workspace=None, dev_status=None, head0=0, heads=None):
    """Block-sparse attention on tile-ordered ``[B, Lp, heads, D]`` bf16 Q, K, V over the kept
    pairs listed in ``kv_idx``/``kv_cnt`` (of the heads ``head0 .. head0 + heads - 1`` when given;
    the other heads of ``out`` are left as they are). Returns the tile-ordered output."""
    B, Lp, nh_row, D = q.shape
    nT, Lp2, _ = _geometry(int(T), int(H), int(W), B, nh_row, D)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (B, Lp2, nh_row, D))
    nh, ht, h0 = _slice(nh_row, head0, heads)
    _need(kv_cnt, "kv_cnt", torch.int32, (B, nh, nT))
    _need(kv_idx, "kv_idx", torch.int32)
    if kv_idx.dim() != 4 or tuple(kv_idx.shape[:3]) != (B, nh, nT):
        raise ValueError(f"kv_idx must have shape [B, heads, nT, kmax], got {tuple(kv_idx.shape)}")
    kmax = int(kv_idx.shape[3])
    if keep is not None:
        _need(keep, "keep", torch.uint8, (B, nh, nT, 64))
        _need(src_row, "src_row", torch.uint8, (B, nh, nT, 64))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, (B, Lp2, nh_row, D))
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    nkv = nh if num_kv_heads is None else int(num_kv_heads)
    g = _geom(B, T, H, W, nh, D, ht, h0)
    need = int(lib.block_sparse_attn_workspace_size(ctypes.byref(g), kmax))
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.block_sparse_attn_fwd(ctypes.byref(g), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                    _ptr(kv_idx), _ptr(kv_cnt), kmax, _ptr(keep), _ptr(src_row),
                                    scale, int(bool(causal)), nkv, _ptr(workspace), ws_bytes,
                                    _ptr(dev_status), _stream()))
    return out


def _attn_common(q, kv_idx, kv_cnt, T, H, W, keep, src_row, head0, heads):
    B, Lp, nh_row, D = q.shape
    nT, Lp2, _ = _geometry(int(T), int(H), int(W), B, nh_row, D)
    nh, ht, h0 = _slice(nh_row, head0, heads)
    _need(kv_cnt, "kv_cnt", torch.int32, (B, nh, nT))
    _need(kv_idx, "kv_idx", torch.int32)
    if kv_idx.dim() != 4 or tuple(kv_idx.shape[:3]) != (B, nh, nT):
        raise ValueError(f"kv_idx must have shape [B, heads, nT, kmax], got {tuple(kv_idx.shape)}")
    if keep is not None:
        _need(keep, "keep", torch.uint8, (B, nh, nT, 64))
        _need(src_row, "src_row", torch.uint8, (B, nh, nT, 64))
    return B, Lp2, nh_row, D, nT, nh, ht, h0


def block_sparse_attn_fwd_lse(q, k, v, kv_idx, kv_cnt, T, H, W, keep=None, src_row=None,
                              softmax_scale=None, out=None, lse=None, workspace=None,
                              dev_status=None, head0=0, heads=None):
    """:func:`block_sparse_attn_fwd` that also returns each query row's log-sum-exp (fp32
    ``[B, heads, Lp]``, natural log), for the backward pass. Returns ``(out, lse)``."""
    B, Lp, nh_row, D, nT, nh, ht, h0 = _attn_common(q, kv_idx, kv_cnt, T, H, W, keep, src_row,
                                                    head0, heads)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (B, Lp, nh_row, D))
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, nh, Lp), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(out, "out", torch.bfloat16, (B, Lp, nh_row, D))
    _need(lse, "lse", torch.float32, (B, nh, Lp))
    kmax = int(kv_idx.shape[3])
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    g = _geom(B, T, H, W, nh, D, ht, h0)
    need = int(lib.block_sparse_attn_workspace_size(ctypes.byref(g), kmax))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    check(lib.block_sparse_attn_fwd_lse(ctypes.byref(g), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                        _ptr(lse), _ptr(kv_idx), _ptr(kv_cnt), kmax, _ptr(keep),
                                        _ptr(src_row), scale, 0, nh, _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _ptr(dev_status), _stream()))
    return out, lse


def block_sparse_attn_bwd_workspace_size(B, T, H, W, heads, D, kmax, heads_total=0, head0=0):
    g = _geom(B, T, H, W, heads, D, heads_total, head0)
    return int(lib.block_sparse_attn_bwd_workspace_size(ctypes.byref(g), int(kmax)))


def block_sparse_attn_bwd(q, k, v, o, dout, lse, kv_idx, kv_cnt, T, H, W, keep=None,
                          src_row=None, softmax_scale=None, dq=None, dk=None, dv=None,
                          workspace=None, dev_status=None, head0=0, heads=None):
    """Gradients ``(dq, dk, dv)`` (bf16, tile order) of :func:`block_sparse_attn_fwd` for the
    output gradient ``dout``, with ``o`` and ``lse`` from :func:`block_sparse_attn_fwd_lse`."""
    B, Lp, nh_row, D, nT, nh, ht, h0 = _attn_common(q, kv_idx, kv_cnt, T, H, W, keep, src_row,
                                                    head0, heads)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _need(t, name, torch.bfloat16, (B, Lp, nh_row, D))
    _need(lse, "lse", torch.float32, (B, nh, Lp))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, torch.bfloat16, (B, Lp, nh_row, D))
    kmax = int(kv_idx.shape[3])
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    g = _geom(B, T, H, W, nh, D, ht, h0)
    need = int(lib.block_sparse_attn_bwd_workspace_size(ctypes.byref(g), kmax))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    check(lib.block_sparse_attn_bwd(ctypes.byref(g), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                    _ptr(dout), _ptr(lse), _ptr(kv_idx), _ptr(kv_cnt), kmax,
                                    _ptr(keep), _ptr(src_row), scale, 0, nh, _ptr(dq), _ptr(dk),
                                    _ptr(dv), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(),
                                    _ptr(dev_status), _stream()))
    return dq, dk, dv


class TileSparseAttention:
    """The whole hot path for one geometry, with its device buffers allocated once.

    ``mode``: ``"topk"`` (keep ``topk`` key tiles per query tile by pooled score), ``"mass"``
    (cumulative softmax mass ``mass`` with floor ``min_k``), ``"bsa"`` (query pruning at cosine
    ``cos_thresh`` — or, with ``keep_ratio`` given, a fixed ``max(1, floor(64 * keep_ratio))`` rows
    per block — then mass selection from the kept queries) or ``"mask"`` (a fixed uint8 block map
    ``[B, heads, nT, nT]``).

    ``forward(q, k, v)`` takes raster ``[B, L, heads_total, D]`` bf16 CUDA tensors and returns the
    raster output; one call = scatter Q, K, V -> coarse selection -> block-sparse attention ->
    gather. With ``head0`` and ``heads_total`` given, the instance works on heads
    ``head0 .. head0 + heads - 1`` of rows of ``heads_total`` heads and writes only those heads'
    columns of the output: one layer's heads shared out over GPUs, each rank with its own range.
    """

    def __init__(self, B, T, H, W, heads, D, mode="topk", topk=None, mass=0.9, min_k=1,
                 cos_thresh=0.95, mask=None, keep_ratio=None, device="cuda", head0=0,
                 heads_total=None):
        self.B, self.T, self.H, self.W, self.heads, self.D = B, T, H, W, heads, D
        self.heads_total = heads if heads_total is None else int(heads_total)
        self.head0 = int(head0)
        _slice(self.heads_total, self.head0, heads)
        self.mode = mode
        self.nT, self.Lp, self.vc = geometry(T, H, W, B, heads, D)
        self.scale = 1.0 / math.sqrt(D)
        self.topk, self.mass, self.min_k, self.cos_thresh = topk, mass, min_k, cos_thresh
        self.keep_ratio = keep_ratio
        dev = torch.device(device)
        shp = (B, self.Lp, self.heads_total, D)
        self.qt = torch.empty(shp, dtype=torch.bfloat16, device=dev)
        self.kt = torch.empty(shp, dtype=torch.bfloat16, device=dev)
        self.vt = torch.empty(shp, dtype=torch.bfloat16, device=dev)
        self.ot = torch.empty(shp, dtype=torch.bfloat16, device=dev)
        self.pq = torch.empty((B, heads, self.nT, D), dtype=torch.float32, device=dev)
        self.pk = torch.empty((B, heads, self.nT, D), dtype=torch.float32, device=dev)
        if mode == "topk":
            if not topk:
                raise ValueError("topk mode needs topk >= 1")
            self.kmax = min(int(topk), self.nT)
        else:
            self.kmax = self.nT
        self.kv_idx = torch.empty((B, heads, self.nT, self.kmax), dtype=torch.int32, device=dev)
        self.kv_cnt = torch.empty((B, heads, self.nT), dtype=torch.int32, device=dev)
        self.keep = self.src_row = None
        if mode == "bsa":
            self.keep = torch.empty((B, heads, self.nT, 64), dtype=torch.uint8, device=dev)
            self.src_row = torch.empty((B, heads, self.nT, 64), dtype=torch.uint8, device=dev)
        self.mask = None
        if mode == "mask":
            if mask is None:
                raise ValueError("mask mode needs a block mask")
            self.mask = mask.to(device=dev, dtype=torch.uint8).contiguous()
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        ws = block_sparse_attn_workspace_size(B, T, H, W, heads, D, self.kmax)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        self.sel_workspace = None
        if mode != "mask":
            ws = tile_select_workspace_size(B, T, H, W, heads, D)
            self.sel_workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def stages(self, q, k, v, out=None):
        """The hot path as an ordered list of ``(name, launch)`` pairs; each ``launch()`` enqueues
        one library call on the current stream. ``forward`` runs them in order; a profiler or a
        benchmark can interleave its own events between them."""
        T, H, W = self.T, self.H, self.W
        hr = {"head0": self.head0, "heads": self.heads}  # this instance's heads of a row
        if out is None:
            out = torch.empty((self.B, T * H * W, self.heads_total, self.D), dtype=torch.bfloat16,
                              device=q.device)
        self._out = out
        if self.mode == "mask":
            st = [
                ("scatter_q", lambda: tile3d_scatter(q, T, H, W, self.qt, **hr)),
                ("scatter_k", lambda: tile3d_scatter(k, T, H, W, self.kt, **hr)),
                ("scatter_v", lambda: tile3d_scatter(v, T, H, W, self.vt, **hr)),
                ("mask_to_index", lambda: block_mask_to_index(
                    self.mask, T, H, W, self.D, self.kmax, self.kv_idx, self.kv_cnt,
                    self.status)),
            ]
        else:
            if self.mode == "bsa":  # queries are pooled over kept rows, by the pruning kernel
                st = [("scatter_q", lambda: tile3d_scatter(q, T, H, W, self.qt, **hr))]
            else:
                st = [("scatter_pool_q",
                       lambda: tile3d_scatter_pool(q, T, H, W, self.qt, self.pq, **hr))]
            st += [
                ("scatter_pool_k", lambda: tile3d_scatter_pool(k, T, H, W, self.kt, self.pk,
                                                               **hr)),
                ("scatter_v", lambda: tile3d_scatter(v, T, H, W, self.vt, **hr)),
            ]
            if self.mode == "bsa" and self.keep_ratio is not None:
                st.append(("prune_q", lambda: tile_prune_queries_ratio(
                    self.qt, T, H, W, self.keep_ratio, self.keep, self.src_row, self.pq, **hr)))
            elif self.mode == "bsa":
                st.append(("prune_q", lambda: tile_prune_queries(
                    self.qt, T, H, W, self.cos_thresh, self.keep, self.src_row, self.pq, **hr)))
            if self.mode == "topk":
                st.append(("select_topk", lambda: tile_select_topk(
                    self.pq, self.pk, T, H, W, self.topk, self.kv_idx, self.kv_cnt, self.status,
                    self.sel_workspace)))
            else:
                st.append(("select_mass", lambda: tile_select_mass(
                    self.pq, self.pk, T, H, W, self.scale, self.mass, self.min_k, self.kmax,
                    self.kv_idx, self.kv_cnt, self.status, self.sel_workspace)))
        st.append(("attention", lambda: block_sparse_attn_fwd(
            self.qt, self.kt, self.vt, self.kv_idx, self.kv_cnt, T, H, W, keep=self.keep,
            src_row=self.src_row, softmax_scale=self.scale, out=self.ot,
            workspace=self.workspace, dev_status=self.status, **hr)))
        st.append(("gather", lambda: tile3d_gather(self.ot, T, H, W, out, **hr)))
        return st

    def forward(self, q, k, v, out=None):
        st = self.stages(q, k, v, out)
        for _, launch in st:
            launch()
        return self._out

    __call__ = forward

    def device_status(self) -> int:
        """The OR of every T3D_DEV_* bit the kernels have recorded since construction (syncs)."""
        return int(self.status.item())
