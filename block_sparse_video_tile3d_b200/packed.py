"""Python binding of the packed multi-region calls (include/tile3d_packed.h) on torch CUDA tensors.

FastVideo API docs, video_sparse_attn_h3 page, build(): a packed sequence is a list of dense
segments (row counts) and video regions (latent shapes, divided by the patch size); the last
region is the generated video, earlier ones are reference videos with their own keep rate; tiles
hold 64 or 128 tokens. Argument marshalling only: the geometry is computed by the library on the
host, every device step runs in its CUDA kernels.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import check, lib
from .api import _need, _ptr, _slice, _stream

__all__ = [
    "TILE_SHAPES", "PackedGeometry", "span_keep_rates", "tile3d_scatter_packed",
    "tile3d_gather_packed", "tile_pool_packed", "tile3d_scatter_pool_packed", "tile_select_packed",
    "block_sparse_attn_fwd_packed",
    "PackedTileSparseAttention",
]

# Tile shapes (t, h, w) by token count; 128 is this library's reading (the page's table is not
# printed).
TILE_SHAPES = {64: (4, 4, 4), 128: (4, 4, 8)}

EXEMPT, COMPETE, DENSE = _lib.T3D_PACKED_EXEMPT, _lib.T3D_PACKED_COMPETE, _lib.T3D_PACKED_DENSE


def span_keep_rates(n_regions: int, sparsity: float, ref_keep_rate=None, exempt: bool = True):
    """Keep rate of every region, reference regions first and the generated one last (build()):
    reference regions need ``ref_keep_rate``; compete mode allows one region; a sparsity of zero
    or below keeps every region dense."""
    if n_regions > 1:
        if ref_keep_rate is None:
            raise ValueError(f"{n_regions - 1} reference-video region(s) need ref_keep_rate")
        if not exempt:
            raise ValueError("compete mode supports the generated-video region only")
    if float(sparsity) <= 0.0:
        return [1.0] * n_regions
    refs = [] if n_regions == 1 else [float(ref_keep_rate)] * (n_regions - 1)
    return refs + [1.0 - float(sparsity)]


class PackedGeometry:
    """Tile buffer of one packed sequence: host layout plus the device slot map and valid counts.

    ``segments``: packed order; an int is a dense segment's row count (0 is dropped), a
    ``(t, h, w)`` tuple a video region's latent shape, which ``patch`` must divide."""

    def __init__(self, segments, patch=(1, 1, 1), tile_size: int = 64, tile_shape=None,
                 device="cuda"):
        segs = []
        for s in segments:
            if isinstance(s, tuple):
                if any(int(v) <= 0 or int(v) % int(p) for v, p in zip(s, patch)):
                    raise ValueError(f"region {tuple(s)} is not a positive multiple of patch {tuple(patch)}")
                t, h, w = (int(v) // int(p) for v, p in zip(s, patch))
                segs.append(_lib.Segment(0, t, h, w))
            elif int(s) > 0:
                segs.append(_lib.Segment(int(s), 0, 0, 0))
        if tile_shape is None:
            if int(tile_size) not in TILE_SHAPES:
                raise ValueError(f"tile_size must be one of {sorted(TILE_SHAPES)}, got {tile_size}")
            tile_shape = TILE_SHAPES[int(tile_size)]
        self.tile_shape = tuple(int(v) for v in tile_shape)
        arr = (_lib.Segment * max(len(segs), 1))(*segs)
        lay = _lib.PackedLayout()
        check(lib.t3d_packed_geometry(arr, len(segs), *self.tile_shape, ctypes.byref(lay), None, None,
                                      None))
        self.E = math.prod(self.tile_shape)
        self.n_tiles, self.rows = lay.n_tiles, lay.rows
        self.n_prefix, self.n_regions = lay.n_prefix, lay.n_regions
        spans = (ctypes.c_int32 * (2 * lay.n_regions))()
        vc = (ctypes.c_int32 * lay.n_tiles)()
        slot = (ctypes.c_int32 * (lay.n_tiles * self.E))()
        check(lib.t3d_packed_geometry(arr, len(segs), *self.tile_shape, ctypes.byref(lay),
                                      ctypes.cast(spans, ctypes.c_void_p),
                                      ctypes.cast(vc, ctypes.c_void_p),
                                      ctypes.cast(slot, ctypes.c_void_p)))
        self.spans_flat = list(spans)
        self.spans = [(spans[2 * r], spans[2 * r + 1]) for r in range(lay.n_regions)]
        self.vc = list(vc)
        self.slot_row_host = list(slot)
        self.slot_row = torch.tensor(self.slot_row_host, dtype=torch.int32, device=device)
        self.vc_dev = torch.tensor(self.vc, dtype=torch.int32, device=device)

    @property
    def buffer_rows(self) -> int:
        return self.n_tiles * self.E

    def struct(self, B: int, heads: int, D: int, heads_total: int = 0, head0: int = 0) -> _lib.Packed:
        return _lib.Packed(int(B), int(heads), int(D), int(heads_total), int(head0), self.E,
                           self.n_tiles, self.rows, self.slot_row.data_ptr(), self.vc_dev.data_ptr())


def _call_struct(geo: PackedGeometry, x: torch.Tensor, head0: int, heads):
    B, _, nh, D = x.shape
    heads, heads_total, head0 = _slice(nh, head0, heads)
    return geo.struct(B, heads, D, heads_total, head0), B, nh, D, heads


def tile3d_scatter_packed(x: torch.Tensor, geo: PackedGeometry, out: torch.Tensor | None = None,
                          head0: int = 0, heads: int | None = None) -> torch.Tensor:
    """Packed ``[B, rows, nh, D]`` bf16 -> buffer ``[B, n_tiles * E, nh, D]`` (pads zero)."""
    B, L, nh, D = x.shape
    _need(x, "x", torch.bfloat16, (B, geo.rows, nh, D))
    if out is None:
        out = torch.empty((B, geo.buffer_rows, nh, D), dtype=torch.bfloat16, device=x.device)
    _need(out, "out", torch.bfloat16, (B, geo.buffer_rows, nh, D))
    p, *_ = _call_struct(geo, x, head0, heads)
    check(lib.tile3d_scatter_packed(ctypes.byref(p), _ptr(x), _ptr(out), _stream()))
    return out


def tile3d_gather_packed(y: torch.Tensor, geo: PackedGeometry, out: torch.Tensor | None = None,
                         head0: int = 0, heads: int | None = None) -> torch.Tensor:
    """Buffer ``[B, n_tiles * E, nh, D]`` -> packed ``[B, rows, nh, D]``."""
    B, _, nh, D = y.shape
    _need(y, "y", torch.bfloat16, (B, geo.buffer_rows, nh, D))
    if out is None:
        out = torch.empty((B, geo.rows, nh, D), dtype=torch.bfloat16, device=y.device)
    _need(out, "out", torch.bfloat16, (B, geo.rows, nh, D))
    p, *_ = _call_struct(geo, y, head0, heads)
    check(lib.tile3d_gather_packed(ctypes.byref(p), _ptr(y), _ptr(out), _stream()))
    return out


def tile_pool_packed(y: torch.Tensor, geo: PackedGeometry, out: torch.Tensor | None = None,
                     head0: int = 0, heads: int | None = None) -> torch.Tensor:
    """Buffer order -> per-tile means ``[B, heads, n_tiles, D]`` fp32."""
    B, _, nh, D = y.shape
    _need(y, "y", torch.bfloat16, (B, geo.buffer_rows, nh, D))
    p, B, nh, D, hh = _call_struct(geo, y, head0, heads)
    if out is None:
        out = torch.empty((B, hh, geo.n_tiles, D), dtype=torch.float32, device=y.device)
    _need(out, "out", torch.float32, (B, hh, geo.n_tiles, D))
    check(lib.tile_pool_packed(ctypes.byref(p), _ptr(y), _ptr(out), _stream()))
    return out


def tile3d_scatter_pool_packed(x: torch.Tensor, geo: PackedGeometry, out: torch.Tensor | None = None,
                               pooled: torch.Tensor | None = None, head0: int = 0,
                               heads: int | None = None):
    """``tile3d_scatter_packed`` and ``tile_pool_packed`` in one pass: ``(y, pooled)``."""
    B, L, nh, D = x.shape
    _need(x, "x", torch.bfloat16, (B, geo.rows, nh, D))
    p, B, nh, D, hh = _call_struct(geo, x, head0, heads)
    if out is None:
        out = torch.empty((B, geo.buffer_rows, nh, D), dtype=torch.bfloat16, device=x.device)
    if pooled is None:
        pooled = torch.empty((B, hh, geo.n_tiles, D), dtype=torch.float32, device=x.device)
    _need(out, "out", torch.bfloat16, (B, geo.buffer_rows, nh, D))
    _need(pooled, "pooled", torch.float32, (B, hh, geo.n_tiles, D))
    check(lib.tile3d_scatter_pool_packed(ctypes.byref(p), _ptr(x), _ptr(out), _ptr(pooled), _stream()))
    return out, pooled


def _spans_args(geo: PackedGeometry, keep_rates, mode: int):
    spans = (ctypes.c_int32 * len(geo.spans_flat))(*geo.spans_flat)
    rates = (ctypes.c_double * geo.n_regions)(*[float(r) for r in keep_rates])
    cap = ctypes.c_int()
    check(lib.tile_select_packed_capacity(geo.n_tiles, int(mode), geo.n_prefix, geo.n_regions,
                                          ctypes.cast(spans, ctypes.c_void_p),
                                          ctypes.cast(rates, ctypes.c_void_p), ctypes.byref(cap)))
    return spans, rates, cap.value


def tile_select_packed(pq: torch.Tensor, pk: torch.Tensor, geo: PackedGeometry, keep_rates,
                       mode: int = EXEMPT, kmax: int | None = None,
                       workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                       kv_idx: torch.Tensor | None = None, kv_cnt: torch.Tensor | None = None):
    """Kept tiles per query tile: ``(kv_idx [B, heads, n_tiles, kmax], kv_cnt [B, heads, n_tiles])``
    int32, lists ascending. ``keep_rates``: one per region (``span_keep_rates``). ``kv_idx`` /
    ``kv_cnt`` / ``workspace`` may be given to reuse buffers."""
    B, hh, nT, D = pq.shape
    _need(pq, "pq", torch.float32, (B, hh, geo.n_tiles, D))
    _need(pk, "pk", torch.float32, (B, hh, geo.n_tiles, D))
    if len(keep_rates) != geo.n_regions:
        raise ValueError(f"{geo.n_regions} keep rates needed, got {len(keep_rates)}")
    spans, rates, cap = _spans_args(geo, keep_rates, mode)
    kmax = (cap if kmax is None else int(kmax)) if kv_idx is None else kv_idx.shape[-1]
    p = geo.struct(B, hh, D)
    need = lib.tile_select_packed_workspace_size(ctypes.byref(p))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=pq.device)
    if kv_idx is None:
        kv_idx = torch.empty((B, hh, geo.n_tiles, kmax), dtype=torch.int32, device=pq.device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, hh, geo.n_tiles), dtype=torch.int32, device=pq.device)
    _need(kv_idx, "kv_idx", torch.int32, (B, hh, geo.n_tiles, kmax))
    _need(kv_cnt, "kv_cnt", torch.int32, (B, hh, geo.n_tiles))
    check(lib.tile_select_packed(ctypes.byref(p), _ptr(pq), _ptr(pk), int(mode), geo.n_prefix,
                                 geo.n_regions, ctypes.cast(spans, ctypes.c_void_p),
                                 ctypes.cast(rates, ctypes.c_void_p), kmax, _ptr(kv_idx),
                                 _ptr(kv_cnt), _ptr(workspace), workspace.numel(),
                                 _ptr(dev_status), _stream()))
    return kv_idx, kv_cnt


def block_sparse_attn_fwd_packed(q, k, v, kv_idx, kv_cnt, geo: PackedGeometry,
                                 out: torch.Tensor | None = None, head0: int = 0,
                                 heads: int | None = None, workspace: torch.Tensor | None = None,
                                 dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Attention over the kept tile pairs of a packed buffer (buffer-order bf16 tensors)."""
    B, _, nh, D = q.shape
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, name, torch.bfloat16, (B, geo.buffer_rows, nh, D))
    p, B, nh, D, hh = _call_struct(geo, q, head0, heads)
    kmax = kv_idx.shape[-1]
    _need(kv_idx, "kv_idx", torch.int32, (B, hh, geo.n_tiles, kmax))
    _need(kv_cnt, "kv_cnt", torch.int32, (B, hh, geo.n_tiles))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, (B, geo.buffer_rows, nh, D))
    need = lib.block_sparse_attn_packed_workspace_size(ctypes.byref(p), kmax)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    check(lib.block_sparse_attn_fwd_packed(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                           _ptr(kv_idx), _ptr(kv_cnt), kmax, 1.0 / math.sqrt(D),
                                           _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                           _stream()))
    return out


class PackedTileSparseAttention:
    """The whole path for one packed sequence: scatter, pool, per-region selection, attention,
    gather. ``dense_layer`` keeps every tile (the page's dense_layers)."""

    def __init__(self, segments, heads: int, D: int, patch=(1, 1, 1), tile_size: int = 64,
                 sparsity: float = 0.875, ref_keep_rate=None, exempt: bool = True,
                 dense_layer: bool = False, device="cuda"):
        self.geo = PackedGeometry(segments, patch, tile_size, device=device)
        self.heads, self.D = int(heads), int(D)
        self.keep_rates = span_keep_rates(self.geo.n_regions, sparsity, ref_keep_rate, exempt)
        self.mode = DENSE if dense_layer else (EXEMPT if exempt else COMPETE)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.kv_idx = self.kv_cnt = None
        self._bufs = None

    def _buffers(self, q: torch.Tensor):
        B = q.shape[0]
        key = (B, q.device)
        if self._bufs is None or self._bufs[0] != key:
            g, dev = self.geo, q.device
            buf = lambda: torch.empty((B, g.buffer_rows, self.heads, self.D), dtype=torch.bfloat16,  # noqa: E731
                                      device=dev)
            pooled = lambda: torch.empty((B, self.heads, g.n_tiles, self.D), dtype=torch.float32,  # noqa: E731
                                         device=dev)
            _, _, cap = _spans_args(g, self.keep_rates, self.mode)
            d = {"qt": buf(), "kt": buf(), "vt": buf(), "ot": buf(), "pq": pooled(), "pk": pooled(),
                 "kv_idx": torch.empty((B, self.heads, g.n_tiles, cap), dtype=torch.int32, device=dev),
                 "kv_cnt": torch.empty((B, self.heads, g.n_tiles), dtype=torch.int32, device=dev)}
            p = g.struct(B, self.heads, self.D)
            d["ws_sel"] = torch.empty(lib.tile_select_packed_workspace_size(ctypes.byref(p)),
                                      dtype=torch.uint8, device=dev)
            d["ws_attn"] = torch.empty(lib.block_sparse_attn_packed_workspace_size(ctypes.byref(p), cap),
                                       dtype=torch.uint8, device=dev)
            self._bufs = (key, d)
            self.kv_idx, self.kv_cnt = d["kv_idx"], d["kv_cnt"]
        return self._bufs[1]

    def stages(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor):
        """The path as named launches over persistent buffers (for timing each stage)."""
        g, d = self.geo, self._buffers(q)
        return [
            ("scatter_pool_q", lambda: tile3d_scatter_pool_packed(q, g, out=d["qt"], pooled=d["pq"])),
            ("scatter_pool_k", lambda: tile3d_scatter_pool_packed(k, g, out=d["kt"], pooled=d["pk"])),
            ("scatter_v", lambda: tile3d_scatter_packed(v, g, out=d["vt"])),
            ("select", lambda: tile_select_packed(d["pq"], d["pk"], g, self.keep_rates, self.mode,
                                                  workspace=d["ws_sel"], dev_status=self.status,
                                                  kv_idx=d["kv_idx"], kv_cnt=d["kv_cnt"])),
            ("attention", lambda: block_sparse_attn_fwd_packed(
                d["qt"], d["kt"], d["vt"], d["kv_idx"], d["kv_cnt"], g, out=d["ot"],
                workspace=d["ws_attn"], dev_status=self.status)),
            ("gather", lambda: tile3d_gather_packed(d["ot"], g, out=out)),
        ]

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 out: torch.Tensor | None = None) -> torch.Tensor:
        if out is None:
            out = torch.empty_like(q)
        for _, launch in self.stages(q, k, v, out):
            launch()
        return out
