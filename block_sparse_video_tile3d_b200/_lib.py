"""ctypes binding of libtile3d.so (the C ABI declared in include/tile3d.h and
include/tile3d_packed.h).

Argument marshalling only. The library must have been built in-tree
(``python -m block_sparse_video_tile3d_b200.build``); importing this module without it raises
``ImportError`` — there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtile3d.so")

T3D_OK, T3D_ERR_INVALID, T3D_ERR_UNSUPPORTED, T3D_ERR_CUDA, T3D_ERR_DEVICE = range(5)
T3D_DEV_INDEX_RANGE, T3D_DEV_OVERFLOW, T3D_DEV_TIMEOUT = 0x1, 0x2, 0x4

STATUS_NAMES = {0: "T3D_OK", 1: "T3D_ERR_INVALID", 2: "T3D_ERR_UNSUPPORTED", 3: "T3D_ERR_CUDA",
                4: "T3D_ERR_DEVICE"}


class Geom(ctypes.Structure):
    """``t3d_geom``: B, T, H, W, heads, D, heads_total (0: = heads), head0."""
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("heads", ctypes.c_int), ("D", ctypes.c_int), ("heads_total", ctypes.c_int),
                ("head0", ctypes.c_int)]


class Segment(ctypes.Structure):
    """``t3d_segment``: a dense run (rows > 0) or a video region of t x h x w tokens (rows = 0)."""
    _fields_ = [("rows", ctypes.c_int), ("t", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int)]


class PackedLayout(ctypes.Structure):
    """``t3d_packed_layout``."""
    _fields_ = [("n_tiles", ctypes.c_int), ("rows", ctypes.c_int), ("n_prefix", ctypes.c_int),
                ("n_regions", ctypes.c_int)]


class Packed(ctypes.Structure):
    """``t3d_packed``: a packed tile buffer as the device calls see it."""
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("D", ctypes.c_int),
                ("heads_total", ctypes.c_int), ("head0", ctypes.c_int), ("tile_elems", ctypes.c_int),
                ("n_tiles", ctypes.c_int), ("rows", ctypes.c_int), ("slot_row", ctypes.c_void_p),
                ("vc", ctypes.c_void_p)]


T3D_PACKED_EXEMPT, T3D_PACKED_COMPETE, T3D_PACKED_DENSE = 0, 1, 2

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t
_G = ctypes.POINTER(Geom)
_PK = ctypes.POINTER(Packed)

# name -> (restype, argtypes), in the order of include/tile3d.h, then include/tile3d_testing.h
SIGNATURES = {
    "t3d_last_error_string": (ctypes.c_char_p, []),
    "t3d_version": (ctypes.c_char_p, []),
    "tile3d_geometry": (_I, [_G, ctypes.POINTER(_I), ctypes.POINTER(_I), _P]),
    "tile3d_scatter": (_I, [_G, _P, _P, _P]),
    "tile3d_gather": (_I, [_G, _P, _P, _P]),
    "tile_pool": (_I, [_G, _P, _P, _P]),
    "tile3d_scatter_pool": (_I, [_G, _P, _P, _P, _P]),
    "tile_select_topk": (_I, [_G, _P, _P, _I, _P, _P, _P, _S, _P, _P]),
    "tile_select_mass": (_I, [_G, _P, _P, _F, _F, _I, _I, _P, _P, _P, _S, _P, _P]),
    "tile_select_workspace_size": (_S, [_G]),
    "tile_prune_queries": (_I, [_G, _P, _F, _P, _P, _P, _P]),
    "tile_prune_queries_ratio": (_I, [_G, _P, _F, _P, _P, _P, _P]),
    "block_mask_to_index": (_I, [_G, _P, _I, _P, _P, _P, _P]),
    "block_sparse_attn_fwd": (_I, [_G, _P, _P, _P, _P, _P, _P, _I, _P, _P, _F, _I, _I, _P, _S,
                                   _P, _P]),
    "block_sparse_attn_workspace_size": (_S, [_G, _I]),
    "block_sparse_attn_fwd_lse": (_I, [_G, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _F, _I, _I, _P,
                                       _S, _P, _P]),
    "block_sparse_attn_bwd": (_I, [_G, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _F, _I, _I,
                                   _P, _P, _P, _P, _S, _P, _P]),
    "block_sparse_attn_bwd_workspace_size": (_S, [_G, _I]),
    "block_sparse_attn_fwd_noalloc": (_I, [_G, _P, _P, _P, _P, _P, _P, _I, _P, _P, _F, _I, _I,
                                           _P, _P]),
    # include/tile3d_packed.h
    "t3d_packed_geometry": (_I, [ctypes.POINTER(Segment), _I, _I, _I, _I,
                                 ctypes.POINTER(PackedLayout), _P, _P, _P]),
    "tile3d_scatter_packed": (_I, [_PK, _P, _P, _P]),
    "tile3d_gather_packed": (_I, [_PK, _P, _P, _P]),
    "tile_pool_packed": (_I, [_PK, _P, _P, _P]),
    "tile3d_scatter_pool_packed": (_I, [_PK, _P, _P, _P, _P]),
    "tile_select_packed_capacity": (_I, [_I, _I, _I, _I, _P, _P, ctypes.POINTER(_I)]),
    "tile_select_packed": (_I, [_PK, _P, _P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _S, _P, _P]),
    "tile_select_packed_workspace_size": (_S, [_PK]),
    "block_sparse_attn_fwd_packed": (_I, [_PK, _P, _P, _P, _P, _P, _P, _I, _F, _P, _S, _P, _P]),
    "block_sparse_attn_packed_workspace_size": (_S, [_PK, _I]),
    # include/tile3d_testing.h
    "t3d_testing_set_wait_cycles": (_I, [ctypes.c_longlong]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libtile3d.so not found at {LIB_PATH}; build it with "
            "`python -m block_sparse_video_tile3d_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class Tile3dError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def check(status: int) -> None:
    if status != T3D_OK:
        raise Tile3dError(status, lib.t3d_last_error_string().decode())
