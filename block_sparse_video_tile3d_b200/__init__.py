"""B200-native tile-sparse attention for video diffusion transformers.

The hot path (3D tile scatter, tile pooling, KV tile selection, block-sparse attention, untile)
runs in the CUDA kernels of ``libtile3d.so`` behind the C ABI of ``include/tile3d.h``; this package
is its Python binding. The library is loaded on first use of any call below; if it is missing (or
out of date) that first use raises ``ImportError`` — there is no CPU fallback. Building it:
``python -m block_sparse_video_tile3d_b200.build``.
"""
__version__ = "0.1.0"

_API = (
    "Geom", "Tile3dError", "TileSparseAttention", "block_mask_to_index", "block_sparse_attn_fwd",
    "block_sparse_attn_workspace_size", "block_sparse_attn_fwd_lse", "block_sparse_attn_bwd",
    "block_sparse_attn_bwd_workspace_size", "geometry", "tile3d_gather", "tile3d_scatter",
    "tile3d_scatter_pool", "tile_pool", "tile_prune_queries", "tile_prune_queries_ratio",
    "tile_select_mass", "tile_select_topk", "tile_select_workspace_size",
)
__all__ = list(_API)


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
