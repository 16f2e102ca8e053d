"""B200-native tile-sparse attention for video diffusion transformers.

The hot path (3D tile scatter, tile pooling, KV tile selection, block-sparse attention, untile)
runs in the CUDA kernels of ``libtile3d.so`` behind the C ABI of ``include/tile3d.h``; this package
is its Python binding. Importing it without the built library raises ``ImportError``.
"""
from .api import (  # noqa: F401
    Geom, Tile3dError, TileSparseAttention, block_mask_to_index, block_sparse_attn_fwd,
    block_sparse_attn_workspace_size, geometry, tile3d_gather, tile3d_scatter, tile_pool,
    tile_prune_queries, tile_select_mass, tile_select_topk,
)

__version__ = "0.1.0"
