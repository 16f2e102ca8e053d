"""CPU oracle for tile-sparse 3D-tiled video attention: test infrastructure, not the product.

A plain, slow, fp64 numpy restatement of what the hot path computes, written from the FastVideo
attention-backend documentation pages (``bsa_attn``, ``sla``, ``video_sparse_attn`` and
``video_sparse_attn_h3``). It shares no code with the CUDA library and imports nothing from the
package. Only the test suite, the smoke check and the benchmark's CPU-baseline leg may call it; the
product path never does.

Modules:
  tiling     raster <-> padded tile order, per-tile valid counts
  pool       mean pooling of each tile over its valid tokens
  select     tile-to-tile scores, top-k and cumulative-mass KV tile selection
  bsa        query pruning and reconstruction of the bidirectional sparse attention variant
  attention  softmax attention restricted to the kept (query tile, key tile) pairs
  attention_bwd  its gradients with respect to Q, K and V (the backward pass)
  pipeline   the four stages chained, as the hot path runs them
  packed     packed multi-region sequences (dense segments plus video regions), tiles of 64 or 128

Every function is pinned by a CPU test against something other than itself (closed forms,
brute force on tiny inputs, invariants, library routines for the dense special case).
"""
from . import tiling, pool, select, bsa, attention, attention_bwd, pipeline, packed  # noqa: F401
