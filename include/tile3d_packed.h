/*
 * tile3d_packed.h — packed multi-region sequences and 128-token tiles (libtile3d.so).
 *
 * FastVideo API docs, video_sparse_attn_h3 page:
 *  - build(): a packed sequence lists, in packed order, dense segments (a row count) and video
 *    regions (a latent shape the patch size divides; the region's tokens form a t x h x w grid);
 *    at least one region; the last region is the generated video and follows VSA_sparsity, every
 *    earlier one is a reference video keeping ref_keep_rate of its tiles; compete mode
 *    (exempt = False) allows the generated region only; a sparsity of zero or below keeps every
 *    region dense; the metadata records num_prefix_tiles, video_tile_spans and a sparsity per
 *    span; tile sizes 64 and 128 exist.
 *  - tile(): every packed row goes to one slot of a padded tile buffer whose pads stay zero.
 * fastvideo.attention.backends page, sla.get_block_map: min(K, int(ratio * K)) tiles of a
 * candidate set of K are kept, by pooled score.
 *
 * Readings where the page is silent (the bodies of its geometry helpers are not printed):
 *  - Buffer order: the dense segments' tiles first (they are the num_prefix_tiles), each segment
 *    cut into consecutive runs of tile_elems rows with a partial last run, segments in packed
 *    order; then each video region's tiles in packed order, the region tiled as a single video
 *    (tiles t-major, then h, then w; raster order inside a tile; partial edge tiles). A tile's
 *    valid rows fill its first vc slots.
 *  - The tile shape is the caller's: 4 x 4 x 4 for 64 tokens; this library's Python binding
 *    uses 4 x 4 x 8 for 128 (the page's shape table is not printed).
 *  - Selection, exempt mode: every query tile keeps every prefix tile; a prefix query tile keeps
 *    every tile; any other query tile keeps, inside each region r separately, the
 *    min(n_r, int(keep_r * n_r)) tiles of r with the highest scores (ties: lower index). Compete
 *    mode: every query tile keeps the min(n, int(keep * n)) best of all n tiles (keep = the last
 *    rate). Dense: every tile for every query tile.
 *  - Attention over the buffer is the single-video one (one softmax over the valid keys of the
 *    kept tiles; pad query rows output zero).
 *
 * Conventions as in tile3d.h: device pointers owned by the caller, bf16 activations
 * [B, rows, heads_total, D] (packed order) and [B, n_tiles * tile_elems, heads_total, D] (buffer
 * order) of which a call works on heads head0 .. head0 + heads - 1, asynchronous calls on
 * `stream`, a t3d_status result, kernel-found errors in the caller's dev_status word.
 */
#ifndef TILE3D_PACKED_H_
#define TILE3D_PACKED_H_

#include "tile3d.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One segment of a packed sequence: a dense run of `rows` rows (rows > 0, t = h = w = 0), or a
 * video region of t x h x w tokens (rows = 0; t, h, w >= 1), the latent shape already divided by
 * the patch size. */
typedef struct {
  int rows;
  int t, h, w;
} t3d_segment;

/* Sizes of a packed geometry. */
typedef struct {
  int n_tiles;   /* tiles of the buffer */
  int rows;      /* packed rows (the sequence length) */
  int n_prefix;  /* dense tiles, which come first */
  int n_regions; /* video regions */
} t3d_packed_layout;

/*
 * t3d_packed_geometry — the tile buffer of a packed sequence (the readings above).
 *   segs, n_segs: in (host), the sequence in packed order; at least one region.
 *   tile_t, tile_h, tile_w: in, the tile shape; tile_t * tile_h * tile_w = 64 or 128.
 *   layout: out (host).
 *   spans: out (host, 2 * n_regions int32) or NULL: tile range [start, end) of every region.
 *   vc: out (host, n_tiles int32) or NULL: valid rows of every tile.
 *   slot_row: out (host, n_tiles * tile_elems int32) or NULL: the packed row each buffer slot
 *             holds, -1 for a pad.
 * Call once with NULL arrays to learn the sizes. Pure host computation. T3D_ERR_INVALID for an
 * empty or malformed segment, no region, a bad tile shape, or more than 2^31 rows or slots.
 */
t3d_status t3d_packed_geometry(const t3d_segment* segs, int n_segs, int tile_t, int tile_h,
                               int tile_w, t3d_packed_layout* layout, int32_t* spans, int32_t* vc,
                               int32_t* slot_row);

/* A packed buffer as the device calls see it. slot_row and vc are t3d_packed_geometry's arrays
 * copied to the device (caller-owned, read-only). */
typedef struct {
  int B;                   /* batch */
  int heads;               /* heads this call works on */
  int D;                   /* head dimension, 64 or 128 */
  int heads_total;         /* heads in one activation row; 0: equal to heads */
  int head0;               /* first head of this call; 0 when heads_total is 0 */
  int tile_elems;          /* rows per tile: 64 or 128 */
  int n_tiles;             /* tiles of the buffer */
  int rows;                /* packed rows per batch entry */
  const int32_t* slot_row; /* device, [n_tiles * tile_elems] */
  const int32_t* vc;       /* device, [n_tiles], each in 1 .. tile_elems */
} t3d_packed;

/*
 * tile3d_scatter_packed — packed order -> buffer order (video_sparse_attn_h3 page, tile()).
 *   x: in, bf16 [B, rows, heads_total, D].  y: out, bf16 [B, n_tiles * tile_elems, heads_total, D];
 *   pad slots are written as zeros. Bit-exact data movement; x and y must not overlap.
 */
t3d_status tile3d_scatter_packed(const t3d_packed* p, const void* x, void* y, t3d_stream stream);

/*
 * tile3d_gather_packed — buffer order -> packed order (the inverse of tile3d_scatter_packed).
 *   y: in, buffer order (pad slots ignored).  x: out, packed order; every packed row is written.
 */
t3d_status tile3d_gather_packed(const t3d_packed* p, const void* y, void* x, t3d_stream stream);

/*
 * tile_pool_packed — mean of every tile over its vc valid rows (sla.mean_pool as used by
 * sla.get_block_map; tiles of 64 or 128 rows).
 *   y: in, buffer order.  pooled: out, fp32 [B, heads, n_tiles, D]. fp32 accumulation.
 */
t3d_status tile_pool_packed(const t3d_packed* p, const void* y, float* pooled, t3d_stream stream);

/*
 * tile3d_scatter_pool_packed — tile3d_scatter_packed and tile_pool_packed in one pass over the
 * packed rows: y and pooled are what the two calls would write, up to the order of the fp32
 * additions. Saves re-reading y.
 *   x: in, packed order.  y: out, buffer order.  pooled: out, fp32 [B, heads, n_tiles, D].
 */
t3d_status tile3d_scatter_pool_packed(const t3d_packed* p, const void* x, void* y, float* pooled,
                                      t3d_stream stream);

#define T3D_PACKED_EXEMPT 0  /* dense tiles exempt from selection; per-region top-k */
#define T3D_PACKED_COMPETE 1 /* one top-k over all tiles (one region only) */
#define T3D_PACKED_DENSE 2   /* every tile kept (a dense layer or a dense step) */

/* At most this many video regions per call. */
#define T3D_PACKED_MAX_REGIONS 16

/*
 * tile_select_packed_capacity — the longest kept list tile_select_packed can write for these
 * arguments (the kmax to allocate). Host computation; arguments as tile_select_packed.
 */
t3d_status tile_select_packed_capacity(int n_tiles, int mode, int n_prefix, int n_regions,
                                       const int32_t* spans, const double* keep_rates, int* kmax);

/*
 * tile_select_packed — kept key tiles of every query tile of a packed buffer (the selection
 * reading above). Scores S = pooled_q . pooled_k^T are computed as in tile_select_topk
 * (tile3d.h): on the tensor cores from fp32 operands split into bf16 pairs.
 *   pq, pk: in, fp32 [B, heads, n_tiles, D] (tile_pool_packed).
 *   mode: T3D_PACKED_EXEMPT, _COMPETE or _DENSE.
 *   n_prefix, n_regions, spans: in (host), as t3d_packed_geometry wrote them (the spans must be
 *             consecutive, start at n_prefix and end at n_tiles; n_regions <= 16; compete: 1).
 *   keep_rates: in (host), n_regions rates in [0, 1] (the regions' keep rates; 1 - sparsity for
 *             the generated region). Region r keeps min(n_r, (int)(rate * n_r)) tiles, computed
 *             in double on the host.
 *   kmax: capacity of each list; at least tile_select_packed_capacity's value.
 *   kv_idx: out, int32 [B, heads, n_tiles, kmax], ascending.  kv_cnt: out, int32 [B, heads, n_tiles].
 *   workspace: at least tile_select_packed_workspace_size() bytes.
 */
t3d_status tile_select_packed(const t3d_packed* p, const float* pq, const float* pk, int mode,
                              int n_prefix, int n_regions, const int32_t* spans,
                              const double* keep_rates, int kmax, int32_t* kv_idx,
                              int32_t* kv_cnt, void* workspace, size_t ws_bytes,
                              int32_t* dev_status, t3d_stream stream);

/* Bytes of device workspace tile_select_packed needs. */
size_t tile_select_packed_workspace_size(const t3d_packed* p);

/*
 * block_sparse_attn_fwd_packed — block_sparse_attn_fwd (tile3d.h) over a packed buffer with tiles
 * of 64 or 128 rows: for every valid query row of tile i, one softmax over the valid keys of the
 * tiles kv_idx lists for i; pad query rows and tiles with kv_cnt == 0 are written as zeros.
 *   q, k, v: in, bf16 buffer order.  o: out, bf16 buffer order.
 *   kv_idx, kv_cnt, kmax: in, lists in units of the buffer's tiles (as tile_select_packed writes).
 *   softmax_scale: 1/sqrt(D) (as block_sparse_attn_fwd).
 *   workspace: at least block_sparse_attn_packed_workspace_size() bytes (the work queue's counter,
 *            the valid rows of every 64-row half, and for 128-row tiles the lists rewritten in
 *            64-row halves); calls that may overlap need workspaces of their own.
 *   dev_status: as block_sparse_attn_fwd.
 * n_tiles * tile_elems / 64 must not exceed 4096.
 */
t3d_status block_sparse_attn_fwd_packed(const t3d_packed* p, const void* q, const void* k,
                                        const void* v, void* o, const int32_t* kv_idx,
                                        const int32_t* kv_cnt, int kmax, float softmax_scale,
                                        void* workspace, size_t ws_bytes, int32_t* dev_status,
                                        t3d_stream stream);

/* Bytes of device workspace block_sparse_attn_fwd_packed needs. */
size_t block_sparse_attn_packed_workspace_size(const t3d_packed* p, int kmax);

#ifdef __cplusplus
}
#endif

#endif /* TILE3D_PACKED_H_ */
