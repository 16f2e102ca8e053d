/*
 * tile3d.h — C ABI of the B200 (sm_100a) tile-sparse 3D-tiled video attention library
 * (libtile3d.so).
 *
 * The method: a T x H x W latent token grid is reordered into contiguous 64-token cubes
 * (4 x 4 x 4 tiles, zero-padded where the grid does not divide), Q and K are mean-pooled per tile,
 * a set of key tiles is kept per query tile (top-k of pooled scores, cumulative softmax mass, or a
 * caller's block mask; the BSA variant also prunes redundant query rows), softmax attention runs
 * over the kept (query tile, key tile) pairs only, and the output is returned to raster order.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library never frees or
 *    keeps them, and allocates no device memory. The only device memory it touches beyond its
 *    arguments is the caller-sized workspace of block_sparse_attn_fwd.
 *  - Activations are bf16, layout [B, L, heads_total, D] with D fastest (raster order,
 *    L = T*H*W) or [B, Lp, heads_total, D] (tile order, Lp = 64 * nT). Tile i occupies rows
 *    [64 i, 64 i + 64); its vc_i valid tokens fill slots 0 .. vc_i - 1 in in-tile raster order,
 *    the rest are zero. A call works on heads head0 .. head0 + heads - 1 of those rows (all of
 *    them by default: heads_total = 0 means heads_total = heads, head0 = 0) and leaves the other
 *    heads' columns untouched; per-head arrays (pooled tiles, kept lists, pruning masks) cover
 *    the call's heads only: [B, heads, ...]. This is how one layer's heads are shared out over
 *    GPUs with no data exchange: each rank passes its own head range of the same full rows.
 *  - Tiles are numbered t-tile major, then h-tile, then w-tile; nT = ceil(T/4)*ceil(H/4)*ceil(W/4).
 *  - Every call is asynchronous on `stream` (0 = legacy default stream), never synchronises, and
 *    returns a t3d_status. Argument errors are detected on the host before anything is enqueued.
 *    Errors found by a kernel (an out-of-range index, a list longer than its capacity) are
 *    recorded in the caller's device status word `dev_status` (an int32 the caller zeroes; the
 *    kernel ORs T3D_DEV_* bits into it) and the offending entry is skipped or clamped.
 *  - No exception or abort crosses the ABI. t3d_last_error_string() describes the last failure
 *    on the calling host thread.
 *  - Pointers must be 16-byte aligned; heads * D must be a multiple of 8.
 *  - Supported: D in {64, 128}; 1 <= B, heads; 1 <= T, H, W; nT <= 4096.
 */
#ifndef TILE3D_H_
#define TILE3D_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* t3d_stream;  /* a cudaStream_t */

typedef enum {
  T3D_OK = 0,
  T3D_ERR_INVALID = 1,     /* bad argument: null/misaligned pointer, bad size, bad scale, k > nT */
  T3D_ERR_UNSUPPORTED = 2, /* valid request this library does not implement (causal, GQA, D) */
  T3D_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  T3D_ERR_DEVICE = 4       /* reserved: returned by t3d_check_status when dev_status != 0 */
} t3d_status;

/* Bits a kernel ORs into the caller's device status word. */
#define T3D_DEV_INDEX_RANGE 0x1 /* a key-tile index outside [0, nT) was skipped */
#define T3D_DEV_OVERFLOW 0x2    /* a selected set was longer than its capacity kmax; truncated */
#define T3D_DEV_TIMEOUT 0x4     /* a bounded wait in a pipelined kernel gave up */

/* Problem geometry. The tile is fixed at 4 x 4 x 4 = 64 tokens. */
typedef struct {
  int B;           /* batch */
  int T;           /* latent frames */
  int H;           /* latent height */
  int W;           /* latent width */
  int heads;       /* attention heads this call works on (query heads == key/value heads) */
  int D;           /* head dimension */
  int heads_total; /* heads in one activation row; 0: equal to `heads` */
  int head0;       /* first head of this call within a row; 0 when heads_total is 0 */
} t3d_geom;

/* Human-readable description of the last error on this host thread ("" if none). */
const char* t3d_last_error_string(void);

/* Library version, e.g. "0.2.0". */
const char* t3d_version(void);

/*
 * tile3d_geometry — tile counts and per-tile valid token counts.
 * FastVideo API docs, fastvideo.attention.backends page, video_sparse_attn.
 * construct_variable_block_sizes: the last tile along a dimension holds dim - (n-1)*4 tokens
 * along it; counts are flattened in (t-tile, h-tile, w-tile) order.
 *   nT, Lp: out (host). vc_host: out (host), nT int32 entries, or NULL.
 * Pure host computation.
 */
t3d_status tile3d_geometry(const t3d_geom* g, int* nT, int* Lp, int32_t* vc_host);

/*
 * tile3d_scatter — raster order -> padded tile order.
 * FastVideo API docs, bsa_attn page, get_tile_partition_indices and BSAAttentionImpl.
 * preprocess_qkv (tiles visited t/h/w-major, raster order inside a tile); video_sparse_attn_h3
 * page, tile() (rows scattered into a padded tile buffer whose pad positions stay zero).
 *   x: in,  bf16 [B, L, heads, D] raster order.
 *   y: out, bf16 [B, Lp, heads, D] tile order; pad slots are written as zeros.
 * Bit-exact data movement. x and y must not overlap.
 */
t3d_status tile3d_scatter(const t3d_geom* g, const void* x, void* y, t3d_stream stream);

/*
 * tile3d_gather — padded tile order -> raster order (the inverse of tile3d_scatter).
 * FastVideo API docs, bsa_attn page, get_reverse_tile_partition_indices and
 * BSAAttentionImpl.postprocess_output.
 *   y: in,  bf16 [B, Lp, heads, D] tile order (pad slots ignored).
 *   x: out, bf16 [B, L, heads, D] raster order.
 */
t3d_status tile3d_gather(const t3d_geom* g, const void* y, void* x, t3d_stream stream);

/*
 * tile_pool — per-tile mean over the tile's valid tokens.
 * FastVideo API docs, fastvideo.attention.backends page, sla.mean_pool (block mean along the
 * sequence, as used by sla.get_block_map). A partial tile is averaged over its vc_i valid rows.
 *   y:      in,  bf16 [B, Lp, heads, D] tile order.
 *   pooled: out, fp32 [B, heads, nT, D]. fp32 accumulation.
 */
t3d_status tile_pool(const t3d_geom* g, const void* y, float* pooled, t3d_stream stream);

/*
 * tile3d_scatter_pool — tile3d_scatter and tile_pool in one pass over the raster rows.
 * Same contracts as the two calls above (bsa_attn page, get_tile_partition_indices; sla page,
 * mean_pool); y and pooled are exactly what tile3d_scatter followed by tile_pool would write, up
 * to the order of the fp32 additions. Saves re-reading y.
 *   x: in, bf16 [B, L, heads, D] raster.  y: out, bf16 [B, Lp, heads, D].  pooled: out, fp32
 *   [B, heads, nT, D].
 */
t3d_status tile3d_scatter_pool(const t3d_geom* g, const void* x, void* y, float* pooled,
                               t3d_stream stream);

/*
 * tile_select_topk — keep the k key tiles with the largest pooled scores per query tile.
 * FastVideo API docs, fastvideo.attention.backends page, sla.get_block_map:
 * S = pooled_q @ pooled_k^T (no softmax scale), top-k per row, recorded as an index list (LUT).
 * Ties at the k-th score go to the lower key-tile index; indices are written in ascending order.
 * Scores are computed on the tensor cores from fp32 operands split into bf16 pairs
 * (hi.hi + hi.lo + lo.hi, fp32 accumulation): within about 2^-16 of sum_d |pq_d pk_d| of the exact
 * dot product, so kept sets are exact wherever the k-th and (k+1)-th scores are further apart.
 *   pq, pk: in,  fp32 [B, heads, nT, D].
 *   k:      1 <= k; k > nT is clamped to nT (every tile kept).
 *   kv_idx: out, int32 [B, heads, nT, min(k, nT)].  kv_cnt: out, int32 [B, heads, nT].
 *   workspace: device scratch of at least tile_select_workspace_size() bytes (the fp32 score
 *           rows, B * heads * nT * ceil4(nT) floats); contents on entry do not matter.
 *   dev_status: in/out device int32, or NULL.
 */
t3d_status tile_select_topk(const t3d_geom* g, const float* pq, const float* pk, int k,
                            int32_t* kv_idx, int32_t* kv_cnt, void* workspace, size_t ws_bytes,
                            int32_t* dev_status, t3d_stream stream);

/*
 * tile_select_mass — keep key tiles by cumulative softmax mass per query tile.
 * FastVideo API docs, bsa_attn page, BSAAttentionImpl.forward (KV blocks chosen with
 * kv_cumulative_threshold and a floor min_kv_blocks). Reading: p = softmax(scale * S_i) over the
 * row; tiles are taken in descending p (ties: lower index) up to and including the one at which
 * the running sum first reaches `mass`; at least min_k tiles are kept; all tiles when the sum
 * never reaches `mass`. Indices ascending.
 *   pq, pk: in, fp32 [B, heads, nT, D].  scale > 0.  0 < mass <= 1.  min_k >= 1.
 *   kmax:   capacity of each row of kv_idx (1 <= kmax <= nT); longer sets are truncated to their
 *           kmax highest-probability tiles and T3D_DEV_OVERFLOW is set.
 *   kv_idx: out, int32 [B, heads, nT, kmax].  kv_cnt: out, int32 [B, heads, nT].
 *   workspace: as tile_select_topk. Scores as tile_select_topk. mass = 1 keeps every tile.
 */
t3d_status tile_select_mass(const t3d_geom* g, const float* pq, const float* pk, float scale,
                            float mass, int min_k, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                            void* workspace, size_t ws_bytes, int32_t* dev_status,
                            t3d_stream stream);

/* Bytes of device workspace tile_select_topk / tile_select_mass need for this geometry. */
size_t tile_select_workspace_size(const t3d_geom* g);

/*
 * tile_prune_queries — BSA query pruning per 64-token block.
 * FastVideo API docs, bsa_attn page, BSAAttentionImpl.forward (query sparsification per block,
 * pruned positions reconstructed after attention). Reading: row r of block i is pruned iff
 * cos(q_r, mean of the block's rows) > cos_thresh (a zero-norm operand gives cosine 0); if every
 * row would be pruned the row with the lowest cosine is kept (lowest index on ties); a pruned row
 * copies the output of the kept row it is most cosine-similar to (lowest index on ties).
 * Requires L == Lp (every tile full), as the page asserts num_blocks * block_size == L.
 *   q:       in,  bf16 [B, Lp, heads, D] tile order.
 *   keep:    out, uint8 [B, heads, nT, 64] (1 = row attends).
 *   src_row: out, uint8 [B, heads, nT, 64] (slot whose output the row takes; itself if kept).
 *   pq_kept: out, fp32 [B, heads, nT, D]: mean of the kept rows (input to tile_select_mass).
 */
t3d_status tile_prune_queries(const t3d_geom* g, const void* q, float cos_thresh, uint8_t* keep,
                              uint8_t* src_row, float* pq_kept, t3d_stream stream);

/*
 * tile_prune_queries_ratio — BSA query pruning with a fixed count of kept rows per block.
 * FastVideo API docs, bsa_attn page, BSAAttentionImpl.forward: the pruning helper takes the
 * metadata's query_keep_ratio and returns a keep_size. Reading: keep_size = max(1, floor(64 *
 * keep_ratio)) (computed in double on the host) rows per block are kept — the rows least similar to
 * the block mean (lowest cosine, lowest index on ties); a pruned row copies the output of the kept
 * row it is most cosine-similar to (lowest index on ties), as in tile_prune_queries.
 * Requires L == Lp (every tile full).
 *   keep_ratio: in (0, 1], else T3D_ERR_INVALID.
 *   q, keep, src_row, pq_kept: as in tile_prune_queries.
 */
t3d_status tile_prune_queries_ratio(const t3d_geom* g, const void* q, float keep_ratio,
                                    uint8_t* keep, uint8_t* src_row, float* pq_kept,
                                    t3d_stream stream);

/*
 * block_mask_to_index — 0/1 block map -> ascending index lists.
 * FastVideo API docs, fastvideo.attention.backends page, sla.get_block_map (the same selection
 * as a block map and as a LUT); video_sparse_attn_h3 page (mask route of the sm100a kernel).
 *   mask:   in,  uint8 [B, heads, nT, nT] (nonzero = keep).
 *   kmax:   capacity per row (1 <= kmax <= nT); longer rows are truncated (lowest indices kept)
 *           and T3D_DEV_OVERFLOW is set.
 *   kv_idx: out, int32 [B, heads, nT, kmax].  kv_cnt: out, int32 [B, heads, nT].
 */
t3d_status block_mask_to_index(const t3d_geom* g, const uint8_t* mask, int kmax, int32_t* kv_idx,
                               int32_t* kv_cnt, int32_t* dev_status, t3d_stream stream);

/*
 * block_sparse_attn_fwd — softmax attention over the kept (query tile, key tile) pairs.
 * FastVideo API docs, bsa_attn page, BSAAttentionImpl.__init__ (no GQA, no causal mask, softmax
 * scale must be 1/sqrt(D) within rel 1e-4 / abs 1e-5) and BSAAttentionImpl.forward (sparse
 * attention on tile-ordered [B, L, heads, D] tensors, then pruned rows reconstructed).
 * For every valid query row r of tile i: o_r = sum over the valid keys c of the kept tiles of
 * softmax_c(scale * q_r . k_c) v_c — one softmax over the union of kept tiles. Pad keys get zero
 * weight; pad query rows, and every row of a tile with kv_cnt == 0, are written as zeros.
 *   q, k, v: in,  bf16 [B, Lp, heads, D] tile order.  o: out, bf16 [B, Lp, heads, D].
 *   kv_idx:  in,  int32 [B, heads, nT, kmax], the first kv_cnt entries of each row used (any
 *            order; each index in [0, nT), duplicates not allowed). kv_cnt: in, int32 [B,heads,nT].
 *   keep, src_row: NULL, or the BSA outputs of tile_prune_queries (then L must equal Lp): only
 *            kept rows attend and pruned rows take the output of src_row (which must name a kept
 *            row of the same tile; an entry >= 64 makes the row take its own result).
 *   softmax_scale: must be 1/sqrt(D) (see above), else T3D_ERR_INVALID.
 *   causal != 0 or num_kv_heads != heads: T3D_ERR_UNSUPPORTED.
 *   workspace: device scratch of at least block_sparse_attn_workspace_size() bytes (256: the
 *            counter of the kernel's work queue, which the call zeroes on `stream` before its
 *            launch). Its contents on entry do not matter; calls that may run at the same time
 *            need workspaces of their own.
 *   dev_status: in/out device int32, or NULL. Out-of-range indices are skipped and a negative
 *            kv_cnt is read as 0 (T3D_DEV_INDEX_RANGE); a kv_cnt above kmax is read as kmax
 *            (T3D_DEV_OVERFLOW); a pipeline wait that gave up sets T3D_DEV_TIMEOUT.
 * The work units (batch, head, query tile) are handed out dynamically to one CTA per SM, so query
 * tiles that keep different numbers of key tiles are balanced across the GPU.
 * fp32 accumulation and softmax; bf16 output rounded to nearest even.
 */
t3d_status block_sparse_attn_fwd(const t3d_geom* g, const void* q, const void* k, const void* v,
                                 void* o, const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                 const uint8_t* keep, const uint8_t* src_row, float softmax_scale,
                                 int causal, int num_kv_heads, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, t3d_stream stream);

/* Bytes of device workspace block_sparse_attn_fwd needs for this geometry and list capacity. */
size_t block_sparse_attn_workspace_size(const t3d_geom* g, int kmax);

/*
 * block_sparse_attn_fwd_lse — block_sparse_attn_fwd that also returns each query row's
 * log-sum-exp, the statistic the backward pass needs (training path).
 * FastVideo API docs, video_sparse_attn_h3 page: tile() gives a gradient-tracking forward its own
 * buffer; bsa_attn page, BSAAttentionImpl.forward for the forward itself.
 *   lse: out, fp32 [B, heads, Lp]: lse_r = log sum_c exp(softmax_scale * q_r . k_c) over the valid
 *        keys of the row's kept tiles (natural log; -inf for a tile with no kept key tile). Pad
 *        and pruned rows get the value of their own (unused) softmax.
 *   Every other argument, result and error: as block_sparse_attn_fwd.
 */
t3d_status block_sparse_attn_fwd_lse(const t3d_geom* g, const void* q, const void* k,
                                     const void* v, void* o, float* lse, const int32_t* kv_idx,
                                     const int32_t* kv_cnt, int kmax, const uint8_t* keep,
                                     const uint8_t* src_row, float softmax_scale, int causal,
                                     int num_kv_heads, void* workspace, size_t ws_bytes,
                                     int32_t* dev_status, t3d_stream stream);

/*
 * block_sparse_attn_bwd — gradients of block_sparse_attn_fwd with respect to q, k and v.
 * The pages train through the sparse attention (video_sparse_attn_h3 page, tile(): the
 * gradient-tracking forward) but print no backward formulas; this is the derivative of the
 * forward's definition. For an attending query row r with kept keys c:
 *   p_rc = exp(scale q_r.k_c - lse_r), delta_r = dO_r . o_r, dS_rc = p_rc (dO_r.v_c - delta_r),
 *   dq_r = scale sum_c dS_rc k_c, dk_c = scale sum_r dS_rc q_r, dv_c = sum_r p_rc dO_r.
 * No gradient flows through the selection. With keep/src_row (BSA), a pruned row's dO is added to
 * its source row's and the pruned row's dq is zero. Pad rows and pad keys get zero gradients; a
 * key tile no query tile kept gets zero dk and dv.
 *   q, k, v: in, bf16 [B, Lp, heads, D] tile order (the forward's inputs).
 *   o:       in, the forward's output.  dout: in, bf16 [B, Lp, heads, D]: the output gradient.
 *   lse:     in, fp32 [B, heads, Lp] from block_sparse_attn_fwd_lse.
 *   kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale, causal, num_kv_heads: as the forward.
 *   dq, dk, dv: out, bf16 [B, Lp, heads, D] (the call's heads only).
 *   workspace: device scratch of at least block_sparse_attn_bwd_workspace_size() bytes (the
 *            effective output gradient, delta, and the per-key-tile lists of query tiles).
 * fp32 accumulation in tensor memory; P, dS and the effective dO are rounded to bf16 as MMA
 * operands; results rounded to bf16 (nearest even). Deterministic: every sum runs in a fixed order.
 */
t3d_status block_sparse_attn_bwd(const t3d_geom* g, const void* q, const void* k, const void* v,
                                 const void* o, const void* dout, const float* lse,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                 const uint8_t* keep, const uint8_t* src_row, float softmax_scale,
                                 int causal, int num_kv_heads, void* dq, void* dk, void* dv,
                                 void* workspace, size_t ws_bytes, int32_t* dev_status,
                                 t3d_stream stream);

/* Bytes of device workspace block_sparse_attn_bwd needs for this geometry. */
size_t block_sparse_attn_bwd_workspace_size(const t3d_geom* g, int kmax);

/*
 * block_sparse_attn_fwd_noalloc — block_sparse_attn_fwd for callers that cannot allocate device
 * memory. The paper has no counterpart: this is a library service, not a step of the method.
 * Some callers own no allocator of their own: a plugin inside a host framework whose allocator
 * manages all device memory, a runtime that fixes its memory budget at start-up and forbids later
 * allocations, or a latency-bound loop that cannot afford cudaMalloc's implicit synchronisation.
 * Such a caller cannot provide the workspace, so this call takes none: the kernel's scratch (the
 * counter of its work queue) lives in a fixed 256-byte array inside the library, which every GPU
 * that loads the library holds until the process exits. The call allocates and frees nothing.
 *   Arguments, results and errors: as block_sparse_attn_fwd without `workspace` / `ws_bytes`. A
 *   problem whose scratch would exceed the fixed 256 bytes is rejected with T3D_ERR_UNSUPPORTED
 *   (the kernel's scratch does not depend on the problem size today, so none is).
 *   The first call on a device looks up the array's device address on that device (with it
 *   current) and caches it; make that first call before any stream capture.
 *   Every call on a device shares the one array (the call zeroes the counter on `stream` before
 *   its launch): calls that may overlap on the GPU race and give undefined results, so calls on
 *   one device must be ordered (one stream, or events between streams).
 */
t3d_status block_sparse_attn_fwd_noalloc(const t3d_geom* g, const void* q, const void* k,
                                         const void* v, void* o, const int32_t* kv_idx,
                                         const int32_t* kv_cnt, int kmax, const uint8_t* keep,
                                         const uint8_t* src_row, float softmax_scale, int causal,
                                         int num_kv_heads, int32_t* dev_status,
                                         t3d_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TILE3D_H_ */
