// Internal launchers of libtile3d (host side). Arguments are validated by the C ABI layer in
// api.cu before any of these is called; each returns the CUDA launch error.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace t3d {

cudaError_t launch_scatter(const Geo& g, const void* x, void* y, cudaStream_t s);
cudaError_t launch_gather(const Geo& g, const void* y, void* x, cudaStream_t s);
cudaError_t launch_pool(const Geo& g, const void* y, float* pooled, cudaStream_t s);
cudaError_t launch_scatter_pool(const Geo& g, const void* x, void* y, float* pooled,
                                cudaStream_t s);

// Selection: tensor-core score product into `workspace` (select_workspace_bytes), then one warp
// per query tile.
size_t select_workspace_bytes(const Geo& g);
cudaError_t launch_select_topk(const Geo& g, const float* pq, const float* pk, int k,
                               int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                               int32_t* dev_status, cudaStream_t s);
cudaError_t launch_select_mass(const Geo& g, const float* pq, const float* pk, float scale,
                               float mass, int min_k, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                               void* workspace, int32_t* dev_status, cudaStream_t s);
cudaError_t launch_mask_to_index(const Geo& g, const uint8_t* mask, int kmax, int32_t* kv_idx,
                                 int32_t* kv_cnt, int32_t* dev_status, cudaStream_t s);
cudaError_t launch_prune(const Geo& g, const void* q, float cos_thresh, int keep_size, uint8_t* keep,
                         uint8_t* src_row, float* pq_kept, cudaStream_t s);

// Tensor map over a bf16 tensor of `rank` (2 or 3) dimensions, innermost first, strides in bytes
// of every dimension but the innermost; 128-byte swizzle, out-of-range elements read as zero.
bool encode_bf16_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box);

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  int kmax;
  const uint8_t* keep;
  const uint8_t* src_row;
  float scale;
  void* workspace;        // at least kAttnWorkspaceBytes: the unit queue's counter
  size_t ws_bytes;
  int32_t* dev_status;
  long long wait_cycles;  // limit of each pipeline wait, in clock cycles
  float* lse;             // NULL, or [B, heads, Lp]: each query row's log-sum-exp (natural log)
  const uint8_t* vc_tab;  // NULL, or the valid rows of every 64-row unit (packed sequences)
};

// Backward pass (attn_bwd.cu): gradients of block_sparse_attn_fwd for an output gradient.
struct AttnBwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;       // the forward output
  const void* dout;    // its gradient
  const float* lse;    // the forward's log-sum-exp per query row, [B, heads, Lp]
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  int kmax;
  const uint8_t* keep;
  const uint8_t* src_row;
  float scale;
  void* dq;
  void* dk;
  void* dv;
  void* workspace;     // attn_bwd_workspace_bytes
  int32_t* dev_status;
  long long wait_cycles;
};
size_t attn_bwd_workspace_bytes(const Geo& g);
cudaError_t launch_attn_bwd(const Geo& g, const AttnBwdArgs& a, cudaStream_t s);

// Device scratch of the attention kernel: one 32-bit unit counter, padded to 256 bytes.
constexpr size_t kAttnWorkspaceBytes = 256;
size_t attn_workspace_bytes(const Geo& g, int kmax);
// tcgen05/TMEM/TMA kernel (attn_sm100.cu), D = 64 or 128.
cudaError_t launch_attn(const Geo& g, const AttnArgs& a, cudaStream_t s);

// Size of the library's own attention scratch (attn_noalloc.cu) and its device address on the
// current device (looked up on the first call per device).
constexpr size_t kNoAllocScratchBytes = 256;
cudaError_t noalloc_scratch(void** ptr);

// Packed multi-region sequences (packed.cu): a padded buffer of n_tiles tiles of E = 64 or 128
// rows whose slot map (packed row of every slot, -1 for a pad) and valid counts are device arrays.
struct PackedGeo {
  int B, heads, D, heads_total, head0;
  int E, n_tiles, rows;  // rows per tile, tiles, packed rows per batch entry
  int row_chunks, row_stride, row_off;  // as in Geo
  const int32_t* slot_row;  // [n_tiles * E]
  const int32_t* vc;        // [n_tiles]
};
cudaError_t launch_scatter_packed(const PackedGeo& p, const void* x, void* y, cudaStream_t s);
cudaError_t launch_gather_packed(const PackedGeo& p, const void* y, void* x, cudaStream_t s);
cudaError_t launch_pool_packed(const PackedGeo& p, const void* y, float* pooled, cudaStream_t s);
cudaError_t launch_scatter_pool_packed(const PackedGeo& p, const void* x, void* y, float* pooled,
                                       cudaStream_t s);
size_t attn_packed_workspace_bytes(const PackedGeo& p, int kmax);
cudaError_t launch_attn_packed(const PackedGeo& p, const AttnArgs& a, cudaStream_t s);
// The 64-row-unit geometry the attention kernel runs a packed buffer with.
Geo packed_attn_geo(const PackedGeo& p);

// Per-region selection of a packed sequence (select.cu), scores as launch_select_topk. mode:
// T3D_PACKED_EXEMPT / _COMPETE / _DENSE; k[r] tiles of region r (tiles lo[r] .. hi[r] - 1) are kept
// per query tile past the n_prefix dense tiles (exempt), k_total of all tiles (compete).
constexpr int kMaxRegions = 16;
struct SpanSpec {
  int mode, n_prefix, n_regions, k_total;
  int lo[kMaxRegions], hi[kMaxRegions], k[kMaxRegions];
};
cudaError_t launch_select_spans(const Geo& g, const float* pq, const float* pk, const SpanSpec& sp,
                                int kmax, int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                                cudaStream_t s);

}  // namespace t3d
