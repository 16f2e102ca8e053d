// Shared device/host helpers of libtile3d: geometry arithmetic, status words, small intrinsics.
//
// Geometry follows the FastVideo attention-backend pages: tiles of 4 x 4 x 4 tokens visited
// t-tile, h-tile, w-tile (bsa_attn page, get_tile_partition_indices), valid counts per tile as in
// video_sparse_attn.construct_variable_block_sizes, and a padded tile buffer whose pad slots are
// zero (video_sparse_attn_h3 page, tile()). Tile i owns padded rows [64 i, 64 i + 64); its valid
// tokens sit in slots 0 .. vc_i - 1 in in-tile raster order.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tile3d.h"
#include "tile3d_packed.h"

namespace t3d {

constexpr int kTile = 4;
constexpr int kTileElems = 64;
constexpr int kMaxTiles = 4096;

// Activations are [B, L or Lp, heads_total, D]; a call works on heads head0 .. head0 + heads - 1
// (per-head outputs such as pooled tiles and kept lists are [B, heads, ...] for those heads only).
struct Geo {
  int B, T, H, W, heads, D;
  int heads_total, head0;
  int nt, nh, nw;  // tiles along t, h, w
  int nT;          // nt * nh * nw
  int L, Lp;       // raster length, padded tile-order length (64 * nT)
  int row_chunks;  // 16-byte chunks of this call's heads in one token row (heads * D bf16)
  int row_stride;  // 16-byte chunks in one whole token row (heads_total * D bf16)
  int row_off;     // 16-byte chunks before this call's first head (head0 * D bf16)
};

inline Geo make_geo(const t3d_geom& g) {
  Geo r;
  r.B = g.B; r.T = g.T; r.H = g.H; r.W = g.W; r.heads = g.heads; r.D = g.D;
  r.heads_total = g.heads_total > 0 ? g.heads_total : g.heads;
  r.head0 = g.head0;
  r.nt = (g.T + kTile - 1) / kTile;
  r.nh = (g.H + kTile - 1) / kTile;
  r.nw = (g.W + kTile - 1) / kTile;
  r.nT = r.nt * r.nh * r.nw;
  r.L = g.T * g.H * g.W;
  r.Lp = kTileElems * r.nT;
  r.row_chunks = g.heads * g.D / 8;
  r.row_stride = r.heads_total * g.D / 8;
  r.row_off = r.head0 * g.D / 8;
  return r;
}

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }

// Valid token count of tile i.
__host__ __device__ inline int tile_valid_count(const Geo& g, int i) {
  const int per_t = g.nh * g.nw;
  const int a = i / per_t;
  const int r = i - a * per_t;
  const int b = r / g.nw;
  const int c = r - b * g.nw;
  return imin(kTile, g.T - kTile * a) * imin(kTile, g.H - kTile * b) * imin(kTile, g.W - kTile * c);
}

// Padded row p in [0, Lp) -> raster token id, or -1 for a pad slot.
__device__ inline int padded_to_raster(const Geo& g, int p) {
  const int i = p >> 6;
  const int s = p & 63;
  const int per_t = g.nh * g.nw;
  const int a = i / per_t;
  const int r = i - a * per_t;
  const int b = r / g.nw;
  const int c = r - b * g.nw;
  const int et = imin(kTile, g.T - kTile * a);
  const int eh = imin(kTile, g.H - kTile * b);
  const int ew = imin(kTile, g.W - kTile * c);
  const int ehw = eh * ew;
  if (s >= et * ehw) return -1;
  const int dt = s / ehw;
  const int rem = s - dt * ehw;
  const int dh = rem / ew;
  const int dw = rem - dh * ew;
  return ((kTile * a + dt) * g.H + kTile * b + dh) * g.W + kTile * c + dw;
}

// Raster token id -> padded row.
__device__ inline int raster_to_padded(const Geo& g, int tok) {
  const int w = tok % g.W;
  const int th = tok / g.W;
  const int h = th % g.H;
  const int t = th / g.H;
  const int a = t >> 2, b = h >> 2, c = w >> 2;
  const int eh = imin(kTile, g.H - kTile * b);
  const int ew = imin(kTile, g.W - kTile * c);
  const int slot = ((t & 3) * eh + (h & 3)) * ew + (w & 3);
  return ((a * g.nh + b) * g.nw + c) * kTileElems + slot;
}

__device__ inline void report(int32_t* dev_status, int bits) {
  if (dev_status != nullptr) atomicOr(dev_status, bits);
}

__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ inline int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ inline unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Order-preserving map of a float to uint32: a > b (as floats, no NaN) <=> key(a) > key(b).
__device__ inline uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace t3d
