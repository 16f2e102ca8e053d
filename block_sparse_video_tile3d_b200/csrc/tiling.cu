// Tile scatter, untile (gather), per-tile mean pooling, and scatter fused with pooling.
//
// FastVideo API docs: bsa_attn page (get_tile_partition_indices, preprocess_qkv,
// postprocess_output), video_sparse_attn_h3 page (tile(): padded tile buffer, zero pads) and the
// fastvideo.attention.backends page (sla.mean_pool).
//
// All of them are HBM-bound streams over the [*, heads * D] bf16 slice of token rows that a call
// covers (heads head0 .. head0 + heads - 1 of rows of heads_total heads). A slice is heads * D * 2
// bytes (3 KB for 12 heads x 128), so one warp moves one row with 16-byte vector accesses; the
// source/destination row is computed arithmetically from the geometry (no index tensor is read).
#include "kernels.h"

namespace t3d {
namespace {

constexpr int kCopyThreads = 256;

__device__ __forceinline__ uint4 ld_nc(const uint4* p) { return __ldg(p); }

// A warp copies one row of n 16-byte chunks; each lane issues up to eight loads before it stores.
__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                         int n, int lane) {
  for (int c0 = 0; c0 < n; c0 += 256) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c < n) u[k] = ld_nc(src + c);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c < n) dst[c] = u[k];
    }
  }
}

__device__ __forceinline__ void zero_row(uint4* __restrict__ dst, int n, int lane) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int c = lane; c < n; c += 32) dst[c] = z;
}

// One warp per padded destination row (pads included, written as zeros).
__global__ void __launch_bounds__(kCopyThreads) scatter_kernel(Geo g, const uint4* __restrict__ x,
                                                               uint4* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (kCopyThreads / 32);
  const long total = (long)g.B * g.Lp;
  const int cpr = g.row_chunks;
  for (long row = (long)blockIdx.x * (kCopyThreads / 32) + (threadIdx.x >> 5); row < total;
       row += nwarps) {
    const int b = (int)(row / g.Lp);
    const int p = (int)(row - (long)b * g.Lp);
    const int src = padded_to_raster(g, p);
    uint4* dst = y + row * g.row_stride + g.row_off;
    if (src < 0) {
      zero_row(dst, cpr, lane);
    } else {
      copy_row(x + ((long)b * g.L + src) * g.row_stride + g.row_off, dst, cpr, lane);
    }
  }
}

// One warp per raster destination row; pad rows of the source are never read.
__global__ void __launch_bounds__(kCopyThreads) gather_kernel(Geo g, const uint4* __restrict__ y,
                                                              uint4* __restrict__ x) {
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (kCopyThreads / 32);
  const long total = (long)g.B * g.L;
  const int cpr = g.row_chunks;
  for (long row = (long)blockIdx.x * (kCopyThreads / 32) + (threadIdx.x >> 5); row < total;
       row += nwarps) {
    const int b = (int)(row / g.L);
    const int tok = (int)(row - (long)b * g.L);
    const int p = raster_to_padded(g, tok);
    copy_row(y + ((long)b * g.Lp + p) * g.row_stride + g.row_off,
             x + row * g.row_stride + g.row_off, cpr, lane);
  }
}

// Grid (ceil(row_chunks / 32), nT, B); block (32, kPoolRows). Thread (lane, ry) sums one 16-byte
// column chunk over the tile's valid rows ry, ry + kPoolRows, ...; the kPoolRows partial sums are
// combined in shared memory and divided by the valid count.
constexpr int kPoolRows = 16;  // warps per CTA: 512 threads, four CTAs per SM

__global__ void __launch_bounds__(32 * kPoolRows) pool_kernel(Geo g, const uint4* __restrict__ y,
                                                              float* __restrict__ pooled) {
  __shared__ float part[kPoolRows][32 * 8 + 4];
  const int lane = threadIdx.x;
  const int ry = threadIdx.y;
  const int i = blockIdx.y;
  const int b = blockIdx.z;
  const int c = blockIdx.x * 32 + lane;
  const int vc = tile_valid_count(g, i);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (c < g.row_chunks) {
    const uint4* base = y + ((long)b * g.Lp + (long)i * kTileElems) * g.row_stride + g.row_off + c;
#pragma unroll 4
    for (int r = ry; r < vc; r += kPoolRows) {
      const uint4 u = ld_nc(base + (long)r * g.row_stride);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[ry][lane * 8 + e] = acc[e];
  __syncthreads();
  // The first 256 threads finalise 32 chunks x 8 elements.
  const int t = ry * 32 + lane;
  const int cc = t >> 3;
  const int e = t & 7;
  const int col_chunk = blockIdx.x * 32 + cc;
  if (t < 32 * 8 && col_chunk < g.row_chunks) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < kPoolRows; ++q) s += part[q][cc * 8 + e];
    const int col = col_chunk * 8 + e;
    const int h = col / g.D;
    const int d = col - h * g.D;
    pooled[(((long)b * g.heads + h) * g.nT + i) * g.D + d] = s / (float)vc;
  }
}

// Fused scatter + pool: grid (ceil(row_chunks / 32), ceil(nT / kSpTiles), B), block (32,
// kPoolRows). The CTA moves one 512-byte column slab of kSpTiles consecutive tiles: thread (lane,
// ry) copies chunk column `lane` of each tile's padded rows ry, ry + kPoolRows, ... from their
// raster rows (zeros for pad slots) and sums the valid ones; the partial sums are combined in
// shared memory and divided by the valid count. All of a thread's loads (kSpTiles * 4 rows) are
// issued before any is used.
constexpr int kSpTiles = 2;

__global__ void __launch_bounds__(32 * kPoolRows) scatter_pool_kernel(Geo g,
                                                                      const uint4* __restrict__ x,
                                                                      uint4* __restrict__ y,
                                                                      float* __restrict__ pooled) {
  __shared__ float part[kSpTiles][kPoolRows][32 * 8 + 4];
  __shared__ int src_row[kSpTiles][kTileElems];
  const int lane = threadIdx.x;
  const int ry = threadIdx.y;
  const int i0 = blockIdx.y * kSpTiles;
  const int b = blockIdx.z;
  const int c = blockIdx.x * 32 + lane;
  const int t = ry * 32 + lane;
  for (int e = t; e < kSpTiles * kTileElems; e += 32 * kPoolRows) {
    const int tt = e / kTileElems, slot = e - tt * kTileElems;
    src_row[tt][slot] = i0 + tt < g.nT ? padded_to_raster(g, (i0 + tt) * kTileElems + slot) : -1;
  }
  __syncthreads();
  constexpr int kPer = kTileElems / kPoolRows;
  float acc[kSpTiles][8];
#pragma unroll
  for (int tt = 0; tt < kSpTiles; ++tt)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
  if (c < g.row_chunks) {
    const long src_b = (long)b * g.L;
    uint4 u[kSpTiles][kPer];
#pragma unroll
    for (int tt = 0; tt < kSpTiles; ++tt) {
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int sr = src_row[tt][ry + kPoolRows * k];
        u[tt][k] = sr >= 0 ? ld_nc(x + (src_b + sr) * g.row_stride + g.row_off + c)
                           : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int tt = 0; tt < kSpTiles; ++tt) {
      if (i0 + tt >= g.nT) break;
      const long dst0 = ((long)b * g.Lp + (long)(i0 + tt) * kTileElems) * g.row_stride + g.row_off + c;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[tt][k]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          acc[tt][2 * e] += f.x;
          acc[tt][2 * e + 1] += f.y;
        }
        y[dst0 + (long)(ry + kPoolRows * k) * g.row_stride] = u[tt][k];
      }
    }
  }
#pragma unroll
  for (int tt = 0; tt < kSpTiles; ++tt)
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tt][ry][lane * 8 + e] = acc[tt][e];
  __syncthreads();
  // The first 256 threads finalise tile 0's 32 chunks x 8 elements, the next 256 tile 1's.
  const int tt = t >> 8;
  const int cc = (t & 255) >> 3;
  const int e = t & 7;
  const int col_chunk = blockIdx.x * 32 + cc;
  if (tt < kSpTiles && i0 + tt < g.nT && col_chunk < g.row_chunks) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < kPoolRows; ++q) sum += part[tt][q][cc * 8 + e];
    const int col = col_chunk * 8 + e;
    const int h = col / g.D;
    const int d = col - h * g.D;
    pooled[(((long)b * g.heads + h) * g.nT + i0 + tt) * g.D + d] =
        sum / (float)tile_valid_count(g, i0 + tt);
  }
}

int copy_grid(long rows) {
  long blocks = (rows + (kCopyThreads / 32) - 1) / (kCopyThreads / 32);
  const long cap = 148L * 16;
  return (int)(blocks < cap ? blocks : cap);
}

}  // namespace

cudaError_t launch_scatter(const Geo& g, const void* x, void* y, cudaStream_t s) {
  const long rows = (long)g.B * g.Lp;
  scatter_kernel<<<copy_grid(rows), kCopyThreads, 0, s>>>(g, static_cast<const uint4*>(x),
                                                          static_cast<uint4*>(y));
  return cudaGetLastError();
}

cudaError_t launch_gather(const Geo& g, const void* y, void* x, cudaStream_t s) {
  const long rows = (long)g.B * g.L;
  gather_kernel<<<copy_grid(rows), kCopyThreads, 0, s>>>(g, static_cast<const uint4*>(y),
                                                         static_cast<uint4*>(x));
  return cudaGetLastError();
}

cudaError_t launch_scatter_pool(const Geo& g, const void* x, void* y, float* pooled,
                                cudaStream_t s) {
  dim3 grid((g.row_chunks + 31) / 32, (g.nT + kSpTiles - 1) / kSpTiles, g.B);
  dim3 block(32, kPoolRows);
  scatter_pool_kernel<<<grid, block, 0, s>>>(g, static_cast<const uint4*>(x), static_cast<uint4*>(y),
                                             pooled);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Geo& g, const void* y, float* pooled, cudaStream_t s) {
  dim3 grid((g.row_chunks + 31) / 32, g.nT, g.B);
  dim3 block(32, kPoolRows);
  pool_kernel<<<grid, block, 0, s>>>(g, static_cast<const uint4*>(y), pooled);
  return cudaGetLastError();
}

}  // namespace t3d
