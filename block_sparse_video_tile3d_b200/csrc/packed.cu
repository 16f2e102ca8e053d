// Packed multi-region sequences: scatter into / gather from the padded tile buffer through a slot
// map, per-tile mean pooling with tiles of 64 or 128 rows, and the attention over such a buffer.
//
// FastVideo API docs, video_sparse_attn_h3 page: build() (a packed sequence of dense segments and
// video regions; tile sizes 64 and 128) and tile() (every packed row goes to one slot of a
// zero-padded tile buffer). The slot map (packed row of every buffer slot, -1 for a pad) and the
// valid count of every tile come from t3d_packed_geometry on the host; the kernels read them from
// device memory instead of computing the slots arithmetically as the single-video kernels do.
//
// The attention kernel works in units of 64 query rows with key tiles taken in pairs of 64 rows.
// A 128-row tile is two such units (its halves), and a kept 128-row key tile is exactly one pair:
// its two halves. So the call rewrites 128-row lists into half-tile lists (key tile j -> halves
// 2j, 2j + 1; both halves of query tile i take the list of i, an empty second half none) and hands
// the kernel a table of valid counts per half; a half past a tile's valid rows is masked like any
// pad key.
#include "kernels.h"

namespace t3d {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kPoolRows = 16;

// A warp copies one row of n 16-byte chunks; each lane issues up to eight loads before it stores.
__device__ __forceinline__ void copy_row16(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                           int n, int lane) {
  for (int c0 = 0; c0 < n; c0 += 256) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c < n) u[k] = __ldg(src + c);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c < n) dst[c] = u[k];
    }
  }
}

// One warp per buffer row (pads written as zeros).
__global__ void __launch_bounds__(kCopyThreads) scatter_packed_kernel(PackedGeo p,
                                                                      const uint4* __restrict__ x,
                                                                      uint4* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const long per_b = (long)p.n_tiles * p.E;
  const long total = (long)p.B * per_b;
  const long nwarps = (long)gridDim.x * (kCopyThreads / 32);
  for (long row = (long)blockIdx.x * (kCopyThreads / 32) + (threadIdx.x >> 5); row < total;
       row += nwarps) {
    const long b = row / per_b;
    const int slot = (int)(row - b * per_b);
    const int src = p.slot_row[slot];
    uint4* dst = y + row * p.row_stride + p.row_off;
    if (src < 0) {
      for (int c = lane; c < p.row_chunks; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      copy_row16(x + (b * p.rows + src) * p.row_stride + p.row_off, dst, p.row_chunks, lane);
    }
  }
}

// One warp per buffer row that holds a token: it goes back to its packed row.
__global__ void __launch_bounds__(kCopyThreads) gather_packed_kernel(PackedGeo p,
                                                                     const uint4* __restrict__ y,
                                                                     uint4* __restrict__ x) {
  const int lane = threadIdx.x & 31;
  const long per_b = (long)p.n_tiles * p.E;
  const long total = (long)p.B * per_b;
  const long nwarps = (long)gridDim.x * (kCopyThreads / 32);
  for (long row = (long)blockIdx.x * (kCopyThreads / 32) + (threadIdx.x >> 5); row < total;
       row += nwarps) {
    const long b = row / per_b;
    const int slot = (int)(row - b * per_b);
    const int dst = p.slot_row[slot];
    if (dst < 0) continue;
    copy_row16(y + row * p.row_stride + p.row_off, x + (b * p.rows + dst) * p.row_stride + p.row_off,
               p.row_chunks, lane);
  }
}

// Grid (ceil(row_chunks / 32), n_tiles, B), block (32, kPoolRows): thread (lane, ry) sums one
// 16-byte column chunk over the tile's valid rows ry, ry + kPoolRows, ...; the partial sums are
// combined in shared memory and divided by the valid count.
__global__ void __launch_bounds__(32 * kPoolRows) pool_packed_kernel(PackedGeo p,
                                                                     const uint4* __restrict__ y,
                                                                     float* __restrict__ pooled) {
  __shared__ float part[kPoolRows][32 * 8 + 4];
  const int lane = threadIdx.x;
  const int ry = threadIdx.y;
  const int i = blockIdx.y;
  const int b = blockIdx.z;
  const int c = blockIdx.x * 32 + lane;
  const int vc = p.vc[i];
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (c < p.row_chunks) {
    const uint4* base = y + ((long)b * p.n_tiles * p.E + (long)i * p.E) * p.row_stride + p.row_off + c;
#pragma unroll 4
    for (int r = ry; r < vc; r += kPoolRows) {
      const uint4 u = __ldg(base + (long)r * p.row_stride);
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
  const int t = ry * 32 + lane;
  const int cc = t >> 3;
  const int e = t & 7;
  const int col_chunk = blockIdx.x * 32 + cc;
  if (t < 32 * 8 && col_chunk < p.row_chunks) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < kPoolRows; ++q) s += part[q][cc * 8 + e];
    const int col = col_chunk * 8 + e;
    const int h = col / p.D;
    const int d = col - h * p.D;
    pooled[(((long)b * p.heads + h) * p.n_tiles + i) * p.D + d] = vc > 0 ? s / (float)vc : 0.f;
  }
}

// Scatter fused with pooling, grid (ceil(row_chunks / 32), n_tiles, B), block (32, kPoolRows): the
// CTA moves one 512-byte column slab of one tile, thread (lane, ry) copying chunk column `lane` of
// the tile's slots ry, ry + kPoolRows, ... from their packed rows (zeros for pads) and summing the
// valid ones; the partial sums are combined in shared memory and divided by the valid count.
__global__ void __launch_bounds__(32 * kPoolRows) scatter_pool_packed_kernel(
    PackedGeo p, const uint4* __restrict__ x, uint4* __restrict__ y, float* __restrict__ pooled) {
  __shared__ float part[kPoolRows][32 * 8 + 4];
  const int lane = threadIdx.x;
  const int ry = threadIdx.y;
  const int i = blockIdx.y;
  const int b = blockIdx.z;
  const int c = blockIdx.x * 32 + lane;
  const int vc = p.vc[i];
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (c < p.row_chunks) {
    const long dst0 = ((long)b * p.n_tiles * p.E + (long)i * p.E) * p.row_stride + p.row_off + c;
    const long src_b = (long)b * p.rows;
    const int32_t* sr = p.slot_row + (long)i * p.E;
    // The tile's rows this thread moves, up to 8 (E / kPoolRows), loaded before any is used.
    constexpr int kMaxPer = 128 / kPoolRows;
    const int per = p.E / kPoolRows;
    uint4 u[kMaxPer];
#pragma unroll
    for (int t = 0; t < kMaxPer; ++t) {
      const int srow = t < per ? sr[ry + kPoolRows * t] : -1;
      u[t] = srow >= 0 ? __ldg(x + (src_b + srow) * p.row_stride + p.row_off + c)
                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < kMaxPer; ++t) {
      if (t >= per) break;
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[t]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
      y[dst0 + (long)(ry + kPoolRows * t) * p.row_stride] = u[t];
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[ry][lane * 8 + e] = acc[e];
  __syncthreads();
  const int t = ry * 32 + lane;
  const int cc = t >> 3;
  const int e = t & 7;
  const int col_chunk = blockIdx.x * 32 + cc;
  if (t < 32 * 8 && col_chunk < p.row_chunks) {  // the first 256 threads: 32 chunks x 8 elements
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < kPoolRows; ++q) sum += part[q][cc * 8 + e];
    const int col = col_chunk * 8 + e;
    const int h = col / p.D;
    const int d = col - h * p.D;
    pooled[(((long)b * p.heads + h) * p.n_tiles + i) * p.D + d] = vc > 0 ? sum / (float)vc : 0.f;
  }
}

// Valid counts of the kernel's 64-row units, and (128-row tiles) the half-tile lists.
__global__ void attn_packed_prep_kernel(PackedGeo p, const int32_t* __restrict__ kv_idx,
                                        const int32_t* __restrict__ kv_cnt, int kmax,
                                        uint8_t* __restrict__ vc8, int32_t* __restrict__ idx2,
                                        int32_t* __restrict__ cnt2, int32_t* dev_status) {
  const long tid = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long nthreads = (long)gridDim.x * blockDim.x;
  const int halves = p.E / 64;
  for (long t = tid; t < (long)p.n_tiles * halves; t += nthreads) {
    const int v = p.vc[t / halves] - 64 * (int)(t % halves);
    vc8[t] = (uint8_t)(v < 0 ? 0 : (v > 64 ? 64 : v));
  }
  if (halves == 1) return;
  const int units = 2 * p.n_tiles;
  const long rows = (long)p.B * p.heads * p.n_tiles;
  for (long e = tid; e < rows * kmax; e += nthreads) {
    const long r = e / kmax;
    const int slot = (int)(e - r * kmax);
    const long bh = r / p.n_tiles;
    const int i = (int)(r - bh * p.n_tiles);
    int c = kv_cnt[r];
    if (c < 0 || c > kmax) {
      if (slot == 0) report(dev_status, c < 0 ? T3D_DEV_INDEX_RANGE : T3D_DEV_OVERFLOW);
      c = c < 0 ? 0 : kmax;
    }
    const int second_valid = p.vc[i] > 64;
    int32_t* row0 = idx2 + (bh * units + 2 * i) * (2L * kmax);
    int32_t* row1 = row0 + 2L * kmax;
    if (slot == 0) {
      cnt2[bh * units + 2 * i] = 2 * c;
      cnt2[bh * units + 2 * i + 1] = second_valid ? 2 * c : 0;
    }
    if (slot < c) {
      const int j = kv_idx[r * kmax + slot];
      const bool ok = j >= 0 && j < p.n_tiles;
      const int ja = ok ? 2 * j : -1, jb = ok ? 2 * j + 1 : -1;
      row0[2 * slot] = ja;
      row0[2 * slot + 1] = jb;
      row1[2 * slot] = ja;
      row1[2 * slot + 1] = jb;
    }
  }
}

long copy_blocks(long rows) {
  long blocks = (rows + (kCopyThreads / 32) - 1) / (kCopyThreads / 32);
  const long cap = 148L * 16;
  return blocks < cap ? blocks : cap;
}

// Byte offsets of the packed attention's workspace: the kernel's queue counter, the unit valid
// counts, then (128-row tiles) the half-tile lists and their counts.
struct PackedWs {
  size_t vc8, idx2, cnt2, total;
};
PackedWs packed_ws(const PackedGeo& p, int kmax) {
  const size_t units = (size_t)p.n_tiles * (p.E / 64);
  PackedWs w;
  w.vc8 = kAttnWorkspaceBytes;
  w.idx2 = (w.vc8 + units + 255) & ~(size_t)255;
  const size_t rows2 = (size_t)p.B * p.heads * units;
  w.cnt2 = p.E == 128 ? (w.idx2 + rows2 * 2 * kmax * sizeof(int32_t) + 255) & ~(size_t)255 : w.idx2;
  w.total = p.E == 128 ? w.cnt2 + rows2 * sizeof(int32_t) : w.idx2;
  return w;
}

}  // namespace

cudaError_t launch_scatter_packed(const PackedGeo& p, const void* x, void* y, cudaStream_t s) {
  const long rows = (long)p.B * p.n_tiles * p.E;
  scatter_packed_kernel<<<(unsigned)copy_blocks(rows), kCopyThreads, 0, s>>>(
      p, static_cast<const uint4*>(x), static_cast<uint4*>(y));
  return cudaGetLastError();
}

cudaError_t launch_gather_packed(const PackedGeo& p, const void* y, void* x, cudaStream_t s) {
  const long rows = (long)p.B * p.n_tiles * p.E;
  gather_packed_kernel<<<(unsigned)copy_blocks(rows), kCopyThreads, 0, s>>>(
      p, static_cast<const uint4*>(y), static_cast<uint4*>(x));
  return cudaGetLastError();
}

cudaError_t launch_pool_packed(const PackedGeo& p, const void* y, float* pooled, cudaStream_t s) {
  dim3 grid((p.row_chunks + 31) / 32, p.n_tiles, p.B);
  dim3 block(32, kPoolRows);
  pool_packed_kernel<<<grid, block, 0, s>>>(p, static_cast<const uint4*>(y), pooled);
  return cudaGetLastError();
}

cudaError_t launch_scatter_pool_packed(const PackedGeo& p, const void* x, void* y, float* pooled,
                                       cudaStream_t s) {
  dim3 grid((p.row_chunks + 31) / 32, p.n_tiles, p.B);
  dim3 block(32, kPoolRows);
  scatter_pool_packed_kernel<<<grid, block, 0, s>>>(p, static_cast<const uint4*>(x),
                                                    static_cast<uint4*>(y), pooled);
  return cudaGetLastError();
}

size_t attn_packed_workspace_bytes(const PackedGeo& p, int kmax) { return packed_ws(p, kmax).total; }

Geo packed_attn_geo(const PackedGeo& p) {
  Geo g;
  const int units = p.n_tiles * (p.E / 64);
  g.B = p.B;
  g.heads = p.heads;
  g.D = p.D;
  g.heads_total = p.heads_total;
  g.head0 = p.head0;
  g.T = 1;  // the geometry fields below describe no grid: valid counts come from the table
  g.H = 1;
  g.W = units * kTileElems;
  g.nt = 1;
  g.nh = 1;
  g.nw = units;
  g.nT = units;
  g.L = units * kTileElems;
  g.Lp = units * kTileElems;
  g.row_chunks = p.row_chunks;
  g.row_stride = p.row_stride;
  g.row_off = p.row_off;
  return g;
}

cudaError_t launch_attn_packed(const PackedGeo& p, const AttnArgs& a_in, cudaStream_t s) {
  const PackedWs w = packed_ws(p, a_in.kmax);
  uint8_t* ws = static_cast<uint8_t*>(a_in.workspace);
  uint8_t* vc8 = ws + w.vc8;
  int32_t* idx2 = reinterpret_cast<int32_t*>(ws + w.idx2);
  int32_t* cnt2 = reinterpret_cast<int32_t*>(ws + w.cnt2);
  const long work = p.E == 128 ? (long)p.B * p.heads * p.n_tiles * a_in.kmax : (long)p.n_tiles;
  long blocks = (work + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 148L * 8) blocks = 148L * 8;
  attn_packed_prep_kernel<<<(unsigned)blocks, 256, 0, s>>>(p, a_in.kv_idx, a_in.kv_cnt, a_in.kmax,
                                                           vc8, idx2, cnt2, a_in.dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  AttnArgs a = a_in;
  a.vc_tab = vc8;
  if (p.E == 128) {
    a.kv_idx = idx2;
    a.kv_cnt = cnt2;
    a.kmax = 2 * a_in.kmax;
  }
  return launch_attn(packed_attn_geo(p), a, s);
}

}  // namespace t3d
