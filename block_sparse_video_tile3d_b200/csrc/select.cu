// Coarse stage: tile-to-tile scores and KV tile selection, mask -> index lists, BSA query pruning.
//
// FastVideo API docs: fastvideo.attention.backends page, sla.get_block_map (pooled Q times pooled
// K transposed, top-k per row, block map and LUT forms); bsa_attn page, BSAAttentionImpl.forward
// (query pruning per block, KV blocks by cumulative threshold with a floor).
//
// Selection is exact on the fp32 scores: the k-th largest value of a row is found by a 32-step
// bitwise search over an order-preserving uint32 image of the floats (no sort), ties at the
// boundary go to the lower index, and kept indices are emitted in ascending order with warp ballots.
#include "kernels.h"

namespace t3d {
namespace {

constexpr int kSelRows = 8;  // query tiles per CTA, one warp each
constexpr int kSelThreads = 32 * kSelRows;
constexpr int kKeyChunk = 32;  // pooled key rows staged in shared memory at a time

// Shared-memory layout of the score kernels (floats): pq rows, a key chunk padded to D+1 columns
// (conflict-free column reads), then one nT-long row of values per warp.
__host__ __device__ inline size_t sel_smem_floats(int D, int nT) {
  return (size_t)kSelRows * D + (size_t)kKeyChunk * (D + 1) + (size_t)kSelRows * nT;
}

// Scores S[i, j] = pq_i . pk_j (fp32, sequential over d) for the CTA's kSelRows rows; row w of the
// CTA lands in vals[w * nT + j].
__device__ void compute_scores(const Geo& g, const float* __restrict__ pq,
                               const float* __restrict__ pk, long bh, int i0, float* sm) {
  const int D = g.D, nT = g.nT;
  float* pq_s = sm;
  float* pk_s = pq_s + kSelRows * D;
  float* vals = pk_s + kKeyChunk * (D + 1);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  for (int e = tid; e < kSelRows * D; e += kSelThreads) {
    const int r = e / D, d = e - r * D;
    const int i = i0 + r;
    pq_s[e] = (i < nT) ? pq[(bh * nT + i) * D + d] : 0.f;
  }
  const float* pkh = pk + bh * nT * D;
  for (int j0 = 0; j0 < nT; j0 += kKeyChunk) {
    __syncthreads();
    const int rows = imin(kKeyChunk, nT - j0);
    for (int e = tid; e < kKeyChunk * D; e += kSelThreads) {
      const int r = e / D, d = e - r * D;
      pk_s[r * (D + 1) + d] = (r < rows) ? pkh[(long)(j0 + r) * D + d] : 0.f;
    }
    __syncthreads();
    if (lane < rows) {
      const float* a = pq_s + w * D;
      const float* kr = pk_s + lane * (D + 1);
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc = fmaf(a[d], kr[d], acc);
      vals[w * nT + j0 + lane] = acc;
    }
  }
  __syncthreads();
}

// Key of the k-th largest value of row[0..n) (1 <= k <= n), by bitwise search from the top bit.
__device__ uint32_t kth_largest_key(const float* row, int n, int k) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = prefix | (1u << bit);
    int c = 0;
    for (int j = lane; j < n; j += 32) c += (float_key(row[j]) >= cand) ? 1 : 0;
    if (warp_sum_int(c) >= k) prefix = cand;
  }
  return prefix;
}

// Emits, in ascending index order, every j with key > thr plus the first `need_eq` (by index) with
// key == thr. Returns the count written (all lanes).
__device__ int emit_threshold(const float* row, int n, uint32_t thr, int need_eq, int32_t* out,
                              int cap) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  int written = 0, eq_seen = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = (j < n) ? float_key(row[j]) : 0u;
    const bool gt = (j < n) && key > thr;
    const bool eq = (j < n) && key == thr;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eqb & lt);
    const bool sel = gt || (eq && eq_rank < need_eq);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(sb & lt);
    if (sel && pos < cap) out[pos] = j;
    written += __popc(sb);
    eq_seen += __popc(eqb);
  }
  return written;
}

// Top-k of row[0..n) into out (ascending indices). Returns k (clamped to n).
__device__ int select_topk_row(const float* row, int n, int k, int32_t* out) {
  k = imin(k, n);
  if (k <= 0) return 0;
  const uint32_t thr = kth_largest_key(row, n, k);
  const int lane = threadIdx.x & 31;
  int gt = 0;
  for (int j = lane; j < n; j += 32) gt += (float_key(row[j]) > thr) ? 1 : 0;
  gt = warp_sum_int(gt);
  emit_threshold(row, n, thr, k - gt, out, k);
  return k;
}

__global__ void __launch_bounds__(kSelThreads) topk_kernel(Geo g, const float* __restrict__ pq,
                                                           const float* __restrict__ pk, int k,
                                                           int32_t* __restrict__ kv_idx,
                                                           int32_t* __restrict__ kv_cnt) {
  extern __shared__ float sm[];
  const int nT = g.nT;
  const int blocks_per_head = (nT + kSelRows - 1) / kSelRows;
  const long bh = blockIdx.x / blocks_per_head;
  const int i0 = (int)(blockIdx.x - bh * blocks_per_head) * kSelRows;
  compute_scores(g, pq, pk, bh, i0, sm);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = i0 + w;
  if (i >= nT) return;
  const float* row = sm + kSelRows * g.D + kKeyChunk * (g.D + 1) + w * nT;
  const int kk = imin(k, nT);
  const int n = select_topk_row(row, nT, kk, kv_idx + (bh * nT + i) * kk);
  if (lane == 0) kv_cnt[bh * nT + i] = n;
}

// Cumulative-mass selection. Values are replaced by e_j = exp(scale * (S_j - max S)); tiles are
// ranked by e (ties: lower index) and the smallest prefix whose sum reaches mass * sum(e) is kept.
__global__ void __launch_bounds__(kSelThreads) mass_kernel(Geo g, const float* __restrict__ pq,
                                                           const float* __restrict__ pk,
                                                           float scale, float mass, int min_k,
                                                           int kmax, int32_t* __restrict__ kv_idx,
                                                           int32_t* __restrict__ kv_cnt,
                                                           int32_t* dev_status) {
  extern __shared__ float sm[];
  const int nT = g.nT;
  const int blocks_per_head = (nT + kSelRows - 1) / kSelRows;
  const long bh = blockIdx.x / blocks_per_head;
  const int i0 = (int)(blockIdx.x - bh * blocks_per_head) * kSelRows;
  compute_scores(g, pq, pk, bh, i0, sm);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = i0 + w;
  if (i >= nT) return;
  float* row = sm + kSelRows * g.D + kKeyChunk * (g.D + 1) + w * nT;
  float mx = -INFINITY;
  for (int j = lane; j < nT; j += 32) mx = fmaxf(mx, row[j]);
  mx = warp_max(mx);
  float tot = 0.f;
  for (int j = lane; j < nT; j += 32) {
    const float e = expf(scale * (row[j] - mx));
    row[j] = e;
    tot += e;
  }
  __syncwarp();
  tot = warp_sum(tot);
  const float target = mass * tot;
  // Largest key thr with sum_{key >= thr} e >= target: the key of the tile at which the running
  // sum (descending order) first reaches the target.
  uint32_t prefix = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = prefix | (1u << bit);
    float s = 0.f;
    for (int j = lane; j < nT; j += 32) s += (float_key(row[j]) >= cand) ? row[j] : 0.f;
    if (warp_sum(s) >= target) prefix = cand;
  }
  float above = 0.f;
  int n_above = 0;
  for (int j = lane; j < nT; j += 32) {
    if (float_key(row[j]) > prefix) {
      above += row[j];
      ++n_above;
    }
  }
  above = warp_sum(above);
  n_above = warp_sum_int(n_above);
  // Tiles tied at the threshold are taken in ascending index until the target is reached.
  int need_eq = 0;
  {
    float acc = above;
    bool done = false;
    for (int j0 = 0; j0 < nT && !done; j0 += 32) {
      const int j = j0 + lane;
      const bool eq = (j < nT) && float_key(row[j]) == prefix;
      unsigned eqb = __ballot_sync(0xffffffffu, eq);
      while (eqb != 0u && !done) {
        const int src = __ffs(eqb) - 1;
        const float e = __shfl_sync(0xffffffffu, (j < nT) ? row[imin(j, nT - 1)] : 0.f, src);
        if (acc < target) {
          acc += e;
          ++need_eq;
        }
        if (acc >= target) done = true;
        eqb &= eqb - 1u;
      }
    }
  }
  int count = n_above + need_eq;
  int32_t* out = kv_idx + (bh * nT + i) * kmax;
  const int floor_k = imin(min_k, nT);
  if (count < floor_k || count > kmax) {
    const int kk = count < floor_k ? floor_k : kmax;
    if (count > kmax && lane == 0) report(dev_status, T3D_DEV_OVERFLOW);
    count = select_topk_row(row, nT, imin(kk, kmax), out);
  } else {
    emit_threshold(row, nT, prefix, need_eq, out, kmax);
  }
  if (lane == 0) kv_cnt[bh * nT + i] = count;
}

// One warp per row of the block map.
__global__ void mask_to_index_kernel(Geo g, const uint8_t* __restrict__ mask, int kmax,
                                     int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
                                     int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const long rows = (long)g.B * g.heads * g.nT;
  const long nwarps = (long)gridDim.x * (blockDim.x >> 5);
  const unsigned lt = lanemask_lt();
  for (long r = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
    const uint8_t* m = mask + r * g.nT;
    int32_t* out = kv_idx + r * kmax;
    int cnt = 0;
    for (int j0 = 0; j0 < g.nT; j0 += 32) {
      const int j = j0 + lane;
      const bool on = (j < g.nT) && m[j] != 0;
      const unsigned b = __ballot_sync(0xffffffffu, on);
      const int pos = cnt + __popc(b & lt);
      if (on && pos < kmax) out[pos] = j;
      cnt += __popc(b);
    }
    if (cnt > kmax) {
      if (lane == 0) report(dev_status, T3D_DEV_OVERFLOW);
      cnt = kmax;
    }
    if (lane == 0) kv_cnt[r] = cnt;
  }
}

// BSA query pruning, one CTA (8 warps) per (batch, head, block of 64 rows).
constexpr int kPruneThreads = 256;

__global__ void __launch_bounds__(kPruneThreads) prune_kernel(Geo g, const __nv_bfloat16* __restrict__ q,
                                                              float cos_thresh,
                                                              uint8_t* __restrict__ keep,
                                                              uint8_t* __restrict__ src_row,
                                                              float* __restrict__ pq_kept) {
  extern __shared__ float sm[];
  const int D = g.D, ld = D + 1;
  float* qs = sm;                       // [64][D+1]
  float* mu = qs + kTileElems * ld;     // [D]
  float* n2 = mu + D;                   // [64] squared row norms
  float* cosm = n2 + kTileElems;        // [64] cosine to the block mean
  int* keep_s = reinterpret_cast<int*>(cosm + kTileElems);  // [64]
  int* src_s = keep_s + kTileElems;                         // [64]
  __shared__ float mu_n2;
  __shared__ int n_keep;
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const long row_stride = (long)g.heads * D;
  const __nv_bfloat16* base = q + ((long)b * g.Lp + (long)i * kTileElems) * row_stride + (long)h * D;
  for (int e = tid; e < kTileElems * D / 8; e += kPruneThreads) {
    const int r = e / (D / 8), c = e - r * (D / 8);
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(base + r * row_stride) + c);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = __bfloat1622float2(h2[t]);
      qs[r * ld + c * 8 + 2 * t] = f.x;
      qs[r * ld + c * 8 + 2 * t + 1] = f.y;
    }
  }
  __syncthreads();
  for (int d = tid; d < D; d += kPruneThreads) {
    float s = 0.f;
    for (int r = 0; r < kTileElems; ++r) s += qs[r * ld + d];
    mu[d] = s / (float)kTileElems;
  }
  __syncthreads();
  if (w == 0) {
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s += mu[d] * mu[d];
    s = warp_sum(s);
    if (lane == 0) mu_n2 = s;
  }
  __syncthreads();
  for (int r = w; r < kTileElems; r += kPruneThreads / 32) {
    float a = 0.f, dm = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float x = qs[r * ld + d];
      a += x * x;
      dm += x * mu[d];
    }
    a = warp_sum(a);
    dm = warp_sum(dm);
    if (lane == 0) {
      n2[r] = a;
      cosm[r] = (a == 0.f || mu_n2 == 0.f) ? 0.f : dm / (sqrtf(a) * sqrtf(mu_n2));
    }
  }
  __syncthreads();
  if (w == 0) {
    int nk = 0;
    for (int r0 = 0; r0 < kTileElems; r0 += 32) {
      const int r = r0 + lane;
      const bool kp = !(cosm[r] > cos_thresh);
      keep_s[r] = kp ? 1 : 0;
      nk += __popc(__ballot_sync(0xffffffffu, kp));
    }
    if (nk == 0) {
      // Keep the row with the lowest cosine (lowest index on ties).
      float best = INFINITY;
      int bi = kTileElems;
      for (int r0 = 0; r0 < kTileElems; r0 += 32) {
        const int r = r0 + lane;
        if (cosm[r] < best || (cosm[r] == best && r < bi)) { best = cosm[r]; bi = r; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob < best || (ob == best && oi < bi)) { best = ob; bi = oi; }
      }
      if (lane == 0) keep_s[bi] = 1;
      nk = 1;
    }
    if (lane == 0) n_keep = nk;
  }
  __syncthreads();
  // Each pruned row takes the most cosine-similar kept row (lowest index on ties).
  for (int r = w; r < kTileElems; r += kPruneThreads / 32) {
    if (keep_s[r]) {
      if (lane == 0) src_s[r] = r;
      continue;
    }
    float best = -INFINITY;
    int bj = kTileElems;
    for (int j = lane; j < kTileElems; j += 32) {
      if (!keep_s[j]) continue;
      float dot = 0.f;
      for (int d = 0; d < D; ++d) dot = fmaf(qs[r * ld + d], qs[j * ld + d], dot);
      const float c = (n2[r] == 0.f || n2[j] == 0.f) ? 0.f : dot / (sqrtf(n2[r]) * sqrtf(n2[j]));
      if (c > best || (c == best && j < bj)) { best = c; bj = j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ob > best || (ob == best && oj < bj)) { best = ob; bj = oj; }
    }
    if (lane == 0) src_s[r] = bj;
  }
  __syncthreads();
  const long blk = (((long)b * g.heads + h) * g.nT + i);
  for (int d = tid; d < D; d += kPruneThreads) {
    float s = 0.f;
    for (int r = 0; r < kTileElems; ++r) s += keep_s[r] ? qs[r * ld + d] : 0.f;
    pq_kept[blk * D + d] = s / (float)n_keep;
  }
  if (tid < kTileElems) {
    keep[blk * kTileElems + tid] = (uint8_t)keep_s[tid];
    src_row[blk * kTileElems + tid] = (uint8_t)src_s[tid];
  }
}

}  // namespace

cudaError_t launch_select_topk(const Geo& g, const float* pq, const float* pk, int k,
                               int32_t* kv_idx, int32_t* kv_cnt, int32_t* dev_status,
                               cudaStream_t s) {
  (void)dev_status;
  const size_t smem = sel_smem_floats(g.D, g.nT) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long blocks = (long)g.B * g.heads * ((g.nT + kSelRows - 1) / kSelRows);
  topk_kernel<<<(unsigned)blocks, kSelThreads, smem, s>>>(g, pq, pk, k, kv_idx, kv_cnt);
  return cudaGetLastError();
}

cudaError_t launch_select_mass(const Geo& g, const float* pq, const float* pk, float scale,
                               float mass, int min_k, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                               int32_t* dev_status, cudaStream_t s) {
  const size_t smem = sel_smem_floats(g.D, g.nT) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(mass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long blocks = (long)g.B * g.heads * ((g.nT + kSelRows - 1) / kSelRows);
  mass_kernel<<<(unsigned)blocks, kSelThreads, smem, s>>>(g, pq, pk, scale, mass, min_k, kmax,
                                                          kv_idx, kv_cnt, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_mask_to_index(const Geo& g, const uint8_t* mask, int kmax, int32_t* kv_idx,
                                 int32_t* kv_cnt, int32_t* dev_status, cudaStream_t s) {
  const long rows = (long)g.B * g.heads * g.nT;
  long blocks = (rows + 7) / 8;
  if (blocks > 148L * 16) blocks = 148L * 16;
  mask_to_index_kernel<<<(unsigned)blocks, 256, 0, s>>>(g, mask, kmax, kv_idx, kv_cnt, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_prune(const Geo& g, const void* q, float cos_thresh, uint8_t* keep,
                         uint8_t* src_row, float* pq_kept, cudaStream_t s) {
  const size_t smem = ((size_t)kTileElems * (g.D + 1) + g.D + 2 * kTileElems) * sizeof(float) +
                      2 * kTileElems * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(prune_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nT, g.heads, g.B);
  prune_kernel<<<grid, kPruneThreads, smem, s>>>(g, static_cast<const __nv_bfloat16*>(q),
                                                 cos_thresh, keep, src_row, pq_kept);
  return cudaGetLastError();
}

}  // namespace t3d
