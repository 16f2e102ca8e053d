// Coarse stage: tile-to-tile scores and KV tile selection, mask -> index lists, BSA query pruning.
//
// FastVideo API docs: fastvideo.attention.backends page, sla.get_block_map (pooled Q times pooled
// K transposed, top-k per row, block map and LUT forms); bsa_attn page, BSAAttentionImpl.forward
// (query pruning per block, KV blocks by cumulative threshold with a floor).
//
// Selection is exact on the fp32 scores: the k-th largest value of a row is found by a radix
// select (four 8-bit passes) over an order-preserving uint32 image of the floats (no sort), ties at
// the boundary go to the lower index, and kept indices are emitted in ascending order with warp
// ballots.
#include "kernels.h"

namespace t3d {
namespace {

constexpr int kSelThreads = 256;  // 8 warps
constexpr int kKeyChunk = 128;    // pooled key rows staged in shared memory at a time (one per thread pair)
constexpr int kPad = 4;           // key row padding (floats): consecutive rows 4 banks apart
constexpr int kRegSelectMax = 512;  // rows up to this many tiles are selected in registers

// Shared memory of a selection CTA with R query tiles (floats): query rows, a key chunk, the score
// rows and, when the selection uses them, the per-warp radix histograms (the mass selection always;
// top-k for rows of more than kRegSelectMax tiles).
inline size_t sel_smem_floats(int D, int nT, int R, bool hist) {
  return (size_t)R * D + (size_t)kKeyChunk * (D + kPad) + (size_t)R * nT + (hist ? 8 * 256 : 0);
}
// Query tiles per CTA of the cumulative-mass selection: 16 (two CTAs per SM for the common sizes),
// or 8 when 16 score rows would not fit next to the staged operands (~200 KB of shared memory).
inline int sel_rows(int D, int nT) {
  return sel_smem_floats(D, nT, 16, true) * 4 <= 200 * 1024 ? 16 : 8;
}
// Query tiles per CTA of the top-k selection: the count (8 .. 24) with the fewest waves over the
// machine, each wave weighted by its rows plus a fixed cost of streaming the head's pooled keys
// (worth about 8 rows).
int topk_rows(const Geo& g, int sms) {
  constexpr size_t kSmPerSm = 233472, kSmPerCta = 232448, kReserve = 1024;
  int best = 8;
  long best_cost = -1;
  for (int R = 8; R <= 24; R += 4) {
    const size_t bytes = sel_smem_floats(g.D, g.nT, R, g.nT > kRegSelectMax) * sizeof(float);
    if (bytes > kSmPerCta) continue;
    long per_sm = (long)(kSmPerSm / (bytes + kReserve));
    if (per_sm > 2048 / kSelThreads) per_sm = 2048 / kSelThreads;
    if (per_sm < 1) continue;
    const long blocks = (long)g.B * g.heads * ((g.nT + R - 1) / R);
    const long waves = (blocks + per_sm * sms - 1) / (per_sm * sms);
    const long cost = waves * (R + 8);
    if (best_cost < 0 || cost < best_cost) {
      best = R;
      best_cost = cost;
    }
  }
  return best;
}

// Scores S[i, j] = pq_i . pk_j in fp32 (fused multiply-adds over d in order) for the CTA's R query
// tiles i0 .. i0 + R - 1; row r lands in vals[r * nT + j]. Shared memory (floats): pq rows [R][D],
// a key chunk [128][D + 4], the score rows [R][nT], then the per-warp histograms of the radix
// select. Thread t owns key j0 + (t mod 128) of each chunk and the R / 2 rows of half t / 128: its
// key row is one conflict-free 16-byte load per four d, the query rows are warp-wide broadcasts.
template <int RH>
__device__ void compute_scores(const Geo& g, const float* __restrict__ pq,
                               const float* __restrict__ pk, long bh, int i0, float* sm) {
  constexpr int R = 2 * RH;
  const int D = g.D, nT = g.nT, ldk = D + kPad, d4 = D / 4;
  float* pq_s = sm;
  float* pk_s = pq_s + R * D;
  float* vals = pk_s + kKeyChunk * ldk;
  const int tid = threadIdx.x;
  for (int e = tid; e < R * d4; e += kSelThreads) {
    const int r = e / d4, c = e - r * d4;
    const int i = i0 + r;
    const float4 v = (i < nT) ? reinterpret_cast<const float4*>(pq + (bh * nT + i) * D)[c]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(pq_s + r * D + 4 * c) = v;
  }
  const float* pkh = pk + bh * nT * D;
  const int kc = tid & (kKeyChunk - 1), rh = tid / kKeyChunk;
  const float* qrow = pq_s + rh * RH * D;
  for (int j0 = 0; j0 < nT; j0 += kKeyChunk) {
    __syncthreads();
    const int rows = imin(kKeyChunk, nT - j0);
    for (int e = tid; e < kKeyChunk * d4; e += kSelThreads) {
      const int r = e / d4, c = e - r * d4;
      const float4 v = (r < rows) ? reinterpret_cast<const float4*>(pkh + (long)(j0 + r) * D)[c]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(pk_s + r * ldk + 4 * c) = v;
    }
    __syncthreads();
    float acc[RH];
#pragma unroll
    for (int a = 0; a < RH; ++a) acc[a] = 0.f;
    const float* krow = pk_s + kc * ldk;
    for (int d = 0; d < D; d += 4) {
      const float4 kb = *reinterpret_cast<const float4*>(krow + d);
#pragma unroll
      for (int a = 0; a < RH; ++a) {
        const float4 qa = *reinterpret_cast<const float4*>(qrow + a * D + d);
        acc[a] = fmaf(qa.x, kb.x, acc[a]);
        acc[a] = fmaf(qa.y, kb.y, acc[a]);
        acc[a] = fmaf(qa.z, kb.z, acc[a]);
        acc[a] = fmaf(qa.w, kb.w, acc[a]);
      }
    }
    if (kc < rows) {
#pragma unroll
      for (int a = 0; a < RH; ++a) vals[(rh * RH + a) * nT + j0 + kc] = acc[a];
    }
  }
  __syncthreads();
}

// R = 8 or 16 (the cumulative-mass selection).
__device__ void compute_scores_8_16(const Geo& g, const float* pq, const float* pk, long bh, int i0,
                                    int R, float* sm) {
  if (R == 16) compute_scores<8>(g, pq, pk, bh, i0, sm);
  else compute_scores<4>(g, pq, pk, bh, i0, sm);
}
// R = 8, 12, 16, 20 or 24 (the top-k selection).
__device__ void compute_scores_any(const Geo& g, const float* pq, const float* pk, long bh, int i0,
                                   int R, float* sm) {
  switch (R) {
    case 24: compute_scores<12>(g, pq, pk, bh, i0, sm); break;
    case 20: compute_scores<10>(g, pq, pk, bh, i0, sm); break;
    case 16: compute_scores<8>(g, pq, pk, bh, i0, sm); break;
    case 12: compute_scores<6>(g, pq, pk, bh, i0, sm); break;
    default: compute_scores<4>(g, pq, pk, bh, i0, sm); break;
  }
}

// Top-k of a row of at most 32 * KPL values held in registers (lane l owns entries l + 32 i):
// the k-th largest order-preserving key is found bit by bit from the top (largest T with at least k
// keys >= T; the search stops early once exactly k keys are >= the candidate), then every key above
// the threshold and the first (by index) ties at it are emitted in ascending index order. Same
// result as the radix select below; no shared-memory histograms.
template <int KPL>
__device__ int select_topk_row_reg(const float* row, int n, int k, int32_t* out) {
  k = imin(k, n);
  if (k <= 0) return 0;
  const int lane = threadIdx.x & 31;
  uint32_t key[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int j = lane + 32 * i;
    key[i] = j < n ? float_key(row[j]) : 0u;  // 0 ranks below every float's key
  }
  uint32_t thr = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = thr | (1u << bit);
    int c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += key[i] >= cand ? 1 : 0;
    const int total = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
    if (total >= k) thr = cand;
    // Exactly k keys at or above the threshold: they are the top k (no tie crosses it), and the
    // emission below keeps every key >= thr, so the remaining low bits change nothing.
    if (total == k) break;
  }
  int gt = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) gt += key[i] > thr ? 1 : 0;
  const int need_eq = k - (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);
  const unsigned lt = lanemask_lt();
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int j = lane + 32 * i;
    const bool eq = j < n && key[i] == thr;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool sel = (j < n && key[i] > thr) || (eq && eq_seen + __popc(eqb & lt) < need_eq);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(sb & lt);
    if (sel && pos < k) out[pos] = j;
    written += __popc(sb);
    eq_seen += __popc(eqb);
  }
  return k;
}

// Key of the k-th largest value of row[0..n) (1 <= k <= n): radix select on the order-preserving
// uint32 keys, 8 bits per pass from the top, with a 256-bin histogram per warp (`hist`, shared
// memory) filled by warp-aggregated atomics.
__device__ uint32_t kth_largest_key(const float* row, int n, int k, int* hist) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int krem = k;  // rank still to find among the keys matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int t = 0; t < 8; ++t) hist[lane * 8 + t] = 0;
    __syncwarp();
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < n ? float_key(row[j]) : 0u;
      const bool in = j < n && (key & mask) == prefix;
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const int bin = (key >> shift) & 255;
        const unsigned peers = __match_any_sync(act, bin);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], __popc(peers));
      }
    }
    __syncwarp();
    // Lane l owns bins 255 - 8 l .. 248 - 8 l (descending); find the bin holding rank krem.
    int c[8], tot = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      c[t] = hist[255 - (lane * 8 + t)];
      tot += c[t];
    }
    int incl = tot;  // inclusive prefix over lanes (bins above and including this lane's)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - tot;
    const unsigned hit = __ballot_sync(0xffffffffu, excl < krem && incl >= krem);
    const int owner = __ffs(hit) - 1;
    int digit = 0, above = 0;
    if (lane == owner) {
      int run = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (run + c[t] >= krem) {
          digit = 255 - (lane * 8 + t);
          above = run;
          break;
        }
        run += c[t];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, owner);
    above = __shfl_sync(0xffffffffu, above, owner);
    prefix |= (uint32_t)digit << shift;
    mask |= 255u << shift;
    krem -= above;
    __syncwarp();
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
__device__ int select_topk_row(const float* row, int n, int k, int32_t* out, int* hist) {
  k = imin(k, n);
  if (k <= 0) return 0;
  const uint32_t thr = kth_largest_key(row, n, k, hist);
  const int lane = threadIdx.x & 31;
  int gt = 0;
  for (int j = lane; j < n; j += 32) gt += (float_key(row[j]) > thr) ? 1 : 0;
  gt = warp_sum_int(gt);
  emit_threshold(row, n, thr, k - gt, out, k);
  return k;
}

__global__ void __launch_bounds__(kSelThreads) topk_kernel(Geo g, const float* __restrict__ pq,
                                                           const float* __restrict__ pk, int k,
                                                           int R, int32_t* __restrict__ kv_idx,
                                                           int32_t* __restrict__ kv_cnt) {
  extern __shared__ float4 sm4[];
  float* sm = reinterpret_cast<float*>(sm4);
  const int nT = g.nT;
  const int blocks_per_head = (nT + R - 1) / R;
  const long bh = blockIdx.x / blocks_per_head;
  const int i0 = (int)(blockIdx.x - bh * blocks_per_head) * R;
  compute_scores_any(g, pq, pk, bh, i0, R, sm);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* vals = sm + R * g.D + kKeyChunk * (g.D + kPad);
  int* hist = reinterpret_cast<int*>(const_cast<float*>(vals) + R * nT) + w * 256;
  const int kk = imin(k, nT);
  for (int r = w; r < R; r += kSelThreads / 32) {
    const int i = i0 + r;
    if (i >= nT) break;
    const float* row = vals + r * nT;
    int32_t* out = kv_idx + (bh * nT + i) * kk;
    int n;
    if (nT <= 128) n = select_topk_row_reg<4>(row, nT, kk, out);
    else if (nT <= 256) n = select_topk_row_reg<8>(row, nT, kk, out);
    else if (nT <= kRegSelectMax) n = select_topk_row_reg<16>(row, nT, kk, out);
    else n = select_topk_row(row, nT, kk, out, hist);
    if (lane == 0) kv_cnt[bh * nT + i] = n;
  }
}

// Cumulative-mass selection of one row (one warp). The scores in row[0..nT) are replaced by
// e_j = exp(scale * (S_j - max S)); tiles are ranked by e (ties: lower index) and the smallest
// prefix whose sum reaches mass * sum(e) is kept (at least min_k, at most kmax tiles, the most
// probable ones; T3D_DEV_OVERFLOW when truncated). Writes ascending indices to out, returns the count.
__device__ int select_mass_row(float* row, int nT, float scale, float mass, int min_k, int kmax,
                               int32_t* out, int32_t* dev_status, int* hist) {
  const int lane = threadIdx.x & 31;
  if (mass >= 1.f) {
    // Every probability of a softmax is positive, so the running sum reaches 1 only with the last
    // tile: all tiles are kept (the most probable kmax when they do not fit). Deciding this before
    // the exponentials keeps tiles whose fp32 exponential underflows to 0.
    if (nT <= kmax) {
      for (int j = lane; j < nT; j += 32) out[j] = j;
      return nT;
    }
    if (lane == 0) report(dev_status, T3D_DEV_OVERFLOW);
    return select_topk_row(row, nT, kmax, out, hist);
  }
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
  const int floor_k = imin(min_k, nT);
  if (count < floor_k || count > kmax) {
    const int kk = count < floor_k ? floor_k : kmax;
    if (count > kmax && lane == 0) report(dev_status, T3D_DEV_OVERFLOW);
    count = select_topk_row(row, nT, imin(kk, kmax), out, hist);
  } else {
    emit_threshold(row, nT, prefix, need_eq, out, kmax);
  }
  return count;
}

__global__ void __launch_bounds__(kSelThreads) mass_kernel(Geo g, const float* __restrict__ pq,
                                                           const float* __restrict__ pk,
                                                           float scale, float mass, int min_k,
                                                           int kmax, int R,
                                                           int32_t* __restrict__ kv_idx,
                                                           int32_t* __restrict__ kv_cnt,
                                                           int32_t* dev_status) {
  extern __shared__ float4 sm4[];
  float* sm = reinterpret_cast<float*>(sm4);
  const int nT = g.nT;
  const int blocks_per_head = (nT + R - 1) / R;
  const long bh = blockIdx.x / blocks_per_head;
  const int i0 = (int)(blockIdx.x - bh * blocks_per_head) * R;
  compute_scores_8_16(g, pq, pk, bh, i0, R, sm);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* vals = sm + R * g.D + kKeyChunk * (g.D + kPad);
  int* hist = reinterpret_cast<int*>(vals + R * nT) + w * 256;
  for (int r = w; r < R; r += kSelThreads / 32) {
    const int i = i0 + r;
    if (i >= nT) break;
    const int count = select_mass_row(vals + r * nT, nT, scale, mass, min_k, kmax,
                                      kv_idx + (bh * nT + i) * kmax, dev_status, hist);
    if (lane == 0) kv_cnt[bh * nT + i] = count;
  }
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

// keep_size == 0: threshold mode (rows with cosine to the block mean above cos_thresh are pruned);
// keep_size > 0: ratio mode (the keep_size rows with the lowest cosine are kept, lowest index on
// ties). Either way a pruned row copies its most cosine-similar kept row.
__global__ void __launch_bounds__(kPruneThreads) prune_kernel(Geo g, const __nv_bfloat16* __restrict__ q,
                                                              float cos_thresh, int keep_size,
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
  if (w == 0 && keep_size > 0) {
    // Ratio mode: rank of row r among (cosine, index) pairs in increasing order.
    for (int r0 = 0; r0 < kTileElems; r0 += 32) {
      const int r = r0 + lane;
      const float c = cosm[r];
      int rank = 0;
      for (int j = 0; j < kTileElems; ++j) {
        const float cj = cosm[j];
        rank += (cj < c || (cj == c && j < r)) ? 1 : 0;
      }
      keep_s[r] = rank < keep_size ? 1 : 0;
    }
    if (lane == 0) n_keep = keep_size;
  } else if (w == 0) {
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
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int R = topk_rows(g, sms > 0 ? sms : 148);
  const size_t smem = sel_smem_floats(g.D, g.nT, R, g.nT > kRegSelectMax) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long blocks = (long)g.B * g.heads * ((g.nT + R - 1) / R);
  topk_kernel<<<(unsigned)blocks, kSelThreads, smem, s>>>(g, pq, pk, k, R, kv_idx, kv_cnt);
  return cudaGetLastError();
}

cudaError_t launch_select_mass(const Geo& g, const float* pq, const float* pk, float scale,
                               float mass, int min_k, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                               int32_t* dev_status, cudaStream_t s) {
  const int R = sel_rows(g.D, g.nT);
  const size_t smem = sel_smem_floats(g.D, g.nT, R, true) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(mass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long blocks = (long)g.B * g.heads * ((g.nT + R - 1) / R);
  mass_kernel<<<(unsigned)blocks, kSelThreads, smem, s>>>(g, pq, pk, scale, mass, min_k, kmax, R,
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

cudaError_t launch_prune(const Geo& g, const void* q, float cos_thresh, int keep_size, uint8_t* keep,
                         uint8_t* src_row, float* pq_kept, cudaStream_t s) {
  const size_t smem = ((size_t)kTileElems * (g.D + 1) + g.D + 2 * kTileElems) * sizeof(float) +
                      2 * kTileElems * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(prune_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nT, g.heads, g.B);
  prune_kernel<<<grid, kPruneThreads, smem, s>>>(g, static_cast<const __nv_bfloat16*>(q),
                                                 cos_thresh, keep_size, keep, src_row, pq_kept);
  return cudaGetLastError();
}

}  // namespace t3d
