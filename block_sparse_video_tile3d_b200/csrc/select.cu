// Coarse stage: tile-to-tile scores and KV tile selection, mask -> index lists, BSA query pruning.
//
// FastVideo API docs: fastvideo.attention.backends page, sla.get_block_map (pooled Q times pooled
// K transposed, top-k per row, block map and LUT forms); bsa_attn page, BSAAttentionImpl.forward
// (query pruning per block, KV blocks by cumulative threshold with a floor).
//
// Selection runs in two kernels. The score product S = pq . pk^T of every head runs on the tcgen05
// tensor cores (scores_tc_kernel) and lands in fp32 in the caller's workspace; then one warp per
// query tile selects its key tiles from its score row (topk_rows_kernel, mass_rows_kernel), so the
// selection, which costs far more instructions than the product, spreads over every SM.
//
// Selection is exact on the fp32 scores: the k-th largest value of a row is found by a bit-by-bit
// search over an order-preserving uint32 image of the floats held in registers (a radix select over
// shared-memory histograms for rows too long for registers), with no sort; ties at the boundary go
// to the lower index, and kept indices are emitted in ascending order with warp ballots.
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace t3d {
namespace {

constexpr int kSelThreads = 256;     // 8 warps: one score row each at a time
constexpr int kRegSelectMax = 1536;  // rows up to this many tiles are selected in registers

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

// Top-k of row[0..n) with the register search when the row fits (n <= kRegSelectMax), else the
// radix select over the per-warp histogram `hist` (256 ints).
__device__ int select_topk_any(const float* row, int n, int k, int32_t* out, int* hist) {
  if (n <= 128) return select_topk_row_reg<4>(row, n, k, out);
  if (n <= 256) return select_topk_row_reg<8>(row, n, k, out);
  if (n <= 512) return select_topk_row_reg<16>(row, n, k, out);
  if (n <= 1024) return select_topk_row_reg<32>(row, n, k, out);
  if (n <= kRegSelectMax) return select_topk_row_reg<48>(row, n, k, out);
  return select_topk_row(row, n, k, out, hist);
}


// Exact end of the value search once the bracket [lo, hi) holds c <= 32 of the row's values: the
// candidates (value v, tile ix) sit one per lane (lanes >= c hold v = -2, below every e). They are
// sorted by value descending, then tile ascending (a bitonic sort across the lanes), and summed in
// that order on top of fhi = F(hi), the mass of the tiles above the bracket, until the target is
// reached. Returns the crossing value; need_eq is how many tiles of that value are taken (the
// lowest-indexed ones, the tie rule of the emission).
__device__ float finish_bracket(float v, int ix, int c, float fhi, float target, int& need_eq) {
  const int lane = threadIdx.x & 31;
  for (int k = 2; k <= 32; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, j);
      const int oi = __shfl_xor_sync(0xffffffffu, ix, j);
      const bool first = v > ov || (v == ov && ix < oi);  // this lane's entry comes first
      const bool lower = (lane & j) == 0, desc = (lane & k) == 0;
      if ((lower == desc) != first) {
        v = ov;
        ix = oi;
      }
    }
  }
  float x = v >= 0.f ? v : 0.f;  // inclusive prefix sum in sorted order
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, lane < c && fhi + x >= target);
  const int js = hit != 0u ? __ffs(hit) - 1 : c - 1;  // rounding: take every candidate
  const float vs = __shfl_sync(0xffffffffu, v, js);
  need_eq = __popc(__ballot_sync(0xffffffffu, lane <= js && v == vs));
  return vs;
}

// Cumulative-mass selection of one row (one warp). The scores in row[0..nT) are replaced by
// e_j = exp(scale * (S_j - max S)); tiles are ranked by e (ties: lower index) and the smallest
// prefix whose sum reaches mass * sum(e) is kept. Writes ascending indices to out and returns the
// count; when the count falls outside [min_k, kmax] (T3D_DEV_OVERFLOW above kmax) it writes
// nothing and returns -1 - k, k the number of highest-scoring tiles to keep instead, which
// mass_fix_kernel then selects from the score row (that rare path stays out of this kernel, whose
// register count, and so its occupancy, it would otherwise set).
__device__ int select_mass_row(float* row, int nT, float scale, float mass, int min_k, int kmax,
                               int32_t* out, int32_t* dev_status, float* cv, int* ci) {
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
    return -1 - kmax;
  }
  float mx = -INFINITY;
  for (int j = lane; j < nT; j += 32) mx = fmaxf(mx, row[j]);
  mx = warp_max(mx);
  float tot = 0.f, mn = INFINITY;
  for (int j = lane; j < nT; j += 32) {
    const float e = expf(scale * (row[j] - mx));
    row[j] = e;
    tot += e;
    mn = fminf(mn, e);
  }
  __syncwarp();
  tot = warp_sum(tot);
  mn = -warp_max(-mn);
  const float target = mass * tot;
  // Largest key thr with sum_{key >= thr} e >= target: the key of the tile at which the running
  // sum (descending order) first reaches the target. First a search on the values: a bracket
  // [lo, hi) with F(lo) >= target > F(hi), F(t) = sum of the e >= t, starting from the row's
  // smallest value and just above its largest (1), narrowed by interpolating F linearly (Illinois
  // rule against a stalling end) until at most 32 values lie in it; those are then ranked and
  // summed exactly (finish_bracket). Rows where that does not happen within the step budget (ties
  // at the crossing value) take the bit-by-bit key search.
  uint32_t prefix = 0;
  bool found = false;
  int need_fin = -1;  // need_eq from finish_bracket, when it ran
  {
    float lo = mn, hi = __int_as_float(0x3f800001);  // every e lies in [mn, 1]
    float Flo = tot, Fhi = 0.f;
    int clo = nT, chi = 0;
    float wlo = 1.f, whi = 1.f;
    int side = 0;
    for (int step = 0; step < 24; ++step) {
      if (clo - chi <= 32) {
        const unsigned lt = lanemask_lt();
        int base = 0;
        for (int j0 = 0; j0 < nT; j0 += 32) {
          const int j = j0 + lane;
          const bool inb = j < nT && row[j] >= lo && row[j] < hi;
          const unsigned bb = __ballot_sync(0xffffffffu, inb);
          if (inb) {
            cv[base + __popc(bb & lt)] = row[j];
            ci[base + __popc(bb & lt)] = j;
          }
          base += __popc(bb);
        }
        __syncwarp();
        const int c = clo - chi;
        const float v = lane < c ? cv[lane] : -2.f;
        const int ix = lane < c ? ci[lane] : 0x7fffffff;
        __syncwarp();
        prefix = float_key(finish_bracket(v, ix, c, Fhi, target, need_fin));
        found = true;
        break;
      }
      const float a = wlo * (Flo - target), bb = whi * (target - Fhi);
      float t = fmaf(hi - lo, __fdividef(a, a + bb), lo);
      if (!(t > lo && t < hi)) t = 0.5f * (lo + hi);
      if (!(t > lo && t < hi)) break;
      float ft = 0.f;
      int ct = 0;
      for (int j = lane; j < nT; j += 32) {
        if (row[j] >= t) {
          ft += row[j];
          ++ct;
        }
      }
      ft = warp_sum(ft);
      ct = warp_sum_int(ct);
      if (ft >= target) {
        lo = t;
        Flo = ft;
        clo = ct;
        whi = side == 1 ? 0.5f * whi : 1.f;
        wlo = 1.f;
        side = 1;
      } else {
        hi = t;
        Fhi = ft;
        chi = ct;
        wlo = side == -1 ? 0.5f * wlo : 1.f;
        whi = 1.f;
        side = -1;
      }
    }
  }
  if (!found) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      float s = 0.f;
      for (int j = lane; j < nT; j += 32) s += (float_key(row[j]) >= cand) ? row[j] : 0.f;
      if (warp_sum(s) >= target) prefix = cand;
    }
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
  int need_eq = need_fin > 0 ? need_fin : 0;
  if (need_fin < 0) {
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
    return -1 - imin(kk, kmax);
  }
  emit_threshold(row, nT, prefix, need_eq, out, kmax);
  return count;
}

// select_mass_row with the row in registers (lane l holds entries l + 32 i, i < KPL): the same
// operations in the same order, so the same sums and the same selection, without the shared-memory
// traffic and address arithmetic of every pass. Pads hold -1, below every e. cv / ci: the warp's
// 32-entry scratch for finish_bracket.
template <int KPL>
__device__ int select_mass_row_reg(const float* __restrict__ srow, int nT, float scale, float mass,
                                   int min_k, int kmax, int32_t* out, int32_t* dev_status,
                                   float* cv, int* ci) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  float e[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int j = lane + 32 * i;
    e[i] = j < nT ? srow[j] : -INFINITY;
  }
  if (mass >= 1.f) {
    if (nT <= kmax) {
      for (int j = lane; j < nT; j += 32) out[j] = j;
      return nT;
    }
    if (lane == 0) report(dev_status, T3D_DEV_OVERFLOW);
    return -1 - kmax;
  }
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < KPL; ++i) mx = fmaxf(mx, e[i]);
  mx = warp_max(mx);
  float tot = 0.f, mn = INFINITY;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    if (lane + 32 * i < nT) {
      e[i] = expf(scale * (e[i] - mx));
      tot += e[i];
      mn = fminf(mn, e[i]);
    } else {
      e[i] = -1.f;
    }
  }
  tot = warp_sum(tot);
  mn = -warp_max(-mn);
  const float target = mass * tot;
  uint32_t prefix = 0;
  bool found = false;
  int need_fin = -1;  // need_eq from finish_bracket, when it ran
  {
    float lo = mn, hi = __int_as_float(0x3f800001);  // every e lies in [mn, 1]
    float Flo = tot, Fhi = 0.f;
    int clo = nT, chi = 0;
    float wlo = 1.f, whi = 1.f;
    int side = 0;
    for (int step = 0; step < 24; ++step) {
      if (clo - chi <= 32) {
        int base = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) {
          const bool inb = e[i] >= lo && e[i] < hi;  // pads hold -1 < lo
          const unsigned bb = __ballot_sync(0xffffffffu, inb);
          if (inb) {
            cv[base + __popc(bb & lt)] = e[i];
            ci[base + __popc(bb & lt)] = lane + 32 * i;
          }
          base += __popc(bb);
        }
        __syncwarp();
        const int c = clo - chi;
        const float v = lane < c ? cv[lane] : -2.f;
        const int ix = lane < c ? ci[lane] : 0x7fffffff;
        __syncwarp();
        prefix = float_key(finish_bracket(v, ix, c, Fhi, target, need_fin));
        found = true;
        break;
      }
      const float a = wlo * (Flo - target), bb = whi * (target - Fhi);
      float t = fmaf(hi - lo, __fdividef(a, a + bb), lo);
      if (!(t > lo && t < hi)) t = 0.5f * (lo + hi);
      if (!(t > lo && t < hi)) break;
      float ft = 0.f;
      int ct = 0;
#pragma unroll
      for (int i = 0; i < KPL; ++i) {
        if (e[i] >= t) {
          ft += e[i];
          ++ct;
        }
      }
      ft = warp_sum(ft);
      ct = warp_sum_int(ct);
      if (ft >= target) {
        lo = t;
        Flo = ft;
        clo = ct;
        whi = side == 1 ? 0.5f * whi : 1.f;
        wlo = 1.f;
        side = 1;
      } else {
        hi = t;
        Fhi = ft;
        chi = ct;
        wlo = side == -1 ? 0.5f * wlo : 1.f;
        whi = 1.f;
        side = -1;
      }
    }
  }
  if (!found) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < KPL; ++i) sum += (e[i] >= 0.f && float_key(e[i]) >= cand) ? e[i] : 0.f;
      if (warp_sum(sum) >= target) prefix = cand;
    }
  }
  float above = 0.f;
  int n_above = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    if (e[i] >= 0.f && float_key(e[i]) > prefix) {
      above += e[i];
      ++n_above;
    }
  }
  above = warp_sum(above);
  n_above = warp_sum_int(n_above);
  // Tiles tied at the threshold are taken in ascending index until the target is reached.
  int need_eq = need_fin > 0 ? need_fin : 0;
  if (need_fin < 0) {
    float acc = above;
    bool done = false;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      if (done) break;
      const bool eq = e[i] >= 0.f && float_key(e[i]) == prefix;
      unsigned eqb = __ballot_sync(0xffffffffu, eq);
      while (eqb != 0u && !done) {
        const int src = __ffs(eqb) - 1;
        const float ev = __shfl_sync(0xffffffffu, e[i], src);
        if (acc < target) {
          acc += ev;
          ++need_eq;
        }
        if (acc >= target) done = true;
        eqb &= eqb - 1u;
      }
    }
  }
  const int count = n_above + need_eq;
  const int floor_k = imin(min_k, nT);
  if (count < floor_k || count > kmax) {
    const int kk = count < floor_k ? floor_k : kmax;
    if (count > kmax && lane == 0) report(dev_status, T3D_DEV_OVERFLOW);
    return -1 - imin(kk, kmax);
  }
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const bool valid = e[i] >= 0.f;
    const uint32_t key = valid ? float_key(e[i]) : 0u;
    const bool eq = valid && key == prefix;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool sel = (valid && key > prefix) || (eq && eq_seen + __popc(eqb & lt) < need_eq);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(sb & lt);
    if (sel && pos < kmax) out[pos] = lane + 32 * i;
    written += __popc(sb);
    eq_seen += __popc(eqb);
  }
  return count;
}

// ------------------------------------------------------------ score product on the tensor cores
//
// S = pq . pk^T per head runs on the tcgen05 tensor cores in two kernels. split_kernel turns the
// fp32 operands into bf16 pairs x = hi + lo (hi = bf16(x), lo = bf16(x - hi)), stored row-major in
// the workspace; scores_tc_kernel then computes S = hi.hi + hi.lo + lo.hi for 128 query tiles
// (MMA M = 128, one TMEM lane per query tile) against 256 key tiles (two MMAs of N = 128, TMEM
// columns 0..255), K = D, fp32 in TMEM, with every operand fetched by TMA into 128-byte-swizzled
// K-major tiles. The dropped lo.lo term and the rounding of lo leave a relative error of about
// 2^-16 of sum_d |q_d k_d|, near fp32 accuracy, where a single bf16 product would err by 2^-8.
// TMEM then goes to the score rows in the workspace, one 128-byte run of 32 key tiles per thread
// and load.
constexpr int kSplitThreads = 256;
constexpr int kScThreads = 256;   // 8 warps: two per TMEM sub-partition for the read-out
constexpr int kScRows = 128;      // query tiles per CTA (MMA M)
constexpr int kScChunk = 128;     // key tiles per MMA (MMA N)
constexpr int kScCols = 256;      // key tiles per CTA (two chunks; TMEM columns allocated)

// Workspace of the selection calls: the score rows, then the four split operands.
struct SelLayout {
  size_t s_bytes, part_elems;  // score rows; elements of one split operand (B * heads * nT * D)
  int ldS;                     // score row stride (floats): nT rounded up to 4
};
inline SelLayout sel_layout(const Geo& g) {
  SelLayout l;
  l.ldS = (g.nT + 3) & ~3;
  l.s_bytes = (((size_t)g.B * g.heads * g.nT * l.ldS * sizeof(float)) + 255) & ~(size_t)255;
  l.part_elems = (size_t)g.B * g.heads * g.nT * g.D;
  return l;
}

// pq, pk -> their hi and lo bf16 parts (8 elements per thread; n8 = elements / 8 of one operand).
__global__ void __launch_bounds__(kSplitThreads) split_kernel(const float4* __restrict__ pq,
                                                              const float4* __restrict__ pk,
                                                              long n8, uint4* __restrict__ qhi,
                                                              uint4* __restrict__ qlo,
                                                              uint4* __restrict__ khi,
                                                              uint4* __restrict__ klo) {
  for (long e = (long)blockIdx.x * kSplitThreads + threadIdx.x; e < 2 * n8;
       e += (long)gridDim.x * kSplitThreads) {
    const bool isk = e >= n8;
    const long i = isk ? e - n8 : e;
    const float4* src = isk ? pk : pq;
    const float4 a = __ldg(src + 2 * i), b = __ldg(src + 2 * i + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * t]);
      const __nv_bfloat16 h1 = __float2bfloat16_rn(v[2 * t + 1]);
      const __nv_bfloat162 hp = __halves2bfloat162(h0, h1);
      const __nv_bfloat162 lp = __floats2bfloat162_rn(v[2 * t] - __bfloat162float(h0),
                                                      v[2 * t + 1] - __bfloat162float(h1));
      h[t] = *reinterpret_cast<const uint32_t*>(&hp);
      l[t] = *reinterpret_cast<const uint32_t*>(&lp);
    }
    (isk ? khi : qhi)[i] = make_uint4(h[0], h[1], h[2], h[3]);
    (isk ? klo : qlo)[i] = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

template <int kD>
struct ScSmem {
  static constexpr int kHalves = kD / 64;
  uint8_t a[2][kHalves][kScRows * 128];                      // query block: hi, lo
  uint8_t b[kScCols / kScChunk][2][kHalves][kScChunk * 128];  // key chunks: hi, lo
  uint64_t full[2];  // the query block and key chunk c landed
  uint64_t mma_done;
  uint32_t tmem_base;
};

struct ScMaps {
  CUtensorMap qhi, qlo, khi, klo;  // [B * heads * nT rows, D] bf16, box 128 rows x 64 elements
};

// Grid: (query blocks of 128) x (key blocks of 256) x (B * heads). S row i of head bh lands at
// S + (bh * nT + i) * ldS. Rows of a box past the head's last tile read the next head's (or zero
// past the tensor); their scores are never stored.
template <int kD>
__global__ void __launch_bounds__(kScThreads, 1)
    scores_tc_kernel(const __grid_constant__ ScMaps maps, Geo g, float* __restrict__ S, int ldS) {
  using namespace sm100;
  constexpr int kHalves = kD / 64;
  extern __shared__ uint8_t smem_raw[];
  ScSmem<kD>& sm = *reinterpret_cast<ScSmem<kD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr uint32_t idesc = idesc_bf16(kScRows, kScChunk, false, false);
  constexpr uint32_t kBox = kScRows * 128;  // bytes of one 128-row x 64-element box
  const int nT = g.nT, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * kScRows, j0 = blockIdx.y * kScCols;
  const long bh = blockIdx.z;
  const int nchunks = imin(kScCols, nT - j0 + kScChunk - 1) / kScChunk;  // 1 or 2
  if (threadIdx.x == 0) {
    mbar_init(&sm.full[0], 1);
    mbar_init(&sm.full[1], 1);
    mbar_init(&sm.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, (uint32_t)kScCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) {
    const int qrow = (int)(bh * nT + i0);
    mbar_expect_tx(&sm.full[0], 2 * kHalves * kBox * 2);  // query block + key chunk 0
    if (nchunks > 1) mbar_expect_tx(&sm.full[1], 2 * kHalves * kBox);
    for (int hh = 0; hh < kHalves; ++hh) {
      tma_load_2d(sm.a[0][hh], &maps.qhi, &sm.full[0], 64 * hh, qrow);
      tma_load_2d(sm.a[1][hh], &maps.qlo, &sm.full[0], 64 * hh, qrow);
    }
    for (int c = 0; c < nchunks; ++c) {
      const int krow = (int)(bh * nT + j0 + c * kScChunk);
      for (int hh = 0; hh < kHalves; ++hh) {
        tma_load_2d(sm.b[c][0][hh], &maps.khi, &sm.full[c], 64 * hh, krow);
        tma_load_2d(sm.b[c][1][hh], &maps.klo, &sm.full[c], 64 * hh, krow);
      }
    }
    const uint64_t ah = sdesc_sw128(smem_u32(sm.a[0][0]), 16, 1024);
    const uint64_t al = sdesc_sw128(smem_u32(sm.a[1][0]), 16, 1024);
    for (int c = 0; c < nchunks; ++c) {
      mbar_wait(&sm.full[c], 0, nullptr);
      tc_fence_after();
      const uint64_t bhd = sdesc_sw128(smem_u32(sm.b[c][0][0]), 16, 1024);
      const uint64_t bld = sdesc_sw128(smem_u32(sm.b[c][1][0]), 16, 1024);
      const uint32_t d = tmem + (uint32_t)(c * kScChunk);
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {  // 16 elements of D per MMA
        const int hh = kk >> 2, st = kk & 3;
        const uint64_t o = (uint64_t)((hh * kBox + st * 32) >> 4);
        mma_bf16(d, ah + o, bhd + o, idesc, kk ? 1u : 0u);
        mma_bf16(d, ah + o, bld + o, idesc, 1u);
        mma_bf16(d, al + o, bhd + o, idesc, 1u);
      }
    }
    mma_commit(&sm.mma_done);
  }
  __syncwarp();
  mbar_wait(&sm.mma_done, 0, nullptr);
  tc_fence_after();
  // TMEM -> S: warp w reads lanes 32 (w % 4) .. + 31 (query tiles i0 + 32 (w % 4) + lane) and the
  // key tiles j0 + 128 (w / 4) .. + 127 in four loads of 32 columns.
  {
    const int sp = warp & 3, part = warp >> 2;
    const int i = i0 + 32 * sp + lane;
    float* srow = S + (bh * nT + i) * (long)ldS;
#pragma unroll
    for (int c32 = 0; c32 < 4; ++c32) {
      const int col = kScChunk * part + 32 * c32;
      if (col >= nchunks * kScChunk) break;  // warp-uniform
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * sp) << 16) + (uint32_t)col, v);
      tmem_wait_ld();
      const int j = j0 + col;
      if (i < nT && j < nT) {
        if (j + 32 <= nT) {
          float4* dst = reinterpret_cast<float4*>(srow + j);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                  __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (j + e < nT) srow[j + e] = __uint_as_float(v[e]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)kScCols);
  }
}

template <int kD>
constexpr size_t sc_smem_bytes() {
  return sizeof(ScSmem<kD>) + 1024;
}

// Top-k of a row of at most 32 * KPL values (lane l holds entries l + 32 i) by an exact threshold
// search on the values: c(t) = #{x >= t} is driven to k, and when c(t) == k the set {x >= t} is
// exactly the k largest values (no tie can straddle t). The first guess is the row's mean plus z
// standard deviations, z the standard normal quantile of 1 - k/n (computed on the host): the
// pooled scores are sums of many products and close to normal, so c lands near k. Then a bracket
// lo (c > k) / hi (c < k) is narrowed by interpolating the count linearly between its ends, with
// the Illinois rule (an end kept twice in a row has its weight halved) so one end cannot stall;
// about 4 counting passes per row on the pooled scores. Rows where no such t exists (ties at the
// boundary) or that do not converge in kMaxSteps go to the bit-by-bit key search, which breaks
// ties toward the lower index.
template <int KPL>
__device__ int select_topk_row_fast(const float* row, int n, int k, float z, int32_t* out) {
  constexpr int kMaxSteps = 24;
  k = imin(k, n);
  if (k <= 0) return 0;
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  float x[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int j = lane + 32 * i;
    x[i] = j < n ? row[j] : -INFINITY;
  }
  if (k == n) {
    for (int j = lane; j < n; j += 32) out[j] = j;
    return n;
  }
  float mx = -INFINITY, mn = INFINITY, s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    if (lane + 32 * i < n) {
      mx = fmaxf(mx, x[i]);
      mn = fminf(mn, x[i]);
      s1 += x[i];
      s2 = fmaf(x[i], x[i], s2);
    }
  }
  mx = sm100::redux_max(mx);
  mn = -sm100::redux_max(-mn);
  s1 = warp_sum(s1);
  s2 = warp_sum(s2);
  auto count_ge = [&](float t) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += x[i] >= t ? 1 : 0;
    return (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
  };
  float lo = mn, hi = mx;
  int clo = n, chi = count_ge(mx);
  float thr = 0.f;
  bool found = false;
  if (chi < k && lo < hi) {
    const float mean = s1 / (float)n;
    const float sd = sqrtf(fmaxf(s2 / (float)n - mean * mean, 0.f));
    float t = fmaf(z, sd, mean);
    float wlo = 1.f, whi = 1.f;
    int side = 0;  // end moved at the previous step: 1 = lo, -1 = hi
    for (int step = 0; step < kMaxSteps; ++step) {
      if (step > 0) {
        const float a = wlo * (float)(clo - k), b = whi * (float)(k - chi);
        t = fmaf(hi - lo, __fdividef(a, a + b), lo);
      }
      if (!(t > lo && t < hi)) t = 0.5f * (lo + hi);
      if (!(t > lo && t < hi)) break;  // the bracket is down to adjacent floats
      const int c = count_ge(t);
      if (c == k) {
        thr = t;
        found = true;
        break;
      }
      if (c > k) {
        lo = t;
        clo = c;
        whi = side == 1 ? 0.5f * whi : 1.f;
        wlo = 1.f;
        side = 1;
      } else {
        hi = t;
        chi = c;
        wlo = side == -1 ? 0.5f * wlo : 1.f;
        whi = 1.f;
        side = -1;
      }
    }
  }
  if (!found) return select_topk_row_reg<KPL>(row, n, k, out);
  int written = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const bool sel = x[i] >= thr;  // pads are -inf
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(sb & lt)] = lane + 32 * i;
    written += __popc(sb);
  }
  return k;
}

// One warp per query tile: its top-k key tiles from its score row. KPL = 0: the radix select for
// rows too long for registers.
template <int KPL>
__global__ void __launch_bounds__(kSelThreads) topk_rows_kernel(Geo g, const float* __restrict__ S,
                                                                int ldS, int k, float z,
                                                                int32_t* __restrict__ kv_idx,
                                                                int32_t* __restrict__ kv_cnt) {
  __shared__ int hist[KPL == 0 ? kSelThreads / 32 : 1][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long rows = (long)g.B * g.heads * g.nT;
  const int kk = imin(k, g.nT);
  for (long r = (long)blockIdx.x * (kSelThreads / 32) + w; r < rows;
       r += (long)gridDim.x * (kSelThreads / 32)) {
    int n;
    if constexpr (KPL == 0) n = select_topk_row(S + r * ldS, g.nT, kk, kv_idx + r * kk, hist[w]);
    else n = select_topk_row_fast<KPL>(S + r * ldS, g.nT, kk, z, kv_idx + r * kk);
    if (lane == 0) kv_cnt[r] = n;
  }
}

// One warp per query tile: cumulative-mass selection from its score row, staged in the warp's
// shared-memory row buffer (the search reads it many times).
template <int KPL>
__global__ void __launch_bounds__(kSelThreads) mass_rows_kernel(Geo g, const float* __restrict__ S,
                                                                int ldS, float scale, float mass,
                                                                int min_k, int kmax,
                                                                int32_t* __restrict__ kv_idx,
                                                                int32_t* __restrict__ kv_cnt,
                                                                int32_t* dev_status) {
  extern __shared__ float rowbuf[];  // KPL == 0: [8 warps][nT]
  __shared__ float cv[kSelThreads / 32][32];  // finish_bracket's candidates, per warp
  __shared__ int ci[kSelThreads / 32][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nT = g.nT;
  const long rows = (long)g.B * g.heads * nT;
  for (long r = (long)blockIdx.x * (kSelThreads / 32) + w; r < rows;
       r += (long)gridDim.x * (kSelThreads / 32)) {
    const float* src = S + r * ldS;
    int count;
    if constexpr (KPL == 0) {
      float* row = rowbuf + (long)w * nT;
      for (int j = lane; j < nT; j += 32) row[j] = src[j];
      __syncwarp();
      count = select_mass_row(row, nT, scale, mass, min_k, kmax, kv_idx + r * kmax, dev_status,
                              cv[w], ci[w]);
    } else {
      count = select_mass_row_reg<KPL>(src, nT, scale, mass, min_k, kmax, kv_idx + r * kmax,
                                       dev_status, cv[w], ci[w]);
    }
    if (lane == 0) kv_cnt[r] = count;  // -1 - k: mass_fix_kernel keeps the top k instead
    __syncwarp();
  }
}

// One warp per row that mass_rows_kernel marked (kv_cnt = -1 - k): its k highest-scoring tiles
// from the score row (ascending indices, ties to the lower index).
__global__ void __launch_bounds__(kSelThreads) mass_fix_kernel(Geo g, const float* __restrict__ S,
                                                               int ldS, int kmax,
                                                               int32_t* __restrict__ kv_idx,
                                                               int32_t* __restrict__ kv_cnt) {
  __shared__ int hist[kSelThreads / 32][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long rows = (long)g.B * g.heads * g.nT;
  for (long r = (long)blockIdx.x * (kSelThreads / 32) + w; r < rows;
       r += (long)gridDim.x * (kSelThreads / 32)) {
    const int c = kv_cnt[r];
    if (c >= 0) continue;
    __syncwarp();
    const int n = select_topk_any(S + r * ldS, g.nT, -1 - c, kv_idx + r * kmax, hist[w]);
    __syncwarp();
    if (lane == 0) kv_cnt[r] = n;
  }
}

// One warp per query tile of a packed buffer: its kept tiles by region (tile3d_packed.h).
// Exempt mode: prefix tiles for every row, everything for a prefix row, else the top k[r] of each
// region's stretch of the score row, shifted to buffer indices; regions follow the prefix in tile
// order, so the concatenation is ascending. Compete mode: one top-k over the row.
__global__ void __launch_bounds__(kSelThreads) spans_rows_kernel(Geo g, const float* __restrict__ S,
                                                                 int ldS, SpanSpec sp, int kmax,
                                                                 int32_t* __restrict__ kv_idx,
                                                                 int32_t* __restrict__ kv_cnt) {
  __shared__ int hist[kSelThreads / 32][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long rows = (long)g.B * g.heads * g.nT;
  for (long r = (long)blockIdx.x * (kSelThreads / 32) + w; r < rows;
       r += (long)gridDim.x * (kSelThreads / 32)) {
    const int i = (int)(r % g.nT);
    const float* row = S + r * ldS;
    int32_t* out = kv_idx + r * kmax;
    int cnt;
    if (sp.mode == T3D_PACKED_DENSE || (sp.mode == T3D_PACKED_EXEMPT && i < sp.n_prefix)) {
      for (int j = lane; j < g.nT; j += 32) out[j] = j;
      cnt = g.nT;
    } else if (sp.mode == T3D_PACKED_COMPETE) {
      cnt = select_topk_any(row, g.nT, sp.k_total, out, hist[w]);
    } else {
      for (int j = lane; j < sp.n_prefix; j += 32) out[j] = j;
      cnt = sp.n_prefix;
      for (int q = 0; q < sp.n_regions; ++q) {
        const int lo = sp.lo[q];
        const int c = select_topk_any(row + lo, sp.hi[q] - lo, sp.k[q], out + cnt, hist[w]);
        __syncwarp();
        for (int j = lane; j < c; j += 32) out[cnt + j] += lo;
        cnt += c;
      }
    }
    if (lane == 0) kv_cnt[r] = cnt;
    __syncwarp();
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
// One CTA per (batch, head, 64-row block), 8 warps of 8 rows each. Lane l of a warp holds 16-byte
// chunk l % kChunks of rows 8 w + kRowsPerLoad t + l / kChunks (t < kLoads) in registers as fp32;
// column sums, row norms and dot products with the block mean come from warp shuffles and a small
// shared-memory combine across warps. The rows go to shared memory only when some row is pruned
// (for the source search), and the kept-row mean is the block mean when nothing is pruned.
// The kernel is bound by load latency: at D = 128 four CTAs per SM (60 registers, no spills; the
// shared memory allows four) keep a third more rows in flight than the three that 74 registers
// allowed.
template <int kD>
__global__ void __launch_bounds__(kPruneThreads, kD == 128 ? 4 : 1) prune_kernel(Geo g, const __nv_bfloat16* __restrict__ q,
                                                              float cos_thresh, int keep_size,
                                                              uint8_t* __restrict__ keep,
                                                              uint8_t* __restrict__ src_row,
                                                              float* __restrict__ pq_kept) {
  constexpr int kChunks = kD / 8;              // 16-byte chunks of a row
  constexpr int kRowsPerLoad = 32 / kChunks;   // rows one warp-wide load covers
  constexpr int kWarps = kPruneThreads / 32;
  constexpr int kRowsPerWarp = kTileElems / kWarps;
  constexpr int kLoads = kRowsPerWarp / kRowsPerLoad;
  constexpr int ld = kD + 1;
  extern __shared__ float sm[];
  float* qs = sm;                          // [64][D+1], filled only when a row is pruned
  __shared__ float part[kWarps][kD];       // per-warp column sums
  __shared__ float mu[kD];
  __shared__ float n2[kTileElems], cosm[kTileElems];
  __shared__ int keep_s[kTileElems], src_s[kTileElems];
  __shared__ float mu_n2;
  __shared__ int n_keep;
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int chunk = lane % kChunks, sub = lane / kChunks;
  const long row_stride = (long)g.heads_total * kD;
  const __nv_bfloat16* base =
      q + ((long)b * g.Lp + (long)i * kTileElems) * row_stride + (long)(g.head0 + h) * kD;
  float x[kLoads][8];
  uint4 u[kLoads];
#pragma unroll
  for (int t = 0; t < kLoads; ++t) {
    const int r = kRowsPerWarp * w + kRowsPerLoad * t + sub;
    u[t] = __ldg(reinterpret_cast<const uint4*>(base + r * row_stride) + chunk);
  }
#pragma unroll
  for (int t = 0; t < kLoads; ++t) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[t]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      x[t][2 * e] = f.x;
      x[t][2 * e + 1] = f.y;
    }
  }
  // Column sums over this warp's rows: over t in registers, then over the lanes holding the same
  // chunk of other rows.
  {
    float cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float v = 0.f;
#pragma unroll
      for (int t = 0; t < kLoads; ++t) v += x[t][e];
#pragma unroll
      for (int o = kChunks; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      cs[e] = v;
    }
    if (sub == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) part[w][chunk * 8 + e] = cs[e];
    }
  }
  __syncthreads();
  if (tid < kD) {
    float v = 0.f;
#pragma unroll
    for (int q2 = 0; q2 < kWarps; ++q2) v += part[q2][tid];
    mu[tid] = v / (float)kTileElems;
  }
  __syncthreads();
  if (w == 0) {
    float v = 0.f;
    for (int d = lane; d < kD; d += 32) v += mu[d] * mu[d];
    v = warp_sum(v);
    if (lane == 0) mu_n2 = v;
  }
  __syncthreads();
  // Row norms and dot products with the mean: per lane over its chunk, then over the chunk lanes.
#pragma unroll
  for (int t = 0; t < kLoads; ++t) {
    float a = 0.f, dm = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      a = fmaf(x[t][e], x[t][e], a);
      dm = fmaf(x[t][e], mu[chunk * 8 + e], dm);
    }
#pragma unroll
    for (int o = 1; o < kChunks; o <<= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      dm += __shfl_xor_sync(0xffffffffu, dm, o);
    }
    if (chunk == 0) {
      const int r = kRowsPerWarp * w + kRowsPerLoad * t + sub;
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
  const long blk = (((long)b * g.heads + h) * g.nT + i);
  const int nk = n_keep;
  if (nk == kTileElems) {
    // Nothing pruned: every row is its own source and the kept-row mean is the block mean.
    if (tid < kD) pq_kept[blk * kD + tid] = mu[tid];
    if (tid < kTileElems) {
      keep[blk * kTileElems + tid] = 1;
      src_row[blk * kTileElems + tid] = (uint8_t)tid;
    }
    return;
  }
  // Some rows are pruned: the rows go to shared memory for the source search, and the kept-row
  // mean is summed from the registers with the keep mask.
#pragma unroll
  for (int t = 0; t < kLoads; ++t) {
    const int r = kRowsPerWarp * w + kRowsPerLoad * t + sub;
#pragma unroll
    for (int e = 0; e < 8; ++e) qs[r * ld + chunk * 8 + e] = x[t][e];
  }
  {
    float cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float v = 0.f;
#pragma unroll
      for (int t = 0; t < kLoads; ++t)
        v += keep_s[kRowsPerWarp * w + kRowsPerLoad * t + sub] ? x[t][e] : 0.f;
#pragma unroll
      for (int o = kChunks; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      cs[e] = v;
    }
    __syncthreads();  // every warp is past reading `part` above
    if (sub == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) part[w][chunk * 8 + e] = cs[e];
    }
  }
  __syncthreads();
  if (tid < kD) {
    float v = 0.f;
#pragma unroll
    for (int q2 = 0; q2 < kWarps; ++q2) v += part[q2][tid];
    pq_kept[blk * kD + tid] = v / (float)nk;
  }
  // Each pruned row takes the most cosine-similar kept row (lowest index on ties).
  for (int r = w; r < kTileElems; r += kWarps) {
    if (keep_s[r]) {
      if (lane == 0) src_s[r] = r;
      continue;
    }
    float best = -INFINITY;
    int bj = kTileElems;
    for (int j = lane; j < kTileElems; j += 32) {
      if (!keep_s[j]) continue;
      float dot = 0.f;
      for (int d = 0; d < kD; ++d) dot = fmaf(qs[r * ld + d], qs[j * ld + d], dot);
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
  if (tid < kTileElems) {
    keep[blk * kTileElems + tid] = (uint8_t)keep_s[tid];
    src_row[blk * kTileElems + tid] = (uint8_t)src_s[tid];
  }
}

}  // namespace

size_t select_workspace_bytes(const Geo& g) {
  const SelLayout l = sel_layout(g);
  return l.s_bytes + 4 * l.part_elems * sizeof(__nv_bfloat16);
}

namespace {

// z with P(N(0, 1) > z) = p, by bisection on the host's erfc (a starting guess only: accuracy
// beyond a few digits does not matter). p = 1 gives the lower end of the search range.
float upper_normal_quantile(double p) {
  double lo = -8.0, hi = 8.0;
  for (int it = 0; it < 60; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * erfc(mid / sqrt(2.0)) > p) lo = mid;
    else hi = mid;
  }
  return (float)(0.5 * (lo + hi));
}

int sel_grid(const Geo& g) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long rows = (long)g.B * g.heads * g.nT;
  long blocks = (rows + (kSelThreads / 32) - 1) / (kSelThreads / 32);
  const long cap = (long)(sms > 0 ? sms : 148) * 8;
  return (int)(blocks < cap ? blocks : cap);
}

template <int kD>
cudaError_t launch_scores_d(const Geo& g, const ScMaps& maps, float* S, int ldS, cudaStream_t s) {
  const size_t smem = sc_smem_bytes<kD>();
  cudaError_t e = cudaFuncSetAttribute(scores_tc_kernel<kD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nT + kScRows - 1) / kScRows, (g.nT + kScCols - 1) / kScCols, g.B * g.heads);
  scores_tc_kernel<kD><<<grid, kScThreads, smem, s>>>(maps, g, S, ldS);
  return cudaGetLastError();
}

// Split the operands into the workspace, then the score rows into its head.
cudaError_t launch_scores(const Geo& g, const float* pq, const float* pk, void* workspace,
                          float** S, int* ldS, cudaStream_t s) {
  const SelLayout l = sel_layout(g);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* part = reinterpret_cast<__nv_bfloat16*>(ws + l.s_bytes);
  __nv_bfloat16 *qhi = part, *qlo = part + l.part_elems, *khi = part + 2 * l.part_elems,
                *klo = part + 3 * l.part_elems;
  const long n8 = (long)(l.part_elems / 8);
  long blocks = (2 * n8 + kSplitThreads - 1) / kSplitThreads;
  if (blocks > 148L * 16) blocks = 148L * 16;
  split_kernel<<<(unsigned)blocks, kSplitThreads, 0, s>>>(
      reinterpret_cast<const float4*>(pq), reinterpret_cast<const float4*>(pk), n8,
      reinterpret_cast<uint4*>(qhi), reinterpret_cast<uint4*>(qlo), reinterpret_cast<uint4*>(khi),
      reinterpret_cast<uint4*>(klo));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ScMaps maps;
  const cuuint64_t dims[2] = {(cuuint64_t)g.D, (cuuint64_t)g.B * g.heads * g.nT};
  const cuuint64_t strides[1] = {(cuuint64_t)g.D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kScRows};
  if (!encode_bf16_map(&maps.qhi, qhi, 2, dims, strides, box) ||
      !encode_bf16_map(&maps.qlo, qlo, 2, dims, strides, box) ||
      !encode_bf16_map(&maps.khi, khi, 2, dims, strides, box) ||
      !encode_bf16_map(&maps.klo, klo, 2, dims, strides, box))
    return cudaErrorInvalidValue;
  *S = reinterpret_cast<float*>(ws);
  *ldS = l.ldS;
  return g.D == 128 ? launch_scores_d<128>(g, maps, *S, l.ldS, s)
                    : launch_scores_d<64>(g, maps, *S, l.ldS, s);
}

}  // namespace

cudaError_t launch_select_topk(const Geo& g, const float* pq, const float* pk, int k,
                               int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                               int32_t* dev_status, cudaStream_t s) {
  (void)dev_status;
  float* S = nullptr;
  int ldS = 0;
  cudaError_t e = launch_scores(g, pq, pk, workspace, &S, &ldS, s);
  if (e != cudaSuccess) return e;
  const int grid = sel_grid(g);
  const float z = upper_normal_quantile((double)imin(k, g.nT) / g.nT);
  if (g.nT <= 128)
    topk_rows_kernel<4><<<grid, kSelThreads, 0, s>>>(g, S, ldS, k, z, kv_idx, kv_cnt);
  else if (g.nT <= 256)
    topk_rows_kernel<8><<<grid, kSelThreads, 0, s>>>(g, S, ldS, k, z, kv_idx, kv_cnt);
  else if (g.nT <= 512)
    topk_rows_kernel<16><<<grid, kSelThreads, 0, s>>>(g, S, ldS, k, z, kv_idx, kv_cnt);
  else if (g.nT <= 1024)
    topk_rows_kernel<32><<<grid, kSelThreads, 0, s>>>(g, S, ldS, k, z, kv_idx, kv_cnt);
  else if (g.nT <= kRegSelectMax)
    topk_rows_kernel<48><<<grid, kSelThreads, 0, s>>>(g, S, ldS, k, z, kv_idx, kv_cnt);
  else
    topk_rows_kernel<0><<<grid, kSelThreads, 0, s>>>(g, S, ldS, k, z, kv_idx, kv_cnt);
  return cudaGetLastError();
}

cudaError_t launch_select_mass(const Geo& g, const float* pq, const float* pk, float scale,
                               float mass, int min_k, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                               void* workspace, int32_t* dev_status, cudaStream_t s) {
  float* S = nullptr;
  int ldS = 0;
  cudaError_t e = launch_scores(g, pq, pk, workspace, &S, &ldS, s);
  if (e != cudaSuccess) return e;
  const int grid = sel_grid(g);
  if (g.nT <= 128)
    mass_rows_kernel<4><<<grid, kSelThreads, 0, s>>>(g, S, ldS, scale, mass, min_k, kmax, kv_idx,
                                                     kv_cnt, dev_status);
  else if (g.nT <= 256)
    mass_rows_kernel<8><<<grid, kSelThreads, 0, s>>>(g, S, ldS, scale, mass, min_k, kmax, kv_idx,
                                                     kv_cnt, dev_status);
  else if (g.nT <= 512)
    mass_rows_kernel<16><<<grid, kSelThreads, 0, s>>>(g, S, ldS, scale, mass, min_k, kmax, kv_idx,
                                                      kv_cnt, dev_status);
  else if (g.nT <= 1024)
    mass_rows_kernel<32><<<grid, kSelThreads, 0, s>>>(g, S, ldS, scale, mass, min_k, kmax, kv_idx,
                                                      kv_cnt, dev_status);
  else {
    const size_t smem = (size_t)(kSelThreads / 32) * (size_t)g.nT * sizeof(float);
    e = cudaFuncSetAttribute(mass_rows_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    mass_rows_kernel<0><<<grid, kSelThreads, smem, s>>>(g, S, ldS, scale, mass, min_k, kmax,
                                                        kv_idx, kv_cnt, dev_status);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mass_fix_kernel<<<sel_grid(g), kSelThreads, 0, s>>>(g, S, ldS, kmax, kv_idx, kv_cnt);
  return cudaGetLastError();
}

cudaError_t launch_select_spans(const Geo& g, const float* pq, const float* pk, const SpanSpec& sp,
                                int kmax, int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                                cudaStream_t s) {
  float* S = nullptr;
  int ldS = 0;
  cudaError_t e = launch_scores(g, pq, pk, workspace, &S, &ldS, s);
  if (e != cudaSuccess) return e;
  spans_rows_kernel<<<sel_grid(g), kSelThreads, 0, s>>>(g, S, ldS, sp, kmax, kv_idx, kv_cnt);
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
  // Dynamic shared memory: the block's rows as fp32 (read only when some row is pruned).
  const size_t smem = (size_t)kTileElems * (g.D + 1) * sizeof(float);
  dim3 grid(g.nT, g.heads, g.B);
  const __nv_bfloat16* qq = static_cast<const __nv_bfloat16*>(q);
  cudaError_t e;
  if (g.D == 128) {
    e = cudaFuncSetAttribute(prune_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    prune_kernel<128><<<grid, kPruneThreads, smem, s>>>(g, qq, cos_thresh, keep_size, keep,
                                                        src_row, pq_kept);
  } else {
    e = cudaFuncSetAttribute(prune_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    prune_kernel<64><<<grid, kPruneThreads, smem, s>>>(g, qq, cos_thresh, keep_size, keep,
                                                       src_row, pq_kept);
  }
  return cudaGetLastError();
}

}  // namespace t3d
