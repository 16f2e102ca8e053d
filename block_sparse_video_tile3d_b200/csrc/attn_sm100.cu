// Fine stage on the sm_100a tensor cores: block-sparse softmax attention over the kept
// (query tile, key tile) pairs with tcgen05 MMAs accumulating in tensor memory (TMEM) and the kept
// key/value tiles fetched by TMA.
//
// FastVideo API docs, bsa_attn page, BSAAttentionImpl.__init__ / forward: bidirectional attention,
// one KV head per query head, softmax scale 1/sqrt(D), tile-ordered [B, L, heads, D] bf16 tensors,
// sparse attention per kept block pair, pruned query rows reconstructed afterwards.
//
// Shape of the computation. A query tile has 64 rows, and a tcgen05 MMA with M = 64 costs as much
// as one with M = 128, so the kernel puts KEYS on the M dimension: each step takes a PAIR of kept key
// tiles (128 keys) and computes
//     S^T[128 keys, 64 queries]  = K_pair . Q^T          (A = K pair, K-major; B = Q, K-major)
//     O^T[D, 64 queries]        += V_pair^T . P^T        (A = V pair, MN-major; B = P^T, MN-major)
// both with M = 128, N = 64, accumulating in fp32 in TMEM. An odd last tile is paired with a copy of
// itself whose keys are all masked.
//
// Roles (one persistent CTA per SM, work units = (batch, head, query tile), static round robin):
//   warp 0        TMA producer for Q (once per unit) and the K pairs (2-stage ring)
//   warp 1        TMEM allocation; one thread issues the S^T MMA chains and their commits
//   warps 2..17   softmax and epilogue: four warpgroups, each owning 16 of the 64 query columns; a
//                 thread owns TMEM lane t (a key of S^T, a column d of O^T) for those 16 queries
//   warp 18       TMA producer for the V pairs (3-stage ring: a V pair waits for its PV MMAs)
//   warp 19       one thread issues the PV MMA chains and their commits
// The softmax is latency-bound (short dependent chains per step, barriers, shared-memory traffic
// that the tensor core's operand reads crowd out), so it is spread over 16 warps, four per SM
// sub-partition; the two MMA-issuing threads let the next scores be computed while P^T waits.
//
// Softmax. Each softmax thread holds one key's 16 logits. The shift subtracted before exp2 is a
// per-query value m[q] shared through shared memory; it is only raised (a "slow step": per-query
// maxima by warp reductions, then a rescale of O^T and of the running sums) when some logit exceeds
// m[q] by more than kShiftSlack (log2 units). Any shift gives the same softmax; the bound keeps P
// within [0, 2^kShiftSlack] so nothing overflows. The first step of a unit is always slow. Each
// thread keeps running sums of P for its own key over all steps; they are reduced across the 128
// threads of its warpgroup once per unit.
//
// Every mbarrier wait is bounded; on a timeout the CTA records T3D_DEV_TIMEOUT, stops issuing work,
// waits (bounded) for its copies and MMAs in flight, frees TMEM and returns.
#include "kernels.h"
#include "sm100.cuh"

namespace t3d {
namespace {

using namespace sm100;

constexpr int kD = 128;             // head dimension handled by this kernel
constexpr int kHalves = kD / 64;    // 64-element (128-byte) column blocks of a row
constexpr int kKStages = 2;         // K-pair ring depth
constexpr int kVStages = 3;         // V-pair ring depth (V waits longer: until its PV MMAs)
constexpr int kQW = 16;             // query columns per softmax warpgroup
constexpr int kWGs = 64 / kQW;      // softmax warpgroups
constexpr int kSoftmaxThreads = 128;
constexpr int kSoftmaxBar = 1;      // named barrier ids 1 .. kWGs: one per softmax warpgroup
constexpr int kSoftmaxWarps = 4 * kWGs;
constexpr int kThreads = 32 * (kSoftmaxWarps + 4);  // + Q/K producer, two MMA issuers, V producer
constexpr float kShiftSlack = 8.f;  // log2 units: P <= 256 between shift updates
constexpr int kSBufs = 2;           // S^T buffers in TMEM
constexpr uint32_t kColS = 0;       // S^T buffer b: columns [64 b, 64 b + 64)
constexpr uint32_t kColO = 64 * kSBufs;  // O^T: 64 columns after the S^T buffers
constexpr uint32_t kTmemCols = kColO + 64 <= 256 ? 256 : 512;

constexpr uint32_t kTileBytes = 64 * 128;                  // 64 rows x 128 B (one half of a tile)
constexpr uint32_t kQBytes = kHalves * kTileBytes;         // 16 KB
constexpr uint32_t kPairBytes = kHalves * 2 * kTileBytes;  // 32 KB: two tiles, both halves
constexpr uint32_t kPBytes = 128 * 128;                    // P^T: 128 keys x 64 queries bf16

struct alignas(1024) SmemLayout {
  uint8_t q[kQBytes];
  uint8_t k[kKStages][kPairBytes];
  uint8_t v[kVStages][kPairBytes];
  uint8_t p[2][kPBytes];
  uint64_t q_full, q_empty, o_full, o_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kSBufs], s_empty[kSBufs];
  uint64_t p_full[2], p_empty[2];
  uint64_t drain;
  uint64_t wg_sync;  // rendezvous of both softmax warpgroups (bounded, unlike bar.sync)
  alignas(16) float shift[64];   // current per-query shift (log2 units)
  alignas(16) float thr[64];     // raw logit above which a step is slow: (shift + slack) / scale
  alignas(16) float nsh[64];     // -shift, or 0 while the shift is -inf
  alignas(16) float red[4][64];  // per-warp partial results
  alignas(16) float alpha[64];   // rescale factors of a slow step
  alignas(16) float lsum[64];    // per-query softmax denominators
  uint8_t vc[kMaxTiles];         // valid token count of every tile
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(SmemLayout) + 1024 <= 232448, "shared memory per CTA");
constexpr int kAbsent = -0x7fffffff - 1;  // list entry beyond kv_cnt

constexpr uint32_t idesc_s = idesc_bf16(128, 64, false, false);
constexpr uint32_t idesc_o = idesc_bf16(128, 64, true, true);

struct UnitInfo {
  int b, h, i, cnt, npairs;
  const int32_t* list;
};

__device__ __forceinline__ UnitInfo unit_info(const Geo& g, const AttnArgs& a, int u) {
  UnitInfo r;
  r.i = u % g.nT;
  const int bh = u / g.nT;
  r.h = bh % g.heads;
  r.b = bh / g.heads;
  int c = a.kv_cnt[(long)bh * g.nT + r.i];
  c = c < 0 ? 0 : (c > a.kmax ? a.kmax : c);
  r.cnt = c;
  r.npairs = (c + 1) >> 1;
  r.list = a.kv_idx + ((long)bh * g.nT + r.i) * a.kmax;
  return r;
}

// Key tile of entry e of the list, or -1 if absent / out of range.
__device__ __forceinline__ int list_tile(const Geo& g, const UnitInfo& u, int e) {
  if (e >= u.cnt) return -1;
  const int j = u.list[e];
  return (j >= 0 && j < g.nT) ? j : -1;
}

__device__ __forceinline__ void fail(SmemLayout& s, int32_t* status) {
  s.abort = 1;
  report(status, T3D_DEV_TIMEOUT);
}

struct Maps {
  CUtensorMap q, k, v;
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ Maps maps, Geo g, AttnArgs a, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  SmemLayout& s = *reinterpret_cast<SmemLayout*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_units = g.B * g.heads * g.nT;
  volatile int* abort_flag = &s.abort;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    mbar_init(&s.q_empty, 1);
    mbar_init(&s.o_full, 1);
    mbar_init(&s.o_empty, kWGs * kSoftmaxThreads);
    for (int t = 0; t < kKStages; ++t) { mbar_init(&s.k_full[t], 1); mbar_init(&s.k_empty[t], 1); }
    for (int t = 0; t < kVStages; ++t) { mbar_init(&s.v_full[t], 1); mbar_init(&s.v_empty[t], 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.p_full[t], kWGs * kSoftmaxThreads);
      mbar_init(&s.p_empty[t], 1);
    }
    for (int t = 0; t < kSBufs; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.s_empty[t], kWGs * kSoftmaxThreads);
    }
    mbar_init(&s.drain, 2);  // one commit from each MMA-issuing thread
    mbar_init(&s.wg_sync, kWGs * kSoftmaxThreads);
    s.abort = 0;
    fence_mbar_init();
  }
  for (int t = threadIdx.x; t < g.nT; t += kThreads) s.vc[t] = (uint8_t)tile_valid_count(g, t);
  if (warp == 0 && lane == 0) {
    tma_prefetch(&maps.q);
    tma_prefetch(&maps.k);
    tma_prefetch(&maps.v);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------- Q and K producer
    if (lane == 0) {
      int active = 0;
      long gp0 = 0;
      long issued = 0;  // K pairs issued
      for (int u = blockIdx.x; u < total_units && !*abort_flag; u += gridDim.x) {
        const UnitInfo ui = unit_info(g, a, u);
        if (ui.npairs == 0) continue;
        if (!mbar_wait(&s.q_empty, (active & 1) ^ 1, abort_flag)) { fail(s, a.dev_status); break; }
        const int row0 = ui.b * g.Lp + ui.i * kTileElems;
        mbar_expect_tx(&s.q_full, kQBytes);
        for (int hh = 0; hh < kHalves; ++hh)
          tma_load_3d(s.q + hh * kTileBytes, &maps.q, &s.q_full, 64 * hh, ui.h, row0);
        bool ok = true;
        for (int n = 0; n < ui.npairs; ++n) {
          const long gp = gp0 + n;
          const int ks = (int)(gp % kKStages);
          if (!mbar_wait(&s.k_empty[ks], ((gp / kKStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
          int ja = list_tile(g, ui, 2 * n), jb = list_tile(g, ui, 2 * n + 1);
          if (ja < 0) ja = 0;  // masked in the softmax; any finite tile will do
          if (jb < 0) jb = ja;
          mbar_expect_tx(&s.k_full[ks], kPairBytes);
          for (int hh = 0; hh < kHalves; ++hh) {
            uint8_t* dst = s.k[ks] + hh * 2 * kTileBytes;
            tma_load_3d(dst, &maps.k, &s.k_full[ks], 64 * hh, ui.h, ui.b * g.Lp + ja * kTileElems);
            tma_load_3d(dst + kTileBytes, &maps.k, &s.k_full[ks], 64 * hh, ui.h,
                        ui.b * g.Lp + jb * kTileElems);
          }
          ++issued;
        }
        if (!ok) { fail(s, a.dev_status); break; }
        gp0 += ui.npairs;
        ++active;
      }
      // Drain: the last loads issued must land before the CTA can exit.
      for (long gp = issued - kKStages; gp < issued; ++gp)
        if (gp >= 0) mbar_wait(&s.k_full[gp % kKStages], (gp / kKStages) & 1, nullptr);
    }
  } else if (warp == 2 + kSoftmaxWarps) {
    // ------------------------------------------------------------- V producer
    if (lane == 0) {
      long gp0 = 0, issued = 0;
      for (int u = blockIdx.x; u < total_units && !*abort_flag; u += gridDim.x) {
        const UnitInfo ui = unit_info(g, a, u);
        if (ui.npairs == 0) continue;
        bool ok = true;
        for (int n = 0; n < ui.npairs; ++n) {
          const long gp = gp0 + n;
          const int vs = (int)(gp % kVStages);
          if (!mbar_wait(&s.v_empty[vs], ((gp / kVStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
          int ja = list_tile(g, ui, 2 * n), jb = list_tile(g, ui, 2 * n + 1);
          if (ja < 0) ja = 0;
          if (jb < 0) jb = ja;
          mbar_expect_tx(&s.v_full[vs], kPairBytes);
          for (int hh = 0; hh < kHalves; ++hh) {
            uint8_t* dst = s.v[vs] + hh * 2 * kTileBytes;
            tma_load_3d(dst, &maps.v, &s.v_full[vs], 64 * hh, ui.h, ui.b * g.Lp + ja * kTileElems);
            tma_load_3d(dst + kTileBytes, &maps.v, &s.v_full[vs], 64 * hh, ui.h,
                        ui.b * g.Lp + jb * kTileElems);
          }
          ++issued;
        }
        if (!ok) { fail(s, a.dev_status); break; }
        gp0 += ui.npairs;
      }
      for (long gp = issued - kVStages; gp < issued; ++gp)
        if (gp >= 0) mbar_wait(&s.v_full[gp % kVStages], (gp / kVStages) & 1, nullptr);
    }
  } else if (warp == 1 || warp == 3 + kSoftmaxWarps) {
    // ------------------------------------------------------------- MMA issuers
    // Two threads issue the MMAs: warp 1 the S^T chains, warp 11 the PV chains. Each waits only on
    // what its own chains read, so a late P^T never holds back the next scores (and vice versa);
    // each commit tracks the MMAs of the thread that issues it.
    if (lane == 0) {
      int active = 0;
      long gp0 = 0;
      bool ok = true;
      // Shared-memory descriptors are linear in the start address (bits 0-13 hold address >> 4 and
      // every buffer lies below 256 KB), so each MMA's operands are a base descriptor plus a
      // constant: the issuing thread builds none of them in the loop.
      const uint64_t dq = sdesc_sw128(smem_u32(s.q), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(s.k[0]), 16, 1024);
      const uint64_t dv = sdesc_sw128(smem_u32(s.v[0]), 2 * kTileBytes, 1024);
      const uint64_t dp = sdesc_sw128(smem_u32(s.p[0]), kPBytes, 1024);
      const bool s_issuer = warp == 1;
      for (int u = blockIdx.x; u < total_units && ok && !*abort_flag; u += gridDim.x) {
        const UnitInfo ui = unit_info(g, a, u);
        if (ui.npairs == 0) continue;
        if (s_issuer) {
          if (!mbar_wait(&s.q_full, active & 1, abort_flag)) { ok = false; break; }
          for (int n = 0; n < ui.npairs && ok; ++n) {
            const long gp = gp0 + n;
            const int ks = (int)(gp % kKStages);
            const int sb = (int)(gp % kSBufs);
            if (!mbar_wait(&s.k_full[ks], (gp / kKStages) & 1, abort_flag) ||
                !mbar_wait(&s.s_empty[sb], ((gp / kSBufs) & 1) ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da0 = dk + (uint64_t)(ks * (kPairBytes >> 4));
            const uint32_t d_s = tmem + kColS + sb * 64;
#pragma unroll
            for (int hh = 0; hh < kHalves; ++hh) {
#pragma unroll
              for (int st = 0; st < 4; ++st)  // 16 elements of D (32 bytes) per MMA
                mma_bf16(d_s, da0 + ((hh * 2 * kTileBytes + st * 32) >> 4),
                         dq + ((hh * kTileBytes + st * 32) >> 4), idesc_s, (hh | st) ? 1u : 0u);
            }
            mma_commit(&s.s_full[sb]);
            mma_commit(&s.k_empty[ks]);
            if (n == ui.npairs - 1) mma_commit(&s.q_empty);
          }
        } else {
          for (int n = 0; n < ui.npairs && ok; ++n) {
            const long gp = gp0 + n;
            const bool first = n == 0;
            const int vs = (int)(gp % kVStages);
            const int pb = (int)(gp & 1);  // P^T buffer
            if ((first && !mbar_wait(&s.o_empty, (active & 1) ^ 1, abort_flag)) ||
                !mbar_wait(&s.v_full[vs], (uint32_t)((gp / kVStages) & 1), abort_flag) ||
                !mbar_wait(&s.p_full[pb], (uint32_t)((gp >> 1) & 1), abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da0 = dv + (uint64_t)(vs * (kPairBytes >> 4));
            const uint64_t db0 = dp + (uint64_t)(pb * (kPBytes >> 4));
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys (2048 bytes of V^T and of P^T) per MMA
              mma_bf16(tmem + kColO, da0 + kk * (2048 >> 4), db0 + kk * (2048 >> 4), idesc_o,
                       (first && kk == 0) ? 0u : 1u);
            mma_commit(&s.p_empty[pb]);
            mma_commit(&s.v_empty[vs]);
          }
          if (ok) mma_commit(&s.o_full);
        }
        if (!ok) break;
        gp0 += ui.npairs;
        ++active;
      }
      if (!ok) fail(s, a.dev_status);
      // Every MMA issued must complete before TMEM is released.
      mma_commit(&s.drain);
      mbar_wait(&s.drain, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------- softmax + epilogue
    // kWGs warpgroups split the 64 query columns: warpgroup wg owns columns [kQW wg, kQW wg + kQW).
    // Within a warpgroup, warp sub-partition sp covers TMEM lanes [32 sp, 32 sp + 32).
    const int wg = (warp - 2) >> 2;
    const int sp = warp & 3;
    const int r = sp * 32 + lane;       // TMEM lane: key row of S^T, column d of O^T
    const int gt = ((warp - 2) & 3) * 32 + lane;  // 0..127 within the warpgroup
    const int bar_id = kSoftmaxBar + wg;
    const int q0 = wg * kQW;
    const uint32_t lane_base = tmem + ((uint32_t)(sp * 32) << 16);
    int active = 0;
    long gp0 = 0;
    bool reported = false;
    uint32_t sync_phase = 0;
    // All softmax warpgroups meet here; false if one never arrives (timeout / abort).
    auto rendezvous = [&]() -> bool {
      mbar_arrive(&s.wg_sync);
      const bool r_ok = mbar_wait(&s.wg_sync, sync_phase, abort_flag);
      sync_phase ^= 1u;
      return r_ok;
    };
    float lpart[kQW];
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const UnitInfo ui = unit_info(g, a, u);
      const long row0 = (long)ui.b * g.Lp + (long)ui.i * kTileElems;
      const int vci = s.vc[ui.i];
      const long ld = (long)g.heads * kD;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.o) + row0 * ld + (long)ui.h * kD;
      if (ui.npairs == 0) {
        // No kept key tile: this warpgroup's output rows are zero.
        for (int e = gt; e < kQW * kD / 8; e += kSoftmaxThreads) {
          const int rr = q0 + e / (kD / 8), c = e % (kD / 8);
          *reinterpret_cast<uint4*>(out + rr * ld + c * 8) = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      if (gt < kQW) {
        s.shift[q0 + gt] = -INFINITY;
        s.thr[q0 + gt] = -INFINITY;
        s.nsh[q0 + gt] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < kQW; ++q) lpart[q] = 0.f;
      named_bar(bar_id, kSoftmaxThreads);
      // Key tile of this thread's row for the first step (list entries are prefetched a step ahead).
      int raw_next = ((r >> 6) < ui.cnt) ? ui.list[r >> 6] : kAbsent;
      bool failed = false;
      for (int n = 0; n < ui.npairs; ++n) {
        const long gp = gp0 + n;
        const int sb = (int)(gp % kSBufs);  // S^T buffer
        const int pb = (int)(gp & 1);       // P^T buffer
        const uint32_t ph = (uint32_t)((gp >> 1) & 1);
        const int raw = raw_next;
        const int e_next = 2 * (n + 1) + (r >> 6);
        raw_next = (e_next < ui.cnt) ? ui.list[e_next] : kAbsent;
        // S^T of this step, and P^T buffer sb free again (its PV MMAs of step gp - 2 complete).
        bool ok = mbar_wait(&s.s_full[sb], (uint32_t)((gp / kSBufs) & 1), abort_flag);
        ok = ok && mbar_wait(&s.p_empty[pb], ph ^ 1, abort_flag);
        tc_fence_after();
        float x[kQW];
        {
          uint32_t v[kQW];
          tmem_ld<kQW>(lane_base + kColS + sb * 64 + q0, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < kQW; ++q) x[q] = __uint_as_float(v[q]);
        }
        tc_fence_before();
        mbar_arrive(&s.s_empty[sb]);
        const bool in_range = raw >= 0 && raw < g.nT;
        const bool valid = in_range && (r & 63) < s.vc[in_range ? raw : 0];
        if (!reported && raw != kAbsent && !in_range) {
          report(a.dev_status, T3D_DEV_INDEX_RANGE);
          reported = true;
        }
        if (!valid) {
#pragma unroll
          for (int q = 0; q < kQW; ++q) x[q] = -INFINITY;
        }
        // x holds raw logits; the softmax scale (> 0) is folded into the thresholds and the exp2.
        bool over = false;
#pragma unroll
        for (int q = 0; q < kQW; q += 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(&s.thr[q0 + q]);
          over |= (x[q] > t4.x) | (x[q + 1] > t4.y) | (x[q + 2] > t4.z) | (x[q + 3] > t4.w);
        }
        const bool bad = !ok || *abort_flag;
        if (named_bar_or(bar_id, kSoftmaxThreads, over || bad)) {
          if (named_bar_or(bar_id, kSoftmaxThreads, bad)) { failed = true; break; }
          // Slow step: raise the shifts to the running maxima and rescale what was accumulated.
#pragma unroll
          for (int q = 0; q < kQW; ++q) {
            const float mq = redux_max(x[q]);
            if (lane == q) s.red[sp][q0 + q] = mq;
          }
          named_bar(bar_id, kSoftmaxThreads);
          if (gt < kQW) {
            const int qq = q0 + gt;
            const float old = s.shift[qq];
            float mx = fmaxf(fmaxf(s.red[0][qq], s.red[1][qq]), fmaxf(s.red[2][qq], s.red[3][qq]));
            mx = fmaxf(mx * sl2, old);
            s.alpha[qq] = (old == -INFINITY) ? (mx == -INFINITY ? 1.f : 0.f) : ex2(old - mx);
            s.shift[qq] = mx;
            s.thr[qq] = mx == -INFINITY ? -INFINITY : (mx + kShiftSlack) / sl2;
            s.nsh[qq] = mx == -INFINITY ? 0.f : -mx;
          }
          named_bar(bar_id, kSoftmaxThreads);
          bool wok = true;
          if (n > 0) {
            // O^T holds the contributions of earlier steps: rescale column q by alpha[q] once the
            // last PV MMA has landed.
            wok = mbar_wait(&s.p_empty[(gp - 1) & 1], ((gp - 1) >> 1) & 1, abort_flag);
            tc_fence_after();
            uint32_t v[kQW];
            tmem_ld<kQW>(lane_base + kColO + q0, v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < kQW; ++q)
              v[q] = __float_as_uint(__uint_as_float(v[q]) * s.alpha[q0 + q]);
            tmem_st<kQW>(lane_base + kColO + q0, v);
            tmem_wait_st();
            tc_fence_before();
          }
#pragma unroll
          for (int q = 0; q < kQW; q += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(&s.alpha[q0 + q]);
            lpart[q] *= a4.x; lpart[q + 1] *= a4.y; lpart[q + 2] *= a4.z; lpart[q + 3] *= a4.w;
          }
          if (named_bar_or(bar_id, kSoftmaxThreads, !wok)) { failed = true; break; }
        }
        // P = exp2(x - shift), running sums, bf16 into this row of P^T (MN-major, 128B swizzle:
        // 16-byte chunk c of row r lives at chunk c ^ (r & 7); this warpgroup owns kQW / 8 chunks).
        uint8_t* prow = s.p[pb] + r * 128;
#pragma unroll
        for (int c = 0; c < kQW / 8; ++c) {
          uint32_t w[4];
          const float4 n0 = *reinterpret_cast<const float4*>(&s.nsh[q0 + c * 8]);
          const float4 n1 = *reinterpret_cast<const float4*>(&s.nsh[q0 + c * 8 + 4]);
          const float nsh[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = c * 8 + 2 * e;
            const float p0 = ex2(fmaf(x[q], sl2, nsh[2 * e]));
            const float p1 = ex2(fmaf(x[q + 1], sl2, nsh[2 * e + 1]));
            lpart[q] += p0;
            lpart[q + 1] += p1;
            __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
            w[e] = *reinterpret_cast<uint32_t*>(&pk);
          }
          const int chunk = (kQW / 8) * wg + c;
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async();
        mbar_arrive(&s.p_full[pb]);
      }
      if (failed) break;
      // ---- epilogue: denominators (reduce the 128 per-key partial sums of each query)
#pragma unroll
      for (int q = 0; q < kQW; ++q) {
        float v = lpart[q];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == q) s.red[sp][q0 + q] = v;
      }
      const bool ook = mbar_wait(&s.o_full, active & 1, abort_flag);
      named_bar(bar_id, kSoftmaxThreads);
      if (gt < kQW) {
        const int qq = q0 + gt;
        s.lsum[qq] = s.red[0][qq] + s.red[1][qq] + s.red[2][qq] + s.red[3][qq];
      }
      if (named_bar_or(bar_id, kSoftmaxThreads, !ook || *abort_flag)) break;
      tc_fence_after();
      // O^T row r (= column d of O) for this warpgroup's queries: divide by the denominators and
      // stage O as [64 q][128 d] bf16 in the P^T buffer 0 (idle here: every PV MMA of the unit is
      // complete and the next unit's first P^T write waits for the closing rendezvous below).
      __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(s.p[0]);
      {
        uint32_t v[kQW];
        tmem_ld<kQW>(lane_base + kColO + q0, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < kQW; ++q) {
          const int qq = q0 + q;
          const float l = s.lsum[qq];
          const float val = l > 0.f ? __uint_as_float(v[q]) / l : 0.f;
          stage[qq * kD + r] = __float2bfloat16_rn(val);
        }
      }
      tc_fence_before();
      mbar_arrive(&s.o_empty);
      named_bar(bar_id, kSoftmaxThreads);
      const long blk = ((long)ui.b * g.heads + ui.h) * g.nT + ui.i;
      const uint8_t* keep = a.keep ? a.keep + blk * kTileElems : nullptr;
      const uint8_t* srcr = a.src_row ? a.src_row + blk * kTileElems : nullptr;
      if (keep != nullptr) {  // source rows span every warpgroup's staging rows
        if (named_bar_or(bar_id, kSoftmaxThreads, !rendezvous())) break;
      }
      for (int e = gt; e < kQW * kD / 8; e += kSoftmaxThreads) {
        const int rr = q0 + e / (kD / 8), c = e % (kD / 8);
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (rr < vci) {
          int sr = rr;
          if (keep != nullptr && !keep[rr]) {
            sr = srcr[rr];
            if (sr >= kTileElems) sr = rr;
          }
          val = *reinterpret_cast<const uint4*>(stage + sr * kD + c * 8);
        }
        *reinterpret_cast<uint4*>(out + rr * ld + c * 8) = val;
      }
      // The staging buffer is free for the next unit once every warpgroup is done with it.
      if (named_bar_or(bar_id, kSoftmaxThreads, !rendezvous())) break;
      gp0 += ui.npairs;
      ++active;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3D map over a [B * Lp, heads, D] bf16 tensor; box = 64 rows x 1 head x 64 elements, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, const Geo& g) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.heads, (cuuint64_t)g.B * g.Lp};
  const cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.heads * g.D * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

cudaError_t launch_attn_sm100(const Geo& g, const AttnArgs& a, cudaStream_t s) {
  Maps maps;
  if (!make_map(&maps.q, a.q, g) || !make_map(&maps.k, a.k, g) || !make_map(&maps.v, a.v, g))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemLayout) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int units = g.B * g.heads * g.nT;
  const int grid = units < sm_count() ? units : sm_count();
  const float sl2 = a.scale * 1.4426950408889634f;
  attn_sm100_kernel<<<grid, kThreads, smem, s>>>(maps, g, a, sl2);
  return cudaGetLastError();
}

}  // namespace t3d
