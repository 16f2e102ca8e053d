// Backward pass of the fine stage on the sm_100a tensor cores: the gradients dQ, dK, dV of the
// block-sparse softmax attention for a given output gradient dO, over the same kept (query tile,
// key tile) pairs as the forward.
//
// FastVideo API docs, video_sparse_attn_h3 page: tile() gives a forward that tracks gradients its
// own buffer, and the sm100a route is taken only without gradients (training keeps another
// route); the pages print no backward formulas, so what is computed is the derivative of the
// forward's definition (bsa_attn page, BSAAttentionImpl.forward). For a valid, attending query
// row r of query tile i, with keys c over the valid rows of its kept key tiles:
//     p_rc = exp(scale q_r.k_c - lse_r)           (lse_r: the forward's log-sum-exp of row r)
//     dV_c += p_rc dO_r        dP_rc = dO_r.v_c        dS_rc = p_rc (dP_rc - delta_r)
//     dQ_r  = scale sum_c dS_rc k_c                    dK_c += scale dS_rc q_r
// with delta_r = sum_c p_rc dP_rc = dO_r.o_r. No gradient flows through the selection. A query
// row pruned by BSA copies the output of its source row, so its dO is added to the source row's
// and its own q gets no gradient; pad query rows and pad keys get none either.
//
// Four steps:
//   bwd_prep_kernel   per (batch, head, query tile): the effective output gradient dOe (pruned
//                     rows' dO added to their sources, pruned and pad rows zero) as bf16, and
//                     delta_r = dOe_r . o_r in fp32;
//   key-to-query lists: the kept pairs as a 0/1 map [key tile][query tile] (csc_scatter_kernel),
//                     then per key tile the ascending list of query tiles that kept it
//                     (csc_build_kernel), so the dK/dV kernel's sums run in a fixed order;
//   bwd_dq_kernel     per query tile (M = 64 rows) over its kept key-tile pairs (N = 128 keys):
//                     S = Q.K^T and dP = dOe.V^T into TMEM, the softmax warps form dS as bf16 in
//                     TMEM, then dQ += dS.K (A = dS from TMEM, B = the K pair, MN-major);
//   bwd_dkdv_kernel   per key tile (M = 64 keys) over the query tiles of its list (N = 64):
//                     S^T = K.Q^T and dP^T = V.dOe^T into one of two TMEM buffers, the softmax
//                     warps write P^T and dS^T as bf16 over them, then dV += P^T.dOe and
//                     dK += dS^T.Q; the next step's products go to the other buffer meanwhile.
// Both contraction kernels are persistent (one CTA per SM, units in static round robin) with one
// TMA producer thread, MMA issuer threads (dQ: S, dP and dQ one each; dK/dV: the step's two
// products, the two accumulations) and one softmax warpgroup; every wait is bounded as
// in the forward kernel (on a timeout: T3D_DEV_TIMEOUT, drain, free TMEM, return).
#include "kernels.h"
#include "sm100.cuh"

namespace t3d {
namespace {

using namespace sm100;

constexpr uint32_t kTileBytes = 64 * 128;  // 64 rows x 128 B: one 64-element column block
constexpr int kBwdThreads = 256;  // warp 0 producer, warps 1-3 MMA issuers, warps 4..7 softmax
constexpr int kTeardown = 1;               // named barrier of all threads before TMEM is freed
constexpr float kLog2e = 1.4426950408889634f;

struct BwdMaps {
  CUtensorMap q, k, v, dout;
};

__device__ __forceinline__ void bwd_fail(int* abort, int32_t* status) {
  *reinterpret_cast<volatile int*>(abort) = 1;
  report(status, T3D_DEV_TIMEOUT);
}

// ------------------------------------------------------------------------------------ prep
// Grid (nT, heads, B), 256 threads. A tile without pruned rows (the common case) goes through
// registers in 16-byte chunks: dOe = dO on valid rows, zero on pad rows, and delta from the
// chunk's eight products summed over the row's chunks by shuffles. A tile with pruned rows
// accumulates rows in fp32 in shared memory, one column per thread with rows in order, so the
// sums are deterministic.
template <int kD>
__global__ void __launch_bounds__(256) bwd_prep_kernel(Geo g, const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const uint8_t* __restrict__ keep,
                                                       const uint8_t* __restrict__ src_row,
                                                       __nv_bfloat16* __restrict__ dout_eff,
                                                       float* __restrict__ delta) {
  constexpr int kChunks = kD / 8;             // 16-byte chunks of a row
  constexpr int kRowsPerPass = 256 / kChunks;  // rows one pass of the block covers
  __shared__ float acc[kTileElems][kD + 1];
  __shared__ int target[kTileElems];  // row whose gradient a row's dO adds to (-1: none)
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vc = tile_valid_count(g, i);
  const long ld = (long)g.heads_total * kD;
  const long base = ((long)b * g.Lp + (long)i * kTileElems) * ld + (long)(g.head0 + h) * kD;
  const long blk = ((long)b * g.heads + h) * g.nT + i;
  bool moved = false;  // this row's dO goes to another row
  if (tid < kTileElems) {
    int t = tid < vc ? tid : -1;
    if (t >= 0 && keep != nullptr && keep[blk * kTileElems + tid] == 0) {
      const int sr = src_row[blk * kTileElems + tid];
      t = sr < kTileElems ? sr : tid;
    }
    target[tid] = t;
    moved = t >= 0 && t != tid;
  }
  if (!__syncthreads_or(moved)) {
    const int c = tid % kChunks, r0 = tid / kChunks;
    uint4 dv[kTileElems / kRowsPerPass], ov[kTileElems / kRowsPerPass];
#pragma unroll
    for (int p = 0; p < kTileElems / kRowsPerPass; ++p) {  // every load in flight first
      const long at = base + (long)(r0 + p * kRowsPerPass) * ld + 8 * c;
      dv[p] = *reinterpret_cast<const uint4*>(dout + at);
      ov[p] = *reinterpret_cast<const uint4*>(o + at);
    }
#pragma unroll
    for (int p = 0; p < kTileElems / kRowsPerPass; ++p) {
      const int r = r0 + p * kRowsPerPass;
      if (r >= vc) dv[p] = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(dout_eff + base + (long)r * ld + 8 * c) = dv[p];
      const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&dv[p]);
      const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&ov[p]);
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 xf = __bfloat1622float2(x[e]), yf = __bfloat1622float2(y[e]);
        sum = fmaf(xf.x, yf.x, sum);
        sum = fmaf(xf.y, yf.y, sum);
      }
#pragma unroll
      for (int off = kChunks / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (c == 0) delta[blk * kTileElems + r] = sum;
    }
    return;
  }
  for (int e = tid; e < kTileElems * kD; e += 256) acc[e / kD][e % kD] = 0.f;
  __syncthreads();
  if (tid < kD) {  // one column per thread, rows in order
    for (int r = 0; r < kTileElems; ++r) {
      const int t = target[r];
      if (t >= 0) acc[t][tid] += __bfloat162float(dout[base + (long)r * ld + tid]);
    }
  }
  __syncthreads();
  // dOe as bf16; delta_r = dOe_r . o_r over the rounded dOe (the operand the MMAs see).
  for (int r = warp; r < kTileElems; r += 8) {
    float s = 0.f;
    for (int d = lane; d < kD; d += 32) {
      const __nv_bfloat16 x = __float2bfloat16_rn(acc[r][d]);
      dout_eff[base + (long)r * ld + d] = x;
      s = fmaf(__bfloat162float(x), __bfloat162float(o[base + (long)r * ld + d]), s);
    }
    s = warp_sum(s);
    if (lane == 0) delta[blk * kTileElems + r] = s;
  }
}

// ------------------------------------------------------------------------------ lists
// One thread per list entry: map[bh][j][i] = 1 for every kept pair (i, j).
__global__ void csc_scatter_kernel(Geo g, const int32_t* __restrict__ kv_idx,
                                   const int32_t* __restrict__ kv_cnt, int kmax,
                                   uint8_t* __restrict__ map) {
  const long total = (long)g.B * g.heads * g.nT * kmax;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long)gridDim.x * blockDim.x) {
    const long row = e / kmax;  // (bh, i)
    const int slot = (int)(e - row * kmax);
    int c = kv_cnt[row];
    c = c < 0 ? 0 : (c > kmax ? kmax : c);
    if (slot >= c) continue;
    const int j = kv_idx[e];
    if (j < 0 || j >= g.nT) continue;
    const long bh = row / g.nT;
    const int i = (int)(row - bh * g.nT);
    map[(bh * g.nT + j) * g.nT + i] = 1;
  }
}

// One warp per (bh, key tile j): the query tiles i with map[bh][j][i] set, ascending.
__global__ void csc_build_kernel(Geo g, const uint8_t* __restrict__ map, int32_t* __restrict__ q_idx,
                                 int32_t* __restrict__ q_cnt) {
  const int lane = threadIdx.x & 31;
  const long rows = (long)g.B * g.heads * g.nT;
  const unsigned lt = lanemask_lt();
  for (long r = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += (long)gridDim.x * (blockDim.x >> 5)) {
    const uint8_t* m = map + r * g.nT;
    int32_t* out = q_idx + r * g.nT;
    int cnt = 0;
    for (int i0 = 0; i0 < g.nT; i0 += 32) {
      const int i = i0 + lane;
      const bool on = i < g.nT && m[i] != 0;
      const unsigned bits = __ballot_sync(0xffffffffu, on);
      if (on) out[cnt + __popc(bits & lt)] = i;
      cnt += __popc(bits);
    }
    if (lane == 0) q_cnt[r] = cnt;
  }
}

// ------------------------------------------------------------------------------ dQ
template <int kD>
struct DqCfg {
  static constexpr int kHalves = kD / 64;
  static constexpr uint32_t kPair = kHalves * 2 * kTileBytes;  // two key tiles, every column block
  static constexpr uint32_t kOne = kHalves * kTileBytes;       // one 64-row tile
  static constexpr int kStages = 2;
};

template <int kD>
struct alignas(1024) DqSmem {
  using C = DqCfg<kD>;
  uint8_t k[C::kStages][C::kPair];
  uint8_t v[C::kStages][C::kPair];
  uint8_t q[C::kOne];
  uint8_t dout[C::kOne];
  uint64_t kv_full[C::kStages], kv_empty[C::kStages];
  uint64_t q_full, q_empty;    // the unit's Q and dOe tiles landed / read by its last S and dP
  uint64_t s_full[2], s_empty[2];  // S ([0]) and dP ([1]) of a step in TMEM / read by the softmax
  uint64_t ds_full, ds_empty;  // dS of a step in TMEM / read by its dQ MMAs
  uint64_t dq_full, dq_empty;  // a unit's dQ complete / read by the epilogue
  uint64_t drain[3];           // every MMA of the S, the dQ, the dP issuer complete
  uint8_t vc[kMaxTiles];
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t kDqColS = 0, kDqColDP = 128, kDqColDQ = 256, kDqColDS = 384;

struct BwdArgs {
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  int kmax;
  const int32_t* q_idx;  // key-to-query lists [B, heads, nT, nT] and counts [B, heads, nT]
  const int32_t* q_cnt;
  const uint8_t* keep;
  const float* lse;    // [B, heads, Lp], natural log
  const float* delta;  // [B, heads, Lp]
  void* dq;
  void* dk;
  void* dv;
  float scale;
  int32_t* dev_status;
  long long wait_cycles;
};

template <int kD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ BwdMaps maps, Geo g, BwdArgs a) {
  using C = DqCfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  DqSmem<kD>& s = *reinterpret_cast<DqSmem<kD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_units = g.B * g.heads * g.nT;
  const long long lim = a.wait_cycles;
  volatile int* abort_flag = &s.abort;
  const float sl2 = a.scale * kLog2e;
  if (threadIdx.x == 0) {
    for (int t = 0; t < C::kStages; ++t) {
      mbar_init(&s.kv_full[t], 1);
      mbar_init(&s.kv_empty[t], 1);
    }
    mbar_init(&s.q_full, 1);
    mbar_init(&s.q_empty, 2);  // one commit from each of the S and dP issuers
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.s_empty[t], 128);
    }
    mbar_init(&s.ds_full, 128);
    mbar_init(&s.ds_empty, 1);
    mbar_init(&s.dq_full, 1);
    mbar_init(&s.dq_empty, 128);
    for (int t = 0; t < 3; ++t) mbar_init(&s.drain[t], 1);
    s.abort = 0;
    fence_mbar_init();
  }
  for (int t = threadIdx.x; t < g.nT; t += kBwdThreads) s.vc[t] = (uint8_t)tile_valid_count(g, t);
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  auto unit_pairs = [&](int u, int& cnt, const int32_t*& list) {
    int c = a.kv_cnt[u];
    c = c < 0 ? 0 : (c > a.kmax ? a.kmax : c);
    cnt = c;
    list = a.kv_idx + (long)u * a.kmax;
    return (c + 1) >> 1;
  };
  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      long gp = 0;
      int nq = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        int cnt;
        const int32_t* list;
        const int np = unit_pairs(u, cnt, list);
        if (np == 0) continue;
        const int i = u % g.nT, bh = u / g.nT, h = bh % g.heads, b = bh / g.heads;
        if (!mbar_wait(&s.q_empty, (uint32_t)((nq & 1) ^ 1), abort_flag, lim)) { ok = false; break; }
        mbar_expect_tx(&s.q_full, 2 * C::kOne);
        for (int hh = 0; hh < C::kHalves; ++hh) {
          tma_load_3d(s.q + hh * kTileBytes, &maps.q, &s.q_full, 64 * hh, g.head0 + h,
                      b * g.Lp + i * kTileElems);
          tma_load_3d(s.dout + hh * kTileBytes, &maps.dout, &s.q_full, 64 * hh, g.head0 + h,
                      b * g.Lp + i * kTileElems);
        }
        ++nq;
        for (int n = 0; n < np; ++n, ++gp) {
          const int st = (int)(gp % C::kStages);
          if (!mbar_wait(&s.kv_empty[st], (uint32_t)(((gp / C::kStages) & 1) ^ 1), abort_flag,
                         lim)) {
            ok = false;
            break;
          }
          int ja = 2 * n < cnt ? list[2 * n] : -1, jb = 2 * n + 1 < cnt ? list[2 * n + 1] : -1;
          if (ja < 0 || ja >= g.nT) ja = 0;  // masked in the softmax
          if (jb < 0 || jb >= g.nT) jb = ja;
          mbar_expect_tx(&s.kv_full[st], 2 * C::kPair);
          for (int hh = 0; hh < C::kHalves; ++hh) {
            uint8_t* kd = s.k[st] + hh * 2 * kTileBytes;
            uint8_t* vd = s.v[st] + hh * 2 * kTileBytes;
            tma_load_3d(kd, &maps.k, &s.kv_full[st], 64 * hh, g.head0 + h, b * g.Lp + ja * kTileElems);
            tma_load_3d(kd + kTileBytes, &maps.k, &s.kv_full[st], 64 * hh, g.head0 + h,
                        b * g.Lp + jb * kTileElems);
            tma_load_3d(vd, &maps.v, &s.kv_full[st], 64 * hh, g.head0 + h, b * g.Lp + ja * kTileElems);
            tma_load_3d(vd + kTileBytes, &maps.v, &s.kv_full[st], 64 * hh, g.head0 + h,
                        b * g.Lp + jb * kTileElems);
          }
        }
      }
      if (!ok) bwd_fail(&s.abort, a.dev_status);
      for (long t = gp - C::kStages; t < gp; ++t)  // drain: the last loads must land
        if (t >= 0) mbar_wait(&s.kv_full[t % C::kStages], (uint32_t)((t / C::kStages) & 1), nullptr);
      if (nq > 0) mbar_wait(&s.q_full, (uint32_t)((nq - 1) & 1), nullptr);
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------- S issuer (warp 1), dP issuer (3)
    // S, dP and dQ have one issuing thread each (as in the forward kernel): an mbarrier wait in
    // the thread that issues MMAs lets its queued MMAs drain first, and the other threads' queued
    // MMAs keep the pipe busy meanwhile. S and dP complete separately, so the softmax forms P
    // while dP is computed, and each product's buffer is free once the softmax has read it.
    if (lane == 0) {
      const int which = warp == 1 ? 0 : 1;  // 0: S = Q . K_pair^T, 1: dP = dOe . V_pair^T
      constexpr uint32_t idesc_s = idesc_bf16(64, 128, false, false);
      const uint64_t da = sdesc_sw128(smem_u32(which ? s.dout : s.q), 16, 1024);
      const uint64_t db = sdesc_sw128(smem_u32(which ? s.v[0] : s.k[0]), 16, 1024);
      const uint32_t d_acc = tmem + (which ? kDqColDP : kDqColS);
      long gp = 0;
      int active = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        int cnt;
        const int32_t* list;
        const int np = unit_pairs(u, cnt, list);
        if (np == 0) continue;
        if (!mbar_wait(&s.q_full, (uint32_t)(active & 1), abort_flag, lim)) { ok = false; break; }
        for (int n = 0; n < np; ++n, ++gp) {
          const int st = (int)(gp % C::kStages);
          if (!mbar_wait(&s.kv_full[st], (uint32_t)((gp / C::kStages) & 1), abort_flag, lim) ||
              !mbar_wait(&s.s_empty[which], (uint32_t)((gp & 1) ^ 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t b0 = db + (uint64_t)(st * (C::kPair >> 4));
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const int hh = kk >> 2, sub = kk & 3;
            const uint64_t ao = (uint64_t)((hh * kTileBytes + sub * 32) >> 4);
            const uint64_t bo = (uint64_t)((hh * 2 * kTileBytes + sub * 32) >> 4);
            mma_bf16(d_acc, da + ao, b0 + bo, idesc_s, kk ? 1u : 0u);
          }
          mma_commit(&s.s_full[which]);
          if (n == np - 1) mma_commit(&s.q_empty);
        }
        ++active;
      }
      if (!ok) bwd_fail(&s.abort, a.dev_status);
      mma_commit(&s.drain[which ? 2 : 0]);
      mbar_wait(&s.drain[which ? 2 : 0], 0, nullptr);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------- dQ issuer
    if (lane == 0) {
      constexpr uint32_t idesc_q = idesc_bf16(64, kD, false, true);
      const uint64_t dkm = sdesc_sw128(smem_u32(s.k[0]), 2 * kTileBytes, 1024);  // K pair, MN-major
      long gp = 0;
      int active = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        int cnt;
        const int32_t* list;
        const int np = unit_pairs(u, cnt, list);
        if (np == 0) continue;
        for (int n = 0; n < np; ++n, ++gp) {
          // dQ += dS(step) . K_pair(step); the unit's first one overwrites dQ once the epilogue
          // has read it. The stage's K and V are free once this completes (its S and dP, which
          // the softmax read before writing dS, completed earlier).
          const int st = (int)(gp % C::kStages);
          if ((n == 0 && !mbar_wait(&s.dq_empty, (uint32_t)((active & 1) ^ 1), abort_flag, lim)) ||
              !mbar_wait(&s.ds_full, (uint32_t)(gp & 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t b0 = dkm + (uint64_t)(st * (C::kPair >> 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 keys per MMA
            mma_bf16_ts(tmem + kDqColDQ, tmem + kDqColDS + 8 * kk, b0 + kk * (2048 >> 4), idesc_q,
                        (n == 0 && kk == 0) ? 0u : 1u);
          mma_commit(&s.ds_empty);
          mma_commit(&s.kv_empty[st]);
        }
        if (ok) mma_commit(&s.dq_full);
        ++active;
      }
      if (!ok) bwd_fail(&s.abort, a.dev_status);
      mma_commit(&s.drain[1]);
      mbar_wait(&s.drain[1], 0, nullptr);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax and epilogue
    const int sp = warp & 3;
    const int t0 = lane & 3, q4 = lane >> 2;
    const int r0 = 16 * sp + q4, r1 = r0 + 8;
    const uint32_t lane_base = tmem + ((uint32_t)(sp * 32) << 16);
    const long ld = (long)g.heads_total * kD;
    long gp = 0;
    int active = 0;
    bool failed = false;
    auto give_up = [&]() {
      failed = true;
      *abort_flag = 1;
    };
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      int cnt;
      const int32_t* list;
      const int np = unit_pairs(u, cnt, list);
      const int i = u % g.nT, bh = u / g.nT, h = bh % g.heads, b = bh / g.heads;
      const int vci = s.vc[i];
      __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(a.dq) +
                          ((long)b * g.Lp + (long)i * kTileElems) * ld + (long)(g.head0 + h) * kD;
      const long rowbase = (long)u * kTileElems;  // [B, heads, Lp] index of the tile's row 0
      if (np == 0) {
        for (int c = 2 * t0; c < kD; c += 8) {
          *reinterpret_cast<uint32_t*>(dq + r0 * ld + c) = 0u;
          *reinterpret_cast<uint32_t*>(dq + r1 * ld + c) = 0u;
        }
        continue;
      }
      const float lse0 = a.lse[rowbase + r0] * kLog2e, lse1 = a.lse[rowbase + r1] * kLog2e;
      const float dl0 = a.delta[rowbase + r0], dl1 = a.delta[rowbase + r1];
      // key tiles of the next step, loaded one step ahead
      int na = 0 < cnt ? list[0] : -1, nb = 1 < cnt ? list[1] : -1;
      for (int n = 0; n < np; ++n, ++gp) {
        const int ja = na, jb = nb;
        na = 2 * n + 2 < cnt ? list[2 * n + 2] : -1;
        nb = 2 * n + 3 < cnt ? list[2 * n + 3] : -1;
        const int ca = (ja >= 0 && ja < g.nT) ? s.vc[ja] : 0;
        const int cb = (jb >= 0 && jb < g.nT) ? s.vc[jb] : 0;
        // P from S while dP is still being computed
        if (!mbar_wait(&s.s_full[0], (uint32_t)(gp & 1), abort_flag, lim)) give_up();
        tc_fence_after();
        uint32_t sv[64], pv[64];
        tmem_ld_16x256b_x16(lane_base + kDqColS, sv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s.s_empty[0]);
        float pr[64];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = 8 * j + 2 * t0 + (e & 1);
            const bool valid = key < 64 ? key < ca : key - 64 < cb;
            const float lse = e < 2 ? lse0 : lse1;
            pr[4 * j + e] = valid ? ex2(fmaf(__uint_as_float(sv[4 * j + e]), sl2, -lse)) : 0.f;
          }
        }
        if (!mbar_wait(&s.s_full[1], (uint32_t)(gp & 1), abort_flag, lim)) give_up();
        tc_fence_after();
        tmem_ld_16x256b_x16(lane_base + kDqColDP, pv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s.s_empty[1]);
        // dS = P (dP - delta) as bf16 pairs, in the layout of the forward's P: keys 8j + 2 t0 and
        // + 1 to column 4j + t0 (tcgen05.st 16x128b), two stores of 32 columns.
        uint32_t dsw[2][16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float d[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float dl = e < 2 ? dl0 : dl1;
            d[e] = pr[4 * j + e] * (__uint_as_float(pv[4 * j + e]) - dl);
          }
          const __nv_bfloat162 q0 = __floats2bfloat162_rn(d[0], d[1]);
          const __nv_bfloat162 q1 = __floats2bfloat162_rn(d[2], d[3]);
          dsw[j >> 3][2 * (j & 7)] = *reinterpret_cast<const uint32_t*>(&q0);
          dsw[j >> 3][2 * (j & 7) + 1] = *reinterpret_cast<const uint32_t*>(&q1);
        }
        if (!mbar_wait(&s.ds_empty, (uint32_t)((gp & 1) ^ 1), abort_flag, lim)) give_up();
        tc_fence_after();
        tmem_st_16x128b_x8(lane_base + kDqColDS, dsw[0]);
        tmem_st_16x128b_x8(lane_base + kDqColDS + 32, dsw[1]);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&s.ds_full);
      }
      // ---- epilogue: dQ * scale for the attending rows, zero for pad and pruned rows
      if (!mbar_wait(&s.dq_full, (uint32_t)(active & 1), abort_flag, lim)) give_up();
      tc_fence_after();
      failed = __any_sync(0xffffffffu, failed);
      if (!failed) {
        const int rown = 16 * sp + (lane & 15);
        const bool live = rown < vci && (a.keep == nullptr || a.keep[rowbase + rown] != 0);
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kDqColDQ + 32 * c, o);
          tmem_wait_ld();
          if (lane < 16) {
            uint4 w4[4];
            uint32_t* w = reinterpret_cast<uint32_t*>(w4);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const __nv_bfloat162 y = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * a.scale,
                                                             __uint_as_float(o[2 * e + 1]) * a.scale);
              w[e] = live ? *reinterpret_cast<const uint32_t*>(&y) : 0u;
            }
            uint4* dst = reinterpret_cast<uint4*>(dq + rown * ld + 32 * c);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) dst[k4] = w4[k4];
          }
        }
        tc_fence_before();
        mbar_arrive(&s.dq_empty);
      }
      ++active;
    }
    if (failed && lane == 0) bwd_fail(&s.abort, a.dev_status);
  }
  tc_fence_before();
  named_bar(kTeardown, kBwdThreads);
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ dK, dV
template <int kD>
struct KvCfg {
  static constexpr int kHalves = kD / 64;
  static constexpr uint32_t kOne = kHalves * kTileBytes;  // one 64-row tile
  static constexpr int kStages = 3;
};

template <int kD>
struct alignas(1024) KvSmem {
  using C = KvCfg<kD>;
  uint8_t q[C::kStages][C::kOne];
  uint8_t dout[C::kStages][C::kOne];
  uint8_t k[C::kOne];
  uint8_t v[C::kOne];
  uint64_t qd_full[C::kStages], qd_empty[C::kStages];
  uint64_t kv_full, kv_empty;  // the unit's K and V tiles landed / no longer read
  uint64_t s_full[2];    // S^T and dP^T of a step in TMEM buffer b (steps alternate buffers)
  uint64_t p_full[2];    // P^T and dS^T of that step written over them by the softmax
  uint64_t buf_free[2];  // the dV / dK MMAs that read buffer b have completed
  uint64_t acc_full, acc_empty;  // a unit's dK and dV complete / read by the epilogue
  uint64_t drain[2];             // every MMA of the S / dP issuer, of the dK / dV issuer, complete
  uint8_t vc[kMaxTiles];
  uint32_t tmem_base;
  int abort;
};

// TMEM columns: S^T of buffers 0 / 1 at 0 / 64, dP^T at 128 / 192 (fp32, 64 query columns each);
// P^T and dS^T (bf16 pairs, 32 columns) are written over the first half of their step's S^T and
// dP^T once the softmax has read them; dV and dK accumulate at 256 and 384.
constexpr uint32_t kKvColS = 0, kKvColDP = 128, kKvBuf = 64, kKvColDV = 256, kKvColDK = 384;

template <int kD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ BwdMaps maps, Geo g, BwdArgs a) {
  using C = KvCfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  KvSmem<kD>& s = *reinterpret_cast<KvSmem<kD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_units = g.B * g.heads * g.nT;
  const long long lim = a.wait_cycles;
  volatile int* abort_flag = &s.abort;
  const float sl2 = a.scale * kLog2e;
  if (threadIdx.x == 0) {
    for (int t = 0; t < C::kStages; ++t) {
      mbar_init(&s.qd_full[t], 1);
      mbar_init(&s.qd_empty[t], 1);
    }
    mbar_init(&s.kv_full, 1);
    mbar_init(&s.kv_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.p_full[t], 128);
      mbar_init(&s.buf_free[t], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.acc_empty, 128);
    mbar_init(&s.drain[0], 1);
    mbar_init(&s.drain[1], 1);
    s.abort = 0;
    fence_mbar_init();
  }
  for (int t = threadIdx.x; t < g.nT; t += kBwdThreads) s.vc[t] = (uint8_t)tile_valid_count(g, t);
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  auto unit_list = [&](int u, const int32_t*& list) {
    int c = a.q_cnt[u];
    c = c < 0 ? 0 : (c > g.nT ? g.nT : c);
    list = a.q_idx + (long)u * g.nT;
    return c;
  };
  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      long gs = 0;
      int nk = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const int32_t* list;
        const int cnt = unit_list(u, list);
        if (cnt == 0) continue;
        const int j = u % g.nT, bh = u / g.nT, h = bh % g.heads, b = bh / g.heads;
        if (!mbar_wait(&s.kv_empty, (uint32_t)((nk & 1) ^ 1), abort_flag, lim)) { ok = false; break; }
        mbar_expect_tx(&s.kv_full, 2 * C::kOne);
        for (int hh = 0; hh < C::kHalves; ++hh) {
          tma_load_3d(s.k + hh * kTileBytes, &maps.k, &s.kv_full, 64 * hh, g.head0 + h,
                      b * g.Lp + j * kTileElems);
          tma_load_3d(s.v + hh * kTileBytes, &maps.v, &s.kv_full, 64 * hh, g.head0 + h,
                      b * g.Lp + j * kTileElems);
        }
        ++nk;
        for (int n = 0; n < cnt; ++n, ++gs) {
          const int st = (int)(gs % C::kStages);
          if (!mbar_wait(&s.qd_empty[st], (uint32_t)(((gs / C::kStages) & 1) ^ 1), abort_flag,
                         lim)) {
            ok = false;
            break;
          }
          int i = list[n];
          if (i < 0 || i >= g.nT) i = 0;
          mbar_expect_tx(&s.qd_full[st], 2 * C::kOne);
          for (int hh = 0; hh < C::kHalves; ++hh) {
            tma_load_3d(s.q[st] + hh * kTileBytes, &maps.q, &s.qd_full[st], 64 * hh, g.head0 + h,
                        b * g.Lp + i * kTileElems);
            tma_load_3d(s.dout[st] + hh * kTileBytes, &maps.dout, &s.qd_full[st], 64 * hh,
                        g.head0 + h, b * g.Lp + i * kTileElems);
          }
        }
      }
      if (!ok) bwd_fail(&s.abort, a.dev_status);
      for (long t = gs - C::kStages; t < gs; ++t)
        if (t >= 0) mbar_wait(&s.qd_full[t % C::kStages], (uint32_t)((t / C::kStages) & 1), nullptr);
      if (nk > 0) mbar_wait(&s.kv_full, (uint32_t)((nk - 1) & 1), nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- S^T and dP^T issuer
    // As in the dQ kernel, the two products of a step and the two accumulations have one issuing
    // thread each.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(64, 64, false, false);
      const uint64_t dkd = sdesc_sw128(smem_u32(s.k), 16, 1024);
      const uint64_t dvd = sdesc_sw128(smem_u32(s.v), 16, 1024);
      const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0]), 16, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(s.dout[0]), 16, 1024);
      long gs = 0;
      int active = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const int32_t* list;
        const int cnt = unit_list(u, list);
        if (cnt == 0) continue;
        if (!mbar_wait(&s.kv_full, (uint32_t)(active & 1), abort_flag, lim)) { ok = false; break; }
        for (int n = 0; n < cnt; ++n, ++gs) {
          // Step gs uses TMEM buffer gs & 1, free once the dV / dK MMAs of step gs - 2 are done.
          const int st = (int)(gs % C::kStages);
          const int bf = (int)(gs & 1);
          if (!mbar_wait(&s.qd_full[st], (uint32_t)((gs / C::kStages) & 1), abort_flag, lim) ||
              !mbar_wait(&s.buf_free[bf], (uint32_t)(((gs >> 1) & 1) ^ 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qb = dq0 + (uint64_t)(st * (C::kOne >> 4));
          const uint64_t dob = ddo0 + (uint64_t)(st * (C::kOne >> 4));
          const uint32_t d_s = tmem + kKvColS + kKvBuf * bf, d_dp = tmem + kKvColDP + kKvBuf * bf;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const int hh = kk >> 2, sub = kk & 3;
            const uint64_t o = (uint64_t)((hh * kTileBytes + sub * 32) >> 4);
            mma_bf16(d_s, dkd + o, qb + o, idesc_s, kk ? 1u : 0u);
            mma_bf16(d_dp, dvd + o, dob + o, idesc_s, kk ? 1u : 0u);
          }
          mma_commit(&s.s_full[bf]);
        }
        if (ok) mma_commit(&s.kv_empty);  // only these MMAs read the unit's K and V
        ++active;
      }
      if (!ok) bwd_fail(&s.abort, a.dev_status);
      mma_commit(&s.drain[0]);
      mbar_wait(&s.drain[0], 0, nullptr);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------- dV and dK issuer
    if (lane == 0) {
      constexpr uint32_t idesc_acc = idesc_bf16(64, kD, false, true);
      const uint64_t dqm0 = sdesc_sw128(smem_u32(s.q[0]), kTileBytes, 1024);     // MN-major
      const uint64_t ddom0 = sdesc_sw128(smem_u32(s.dout[0]), kTileBytes, 1024);  // MN-major
      long gs = 0;
      int active = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const int32_t* list;
        const int cnt = unit_list(u, list);
        if (cnt == 0) continue;
        for (int n = 0; n < cnt; ++n, ++gs) {
          // dV += P^T(step) . dOe(step) and dK += dS^T(step) . Q(step); the unit's first ones
          // overwrite the accumulators once the epilogue has read them. The stage's Q and dOe are
          // free once these complete (the step's S^T and dP^T completed earlier).
          const int st = (int)(gs % C::kStages);
          const int bf = (int)(gs & 1);
          if ((n == 0 && !mbar_wait(&s.acc_empty, (uint32_t)((active & 1) ^ 1), abort_flag, lim)) ||
              !mbar_wait(&s.p_full[bf], (uint32_t)((gs >> 1) & 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bq = dqm0 + (uint64_t)(st * (C::kOne >> 4));
          const uint64_t bdo = ddom0 + (uint64_t)(st * (C::kOne >> 4));
          const uint32_t a_p = tmem + kKvColS + kKvBuf * bf, a_ds = tmem + kKvColDP + kKvBuf * bf;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 16 query rows per MMA
            const uint32_t accum = (n == 0 && kk == 0) ? 0u : 1u;
            mma_bf16_ts(tmem + kKvColDV, a_p + 8 * kk, bdo + kk * (2048 >> 4), idesc_acc, accum);
            mma_bf16_ts(tmem + kKvColDK, a_ds + 8 * kk, bq + kk * (2048 >> 4), idesc_acc, accum);
          }
          mma_commit(&s.buf_free[bf]);
          mma_commit(&s.qd_empty[st]);
        }
        if (ok) mma_commit(&s.acc_full);
        ++active;
      }
      if (!ok) bwd_fail(&s.abort, a.dev_status);
      mma_commit(&s.drain[1]);
      mbar_wait(&s.drain[1], 0, nullptr);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax and epilogue
    // Thread t of warp w holds key rows 16 (w % 4) + t/4 and + 8 (M = 64 keys) and query columns
    // 8j + 2(t%4) + {0, 1}, j < 8, of a step's 64 queries (tcgen05.ld 16x256b).
    const int sp = warp & 3;
    const int t0 = lane & 3, q4 = lane >> 2;
    const int r0 = 16 * sp + q4, r1 = r0 + 8;
    const uint32_t lane_base = tmem + ((uint32_t)(sp * 32) << 16);
    const long ld = (long)g.heads_total * kD;
    long gs = 0;
    int active = 0;
    bool failed = false;
    auto give_up = [&]() {
      failed = true;
      *abort_flag = 1;
    };
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const int32_t* list;
      const int cnt = unit_list(u, list);
      const int j = u % g.nT, bh = u / g.nT, h = bh % g.heads, b = bh / g.heads;
      const int vcj = s.vc[j];
      const long off = ((long)b * g.Lp + (long)j * kTileElems) * ld + (long)(g.head0 + h) * kD;
      __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(a.dk) + off;
      __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(a.dv) + off;
      if (cnt == 0) {
        for (int c = 2 * t0; c < kD; c += 8) {
          *reinterpret_cast<uint32_t*>(dk + r0 * ld + c) = 0u;
          *reinterpret_cast<uint32_t*>(dk + r1 * ld + c) = 0u;
          *reinterpret_cast<uint32_t*>(dv + r0 * ld + c) = 0u;
          *reinterpret_cast<uint32_t*>(dv + r1 * ld + c) = 0u;
        }
        continue;
      }
      const bool key0 = r0 < vcj, key1 = r1 < vcj;
      // A step's query tile and the lse, delta and keep flags of this thread's 16 query columns
      // are loaded one step ahead (and the list entry two steps ahead), so that no step waits on
      // a chain of global loads.
      auto tile_at = [&](int n) {
        const int i = n < cnt ? list[n] : 0;
        return (i < 0 || i >= g.nT) ? 0 : i;  // out-of-range: unreachable, lists are in range
      };
      struct Meta {
        int i;
        float l[16], d[16];
        uint8_t k[16];
      };
      auto fetch = [&](int i, Meta& m) {
        m.i = i;
        const long qrow = ((long)bh * g.nT + i) * kTileElems;  // [B, heads, Lp] index of row 0
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const long qc = qrow + 8 * (c >> 1) + 2 * t0 + (c & 1);
          m.l[c] = a.lse[qc];
          m.d[c] = a.delta[qc];
          m.k[c] = a.keep != nullptr ? a.keep[qc] : (uint8_t)1;
        }
      };
      Meta nxt;
      fetch(tile_at(0), nxt);
      int i_ahead = tile_at(1);
      for (int n = 0; n < cnt; ++n, ++gs) {
        const Meta cur = nxt;
        if (n + 1 < cnt) fetch(i_ahead, nxt);
        i_ahead = tile_at(n + 2);
        const int vci = s.vc[cur.i];
        // lse (log2 units) and delta of this thread's 16 query columns; +inf lse masks a column
        float lq[16], dq[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int qc = 8 * (c >> 1) + 2 * t0 + (c & 1);
          const bool live = qc < vci && cur.k[c] != 0;
          lq[c] = live ? cur.l[c] * kLog2e : INFINITY;
          dq[c] = live ? cur.d[c] : 0.f;
        }
        const int bf = (int)(gs & 1);
        const uint32_t t_s = lane_base + kKvColS + kKvBuf * bf;
        const uint32_t t_dp = lane_base + kKvColDP + kKvBuf * bf;
        if (!mbar_wait(&s.s_full[bf], (uint32_t)((gs >> 1) & 1), abort_flag, lim)) give_up();
        tc_fence_after();
        uint32_t sv[32], pv[32];
        tmem_ld_16x256b_x8(t_s, sv);
        tmem_ld_16x256b_x8(t_dp, pv);
        tmem_wait_ld();
        uint32_t pw[16], dw[16];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          float p[4], d[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 2 * jj + (e & 1);  // this thread's column index 0..15
            const bool kv = e < 2 ? key0 : key1;
            const float x = ex2(fmaf(__uint_as_float(sv[4 * jj + e]), sl2, -lq[c]));
            p[e] = kv ? x : 0.f;  // exp2(-inf) = 0 for a masked query column
            d[e] = p[e] * (__uint_as_float(pv[4 * jj + e]) - dq[c]);
          }
          const __nv_bfloat162 p0 = __floats2bfloat162_rn(p[0], p[1]);
          const __nv_bfloat162 p1 = __floats2bfloat162_rn(p[2], p[3]);
          const __nv_bfloat162 d0 = __floats2bfloat162_rn(d[0], d[1]);
          const __nv_bfloat162 d1 = __floats2bfloat162_rn(d[2], d[3]);
          pw[2 * jj] = *reinterpret_cast<const uint32_t*>(&p0);
          pw[2 * jj + 1] = *reinterpret_cast<const uint32_t*>(&p1);
          dw[2 * jj] = *reinterpret_cast<const uint32_t*>(&d0);
          dw[2 * jj + 1] = *reinterpret_cast<const uint32_t*>(&d1);
        }
        // Written over the S^T and dP^T just read (no other reader: the buffer's next MMAs wait
        // for the dV / dK MMAs of this step).
        tmem_st_16x128b_x8(t_s, pw);
        tmem_st_16x128b_x8(t_dp, dw);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&s.p_full[bf]);
      }
      // ---- epilogue: dV and scale * dK for the valid key rows, zero for pad rows
      if (!mbar_wait(&s.acc_full, (uint32_t)(active & 1), abort_flag, lim)) give_up();
      tc_fence_after();
      failed = __any_sync(0xffffffffu, failed);
      if (!failed) {
        const int rown = 16 * sp + (lane & 15);
        const bool live = rown < vcj;
        for (int which = 0; which < 2; ++which) {
          const uint32_t col = which ? kKvColDK : kKvColDV;
          const float mul = which ? a.scale : 1.f;
          __nv_bfloat16* dst0 = which ? dk : dv;
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + col + 32 * c, o);
            tmem_wait_ld();
            if (lane < 16) {
              uint4 w4[4];
              uint32_t* w = reinterpret_cast<uint32_t*>(w4);
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const __nv_bfloat162 y = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * mul,
                                                               __uint_as_float(o[2 * e + 1]) * mul);
                w[e] = live ? *reinterpret_cast<const uint32_t*>(&y) : 0u;
              }
              uint4* dst = reinterpret_cast<uint4*>(dst0 + rown * ld + 32 * c);
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) dst[k4] = w4[k4];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&s.acc_empty);
      }
      ++active;
    }
    if (failed && lane == 0) bwd_fail(&s.abort, a.dev_status);
  }
  tc_fence_before();
  named_bar(kTeardown, kBwdThreads);
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ host side

bool make_map(CUtensorMap* m, const void* base, const Geo& g) {
  const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.heads_total, (cuuint64_t)g.B * g.Lp};
  const cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.heads_total * g.D * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  return encode_bf16_map(m, base, 3, dims, strides, box);
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Dynamic shared memory: the layout plus alignment slack, never less than half of an SM's 228 KB
// (one CTA per SM: each holds all 512 TMEM columns).
constexpr size_t one_per_sm(size_t bytes) { return bytes > 120 * 1024 ? bytes : 120 * 1024; }

template <int kD>
cudaError_t launch_bwd_d(const Geo& g, const BwdMaps& maps, const BwdArgs& a, cudaStream_t s) {
  const int units = g.B * g.heads * g.nT;
  const int grid = units < sm_count() ? units : sm_count();
  const size_t dq_smem = one_per_sm(sizeof(DqSmem<kD>) + 1024);
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<kD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<kD><<<grid, kBwdThreads, dq_smem, s>>>(maps, g, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t kv_smem = one_per_sm(sizeof(KvSmem<kD>) + 1024);
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kv_smem);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<kD><<<grid, kBwdThreads, kv_smem, s>>>(maps, g, a);
  return cudaGetLastError();
}

// Workspace of the backward pass, in order: dOe (bf16, [B, Lp, heads_total, D]: the call's heads
// only are written), delta (fp32 [B, heads, Lp]), the pair map (u8 [B, heads, nT, nT]), the
// key-to-query lists (int32 [B, heads, nT, nT]) and their counts (int32 [B, heads, nT]); each
// part starts on a 256-byte boundary.
struct BwdLayout {
  size_t dout, delta, map, q_idx, q_cnt, total;
};
inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
BwdLayout bwd_layout(const Geo& g) {
  BwdLayout l;
  const size_t bh = (size_t)g.B * g.heads;
  l.dout = 0;
  l.delta = l.dout + up256((size_t)g.B * g.Lp * g.heads_total * g.D * 2);
  l.map = l.delta + up256(bh * g.Lp * sizeof(float));
  l.q_idx = l.map + up256(bh * g.nT * g.nT);
  l.q_cnt = l.q_idx + up256(bh * g.nT * g.nT * sizeof(int32_t));
  l.total = l.q_cnt + up256(bh * g.nT * sizeof(int32_t));
  return l;
}

}  // namespace

size_t attn_bwd_workspace_bytes(const Geo& g) { return bwd_layout(g).total; }

cudaError_t launch_attn_bwd(const Geo& g, const AttnBwdArgs& in, cudaStream_t s) {
  const BwdLayout l = bwd_layout(g);
  uint8_t* ws = static_cast<uint8_t*>(in.workspace);
  __nv_bfloat16* dout_eff = reinterpret_cast<__nv_bfloat16*>(ws + l.dout);
  float* delta = reinterpret_cast<float*>(ws + l.delta);
  uint8_t* map = ws + l.map;
  int32_t* q_idx = reinterpret_cast<int32_t*>(ws + l.q_idx);
  int32_t* q_cnt = reinterpret_cast<int32_t*>(ws + l.q_cnt);
  // 1. dOe and delta
  dim3 pgrid(g.nT, g.heads, g.B);
  if (g.D == 128)
    bwd_prep_kernel<128><<<pgrid, 256, 0, s>>>(
        g, static_cast<const __nv_bfloat16*>(in.o), static_cast<const __nv_bfloat16*>(in.dout),
        in.keep, in.src_row, dout_eff, delta);
  else
    bwd_prep_kernel<64><<<pgrid, 256, 0, s>>>(
        g, static_cast<const __nv_bfloat16*>(in.o), static_cast<const __nv_bfloat16*>(in.dout),
        in.keep, in.src_row, dout_eff, delta);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. key-to-query lists
  const size_t map_bytes = (size_t)g.B * g.heads * g.nT * g.nT;
  e = cudaMemsetAsync(map, 0, map_bytes, s);
  if (e != cudaSuccess) return e;
  const long entries = (long)g.B * g.heads * g.nT * in.kmax;
  long blocks = (entries + 255) / 256;
  if (blocks > 148L * 16) blocks = 148L * 16;
  csc_scatter_kernel<<<(unsigned)blocks, 256, 0, s>>>(g, in.kv_idx, in.kv_cnt, in.kmax, map);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long rows = (long)g.B * g.heads * g.nT;
  blocks = (rows + 7) / 8;
  if (blocks > 148L * 16) blocks = 148L * 16;
  csc_build_kernel<<<(unsigned)blocks, 256, 0, s>>>(g, map, q_idx, q_cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. dQ, then dK and dV
  BwdMaps maps;
  if (!make_map(&maps.q, in.q, g) || !make_map(&maps.k, in.k, g) || !make_map(&maps.v, in.v, g) ||
      !make_map(&maps.dout, dout_eff, g))
    return cudaErrorInvalidValue;
  BwdArgs a{in.kv_idx, in.kv_cnt, in.kmax, q_idx, q_cnt, in.keep, in.lse, delta,
            in.dq,     in.dk,     in.dv,   in.scale, in.dev_status, in.wait_cycles};
  return g.D == 128 ? launch_bwd_d<128>(g, maps, a, s) : launch_bwd_d<64>(g, maps, a, s);
}

}  // namespace t3d
