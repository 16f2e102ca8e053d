// Fine stage on the sm_100a tensor cores: block-sparse softmax attention over the kept
// (query tile, key tile) pairs with tcgen05 MMAs accumulating in tensor memory (TMEM) and the kept
// key/value tiles fetched by TMA. One kernel template for head dimensions 64 and 128.
//
// FastVideo API docs, bsa_attn page, BSAAttentionImpl.__init__ / forward: bidirectional attention,
// one KV head per query head, softmax scale 1/sqrt(D), tile-ordered [B, L, heads, D] bf16 tensors,
// sparse attention per kept block pair, pruned query rows reconstructed afterwards.
//
// Shape of the computation. A work unit is one (batch, head, query tile): 64 query rows. Each step
// takes a PAIR of its kept key tiles (128 keys; an odd last tile is paired with a fully masked copy
// of itself) and computes, with M = 64 query rows,
//     S[64 q, 128 keys]  = Q . K_pair^T      (A = Q, B = K pair: shared memory, K-major)
//     O[64 q, D]        += P . V_pair         (A = P in TMEM, B = V pair in shared memory, MN-major)
// fp32 accumulation in TMEM. P lives in TMEM, so the tensor core's shared-memory operands are the
// query tile and the K and V pairs; its operand reads never compete with a P^T in shared memory.
//
// TMEM (512 columns; an M = 64 tile occupies lanes 0..15 of each 32-lane sub-partition):
//   S buffer b: columns 128 b .. 128 b + 127 (fp32)    O: 256 .. 255 + D (fp32)
//   P buffer b: 384 + 64 b .. 447 + 64 b (bf16 pairs: column c holds keys 2c, 2c + 1)
// Step n uses S and P buffer n & 1, so the softmax of step n + 1 never waits for the PV of step n.
//
// Scheduling. One persistent CTA per SM takes units from a queue: an atomic counter in the
// caller's workspace (zeroed on the stream before each launch), read by the K producer, which
// publishes each unit through a small ring in shared memory to the other roles. Units come in
// head-major order, so the CTAs working at one time share a head's K and V in L2; a CTA that drew
// short units simply draws more, so lists of uneven length (cumulative-mass selection, block masks,
// pruned queries) leave no CTA idle before the queue is empty.
//
// Roles (12 warps):
//   warp 0       TMA producer for the K pairs (2-stage ring) and the unit queue
//   warp 1       TMEM allocation; one thread issues the S MMAs and their commits
//   warp 2       one thread issues the PV MMAs and their commits
//   warp 3       TMA producer for the V pairs (2-stage ring) and for each unit's query tile (one
//                buffer, refilled once the previous unit's last S has completed, so the next unit's
//                scores start during the epilogue)
//   warps 4..11  softmax and epilogue, two warpgroups: warpgroup X takes the steps n with n % 2 == X
//                (S and P buffer X) and, in the epilogue, output columns X D/2 .. X D/2 + D/2 - 1.
//                Thread t of warp w owns query rows 16 (w % 4) + t/4 and that + 8, and the key
//                columns 8j + 2(t%4) + {0, 1} of its steps (tcgen05.ld 16x256b).
// S(n) is issued as soon as its K pair has landed and the softmax has read S(n - 2), so scores run
// up to two steps ahead; PV(n) as soon as P(n) is in TMEM.
//
// Softmax. The two warpgroups alternate steps, so each has two steps' time for one and their
// phases interleave: one computes exponentials while the other loads scores or reduces maxima.
// The per-row shift m (log2 units) is a chain along the steps: step n takes the shift after step
// n - 1 from the other warpgroup through shared memory (an mbarrier per parity), raises it only when
// a row's logits exceed it by more than kShiftSlack, publishes it, and then rescales the O rows
// concerned in TMEM (factor 1 for rows that did not move) once PV(n - 1) has landed. Any shift gives
// the same softmax; the bound keeps P within [0, 2^kShiftSlack] so nothing overflows. Each
// warpgroup keeps the running sums of its own steps relative to the last shift it used; the
// epilogue brings both to the final (largest) shift and adds them.
//
// Every mbarrier wait of the pipeline is bounded (AttnArgs::wait_cycles); on a timeout the CTA
// records T3D_DEV_TIMEOUT, stops issuing work, waits (bounded by the full limit) for its copies and
// MMAs in flight, frees TMEM and returns. The two warps of a pair leave their loops together: a
// failure is carried to the pair's next barrier, which ORs it.
#include "kernels.h"
#include "sm100.cuh"

namespace t3d {
namespace {

using namespace sm100;

// K and V pair rings of two stages, one per S / P buffer: stage gp & 1 is free once S(gp - 2)
// (for K) or PV(gp - 2) (for V) has completed, which the S and PV issuers already signal on
// s_full / pv_done, so the producers wait on those barriers and no separate "stage empty" commit
// is issued (an MMA-side commit costs the issuing thread about as much as an MMA).
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kUnitRing = 8;        // units published ahead by the queue reader
constexpr int kThreads = 384;       // 12 warps: producers / MMA, two softmax halves
constexpr int kSoftmaxThreads = 256;  // both softmax warpgroups
constexpr int kWgThreads = 128;       // one softmax warpgroup
constexpr int kTeardownBar = 5;       // named barrier of all threads before TMEM is released
constexpr int kLaunchRegs = 168;      // 65536 / 384, rounded down to a multiple of 8
constexpr int kProducerRegs = 72;
constexpr int kSoftmaxRegs = 216;
static_assert(128 * kProducerRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kShiftSlack = 8.f;  // log2 units: P <= 256 between shift updates
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;       // S buffer b at 128 b
constexpr uint32_t kColO = 256;
constexpr uint32_t kColP = 384;     // P buffer b at 384 + 64 b
constexpr uint32_t kTileBytes = 64 * 128;  // 64 rows x 128 B (one 64-element column block of a tile)
// The unit queue's readers: the V/Q producer, the two MMA issuers and every softmax thread.
constexpr uint32_t kUnitReaders = 3 + kSoftmaxThreads;

template <int kD>
struct Cfg {
  static_assert(kD == 64 || kD == 128, "head dimension 64 or 128");
  static constexpr int kHalves = kD / 64;                      // 128-byte column blocks of a row
  static constexpr uint32_t kPairBytes = kHalves * 2 * kTileBytes;  // two tiles, every block
  static constexpr uint32_t kQBytes = kHalves * kTileBytes;
  static constexpr uint32_t idesc_s = idesc_bf16(64, 128, false, false);  // A = Q, B = K, K-major
  static constexpr uint32_t idesc_o = idesc_bf16(64, kD, false, true);    // A = P (TMEM), B = V
};

template <int kD>
struct alignas(1024) SmemLayout {
  uint8_t k[kKStages][Cfg<kD>::kPairBytes];
  uint8_t v[kVStages][Cfg<kD>::kPairBytes];
  uint8_t q[2][Cfg<kD>::kQBytes];  // query tiles of consecutive units alternate buffers
  uint64_t k_full[kKStages];  // a K pair landed (TMA -> S issuer)
  uint64_t v_full[kVStages];  // a V pair landed (TMA -> PV issuer)
  uint64_t s_full[2], s_empty[2];  // s_full[b]: S of a step in buffer b (also frees K stage b)
  uint64_t p_full[2];   // P of a step written to TMEM buffer (step & 1) (softmax -> MMA)
  uint64_t pv_done[2];  // that step's PV MMAs complete: its P buffer and V stage free, O current
  uint64_t q_full[2];   // a unit's Q loaded into buffer (unit & 1) (TMA -> MMA)
  uint64_t q_empty[2];  // that unit's last S MMA complete: the buffer may be refilled
  uint64_t o_full;    // the unit's last PV complete (MMA -> softmax)
  uint64_t o_empty;   // O read by the epilogue (softmax -> MMA)
  uint64_t drain[2];  // all MMAs of the S issuer / the PV issuer complete
  uint64_t m_ready[2];      // shift of a step (parity b) published by warpgroup b
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];  // the unit queue's ring
  int unit[kUnitRing];      // unit index, or -1 once the queue is exhausted
  int ucnt[kUnitRing];      // its kv_cnt entry as read from global memory
  float mrow[2][64];        // [step & 1][row]: that shift
  float xsum[2][2][4][16];  // [unit & 1][warpgroup][warp % 4][row]: running sums, end of a unit
  float xm[2][2][4][16];    // [unit & 1][warpgroup][warp % 4][row]: the shift they are relative to
  uint8_t vc[kMaxTiles];    // valid token count of every tile
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(SmemLayout<128>) + 1024 <= 232448, "shared memory per CTA");
constexpr int kAbsent = -0x7fffffff - 1;  // list entry beyond kv_cnt

struct UnitInfo {
  int b, h, i, cnt, npairs;
  bool over, under;  // kv_cnt above kmax (clamped) / negative (treated as 0)
  const int32_t* list;
};

// kv_cnt entry of unit u (one global load; the queue reader publishes it with the unit).
__device__ __forceinline__ int unit_count(const AttnArgs& a, int u) {
  return a.kv_cnt[u];  // units are numbered (b, h, i) row-major, like kv_cnt
}

__device__ __forceinline__ UnitInfo unit_info(const Geo& g, const AttnArgs& a, int u, int c) {
  UnitInfo r;
  r.i = u % g.nT;
  const int bh = u / g.nT;
  r.h = bh % g.heads;
  r.b = bh / g.heads;
  r.over = c > a.kmax;
  r.under = c < 0;
  r.cnt = r.under ? 0 : (r.over ? a.kmax : c);
  r.npairs = (r.cnt + 1) >> 1;
  r.list = a.kv_idx + ((long)bh * g.nT + r.i) * a.kmax;
  return r;
}

// Key tile of entry e of the list, or -1 if absent / out of range.
__device__ __forceinline__ int list_tile(const Geo& g, const UnitInfo& u, int e) {
  if (e >= u.cnt) return -1;
  const int j = u.list[e];
  return (j >= 0 && j < g.nT) ? j : -1;
}

template <int kD>
__device__ __forceinline__ void fail(SmemLayout<kD>& s, int32_t* status) {
  s.abort = 1;
  report(status, T3D_DEV_TIMEOUT);
}

// Next unit from the ring (every reader calls it once per unit, in the same order): the unit index
// and its kv_cnt entry, or -1 when the queue is exhausted or the wait gave up (then `ok` is
// cleared).
template <int kD>
__device__ __forceinline__ int take_unit(SmemLayout<kD>& s, long& nu, volatile int* abort_flag,
                                         long long lim, bool& ok, int& cnt) {
  const int slot = (int)(nu % kUnitRing);
  if (!mbar_wait(&s.unit_full[slot], (uint32_t)((nu / kUnitRing) & 1), abort_flag, lim)) {
    ok = false;
    return -1;
  }
  const int u = s.unit[slot];
  cnt = s.ucnt[slot];
  mbar_arrive(&s.unit_empty[slot]);
  ++nu;
  return u;
}

struct Maps {
  CUtensorMap q, k, v;
};

// Loads the K or V pair of step gp of unit ui into stage gp % kStages of a ring once the MMAs that
// read the stage's previous pair have completed, as signalled on `done` (s_full for K, pv_done
// for V: with two stages, stage gp % 2 is step gp's buffer) (lane 0 of a producer warp). False on
// a timeout.
template <int kD, int kStages>
__device__ __forceinline__ bool load_pair(const Geo& g, const UnitInfo& ui, int n, long gp,
                                          const CUtensorMap* map,
                                          uint8_t (*ring)[Cfg<kD>::kPairBytes], uint64_t* full,
                                          uint64_t* done, volatile int* abort_flag, long long lim) {
  static_assert(kStages == 2, "a stage is step gp's S / P buffer");
  const int st = (int)(gp % kStages);
  int ja = list_tile(g, ui, 2 * n), jb = list_tile(g, ui, 2 * n + 1);  // read while waiting
  if (!mbar_wait(&done[st], (uint32_t)(((gp / kStages) & 1) ^ 1), abort_flag, lim)) return false;
  if (ja < 0) ja = 0;  // masked in the softmax; any finite tile will do
  if (jb < 0) jb = ja;
  mbar_expect_tx(&full[st], Cfg<kD>::kPairBytes);
  for (int hh = 0; hh < Cfg<kD>::kHalves; ++hh) {
    uint8_t* dst = ring[st] + hh * 2 * kTileBytes;
    tma_load_3d(dst, map, &full[st], 64 * hh, g.head0 + ui.h, ui.b * g.Lp + ja * kTileElems);
    tma_load_3d(dst + kTileBytes, map, &full[st], 64 * hh, g.head0 + ui.h,
                ui.b * g.Lp + jb * kTileElems);
  }
  return true;
}

// Before exit, the last loads issued to a ring must have landed (bounded by the full limit).
template <int kStages>
__device__ __forceinline__ void drain_ring(uint64_t* full, long issued) {
  for (long t = issued - kStages; t < issued; ++t)
    if (t >= 0) mbar_wait(&full[t % kStages], (uint32_t)((t / kStages) & 1), nullptr);
}

template <int kD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ Maps maps, Geo g, AttnArgs a, float sl2) {
  using C = Cfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  SmemLayout<kD>& s = *reinterpret_cast<SmemLayout<kD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_units = g.B * g.heads * g.nT;
  const long long lim = a.wait_cycles;
  volatile int* abort_flag = &s.abort;

  if (threadIdx.x == 0) {
    for (int t = 0; t < kKStages; ++t) mbar_init(&s.k_full[t], 1);
    for (int t = 0; t < kVStages; ++t) mbar_init(&s.v_full[t], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.s_empty[t], kWgThreads);
      mbar_init(&s.p_full[t], kWgThreads);
      mbar_init(&s.m_ready[t], kWgThreads);
      mbar_init(&s.pv_done[t], 1);
    }
    for (int t = 0; t < kUnitRing; ++t) {
      mbar_init(&s.unit_full[t], 1);
      mbar_init(&s.unit_empty[t], kUnitReaders);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.q_full[t], 1);
      mbar_init(&s.q_empty[t], 1);
    }
    mbar_init(&s.o_full, 1);
    mbar_init(&s.o_empty, kSoftmaxThreads);
    mbar_init(&s.drain[0], 1);
    mbar_init(&s.drain[1], 1);
    s.abort = 0;
    fence_mbar_init();
  }
  for (int t = threadIdx.x; t < g.nT; t += kThreads)
    s.vc[t] = a.vc_tab != nullptr ? a.vc_tab[t] : (uint8_t)tile_valid_count(g, t);
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
  // Registers move from the producer / issuer warpgroup to the softmax warpgroups: 384 threads
  // launch with 168 each; 128 x 72 + 256 x 216 is the same total. The two sides never share code
  // after the split (each ends with its own arrival at the teardown barrier).
  if (warp < 4) {
    regs_dec<kProducerRegs>();
    if (warp == 0) {
      // ------------------------------------------------------------- queue reader and K producer
      if (lane == 0) {
        uint32_t* next_unit = static_cast<uint32_t*>(a.workspace);
        long nu = 0, gp = 0;
        bool ok = true;
        int cur = (int)atomicAdd(next_unit, 1u);
        int cur_cnt = cur < total_units ? unit_count(a, cur) : 0;
        while (ok) {
          const int slot = (int)(nu % kUnitRing);
          if (!mbar_wait(&s.unit_empty[slot], (uint32_t)(((nu / kUnitRing) & 1) ^ 1), abort_flag,
                         lim)) {
            ok = false;
            break;
          }
          const int u = cur < total_units ? cur : -1;
          s.unit[slot] = u;
          s.ucnt[slot] = cur_cnt;
          mbar_arrive(&s.unit_full[slot]);
          ++nu;
          if (u < 0) break;
          // The next index (and then its count) is fetched now and used after this unit's loads,
          // hiding both latencies.
          const int nxt = (int)atomicAdd(next_unit, 1u);
          const UnitInfo ui = unit_info(g, a, u, cur_cnt);
          int nxt_cnt = 0;
          for (int n = 0; n < ui.npairs; ++n, ++gp) {  // gp counts the loads issued
            if (!load_pair<kD, kKStages>(g, ui, n, gp, &maps.k, s.k, s.k_full, s.s_full,
                                         abort_flag, lim)) {
              ok = false;
              break;
            }
            if (n == 0 && nxt < total_units) nxt_cnt = unit_count(a, nxt);
          }
          if (ui.npairs == 0 && nxt < total_units) nxt_cnt = unit_count(a, nxt);
          cur = nxt;
          cur_cnt = nxt_cnt;
        }
        if (!ok) fail(s, a.dev_status);
        drain_ring<kKStages>(s.k_full, gp);
      }
    } else if (warp == 3) {
      // ------------------------------------------------------------- V and Q producer
      if (lane == 0) {
        long nu = 0, gp = 0;
        int nq = 0;  // query tiles loaded
        bool ok = true;
        while (ok) {
          int cnt = 0;
          const int u = take_unit(s, nu, abort_flag, lim, ok, cnt);
          if (u < 0) break;
          const UnitInfo ui = unit_info(g, a, u, cnt);
          if (ui.npairs == 0) continue;
          // Q buffer nq & 1 is free once the last S of the unit two back has completed, so a
          // unit's query tile loads while the previous unit is still running.
          const int qb = nq & 1;
          if (!mbar_wait(&s.q_empty[qb], (uint32_t)(((nq >> 1) & 1) ^ 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&s.q_full[qb], C::kQBytes);
          const int row0 = ui.b * g.Lp + ui.i * kTileElems;
          for (int hh = 0; hh < C::kHalves; ++hh)
            tma_load_3d(s.q[qb] + hh * kTileBytes, &maps.q, &s.q_full[qb], 64 * hh,
                        g.head0 + ui.h, row0);
          ++nq;
          for (int n = 0; n < ui.npairs; ++n, ++gp) {  // gp counts the loads issued
            if (!load_pair<kD, kVStages>(g, ui, n, gp, &maps.v, s.v, s.v_full, s.pv_done,
                                         abort_flag, lim)) {
              ok = false;
              break;
            }
          }
        }
        if (!ok) fail(s, a.dev_status);
        drain_ring<kVStages>(s.v_full, gp);
        for (int t = nq - 2; t < nq; ++t)
          if (t >= 0) mbar_wait(&s.q_full[t & 1], (uint32_t)((t >> 1) & 1), nullptr);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------- S issuer
      // An mbarrier wait (or any acquire followed by tcgen05.fence) in the thread that issues MMAs
      // lets that thread's queued MMAs drain before its next MMA issues, about 150 cycles of idle
      // pipe per wait point, while the same wait in another thread costs the pipe nothing. So S and
      // PV have one issuing thread each: the pipe takes work from whichever is ready, and each
      // thread's waits are covered by the other's queued MMAs. tcgen05.commit tracks the MMAs of
      // the committing thread only, which is what each barrier below needs.
      if (lane == 0) {
        int active = 0;  // units with at least one pair, in order
        long nu = 0, gp = 0;  // units taken, global step index
        bool ok = true;
        // Shared-memory descriptors are linear in the start address (bits 0-13 hold address >> 4 and
        // every buffer lies below 256 KB), so each MMA's operand is a base descriptor plus a constant.
        const uint64_t dk = sdesc_sw128(smem_u32(s.k[0]), 16, 1024);
        const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0]), 16, 1024);
        while (ok) {
          int cnt = 0;
          const int u = take_unit(s, nu, abort_flag, lim, ok, cnt);
          if (u < 0) break;
          const int np = unit_info(g, a, u, cnt).npairs;
          if (np == 0) continue;
          const int qb = active & 1;
          if (!mbar_wait(&s.q_full[qb], (uint32_t)((active >> 1) & 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint64_t dq = dq0 + (uint64_t)(qb * (C::kQBytes >> 4));
          for (int n = 0; n < np; ++n, ++gp) {
            // S(gp) = Q . K_pair^T into S buffer gp & 1, once the softmax has read S(gp - 2).
            const int ks = (int)(gp % kKStages);
            const int b = (int)(gp & 1);
            if (!mbar_wait(&s.k_full[ks], (uint32_t)((gp / kKStages) & 1), abort_flag, lim) ||
                !mbar_wait(&s.s_empty[b], (uint32_t)(((gp >> 1) & 1) ^ 1), abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t db0 = dk + (uint64_t)(ks * (C::kPairBytes >> 4));
            const uint32_t d_s = tmem + kColS + 128 * b;
  #pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {  // 16 elements of D per MMA
              const int hh = kk >> 2, st = kk & 3;
              mma_bf16(d_s, dq + ((hh * kTileBytes + st * 32) >> 4),
                       db0 + ((hh * 2 * kTileBytes + st * 32) >> 4), C::idesc_s, kk ? 1u : 0u);
            }
            mma_commit(&s.s_full[b]);
            if (n == np - 1) mma_commit(&s.q_empty[qb]);
          }
          ++active;
        }
        if (!ok) fail(s, a.dev_status);
        // Every MMA issued must complete before TMEM is released.
        mma_commit(&s.drain[0]);
        mbar_wait(&s.drain[0], 0, nullptr);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------- PV issuer
      if (lane == 0) {
        int active = 0;
        long nu = 0, gp = 0;
        bool ok = true;
        const uint64_t dv = sdesc_sw128(smem_u32(s.v[0]), 2 * kTileBytes, 1024);
        while (ok) {
          int cnt = 0;
          const int u = take_unit(s, nu, abort_flag, lim, ok, cnt);
          if (u < 0) break;
          const int np = unit_info(g, a, u, cnt).npairs;
          if (np == 0) continue;
          for (int n = 0; n < np; ++n, ++gp) {
            // O (+)= P . V_pair of step gp; the unit's first PV overwrites O once the epilogue of the
            // previous unit has read it.
            const int vs = (int)(gp % kVStages);
            if ((n == 0 && !mbar_wait(&s.o_empty, (uint32_t)((active & 1) ^ 1), abort_flag, lim)) ||
                !mbar_wait(&s.v_full[vs], (uint32_t)((gp / kVStages) & 1), abort_flag, lim) ||
                !mbar_wait(&s.p_full[gp & 1], (uint32_t)((gp >> 1) & 1), abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t db0 = dv + (uint64_t)(vs * (C::kPairBytes >> 4));
  #pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys (16 rows x 128 B of each column block) per MMA
              mma_bf16_ts(tmem + kColO, tmem + kColP + 64 * (uint32_t)(gp & 1) + 8 * kk,
                          db0 + kk * (2048 >> 4), C::idesc_o, (n == 0 && kk == 0) ? 0u : 1u);
            mma_commit(&s.pv_done[gp & 1]);
            if (n == np - 1) mma_commit(&s.o_full);
          }
          ++active;
        }
        if (!ok) fail(s, a.dev_status);
        mma_commit(&s.drain[1]);
        mbar_wait(&s.drain[1], 0, nullptr);
      }
    }
    tc_fence_before();
    named_bar(kTeardownBar, kThreads);
    tc_fence_after();
    if (warp == 1) {
      __syncwarp();
      tmem_dealloc(tmem, kTmemCols);
    }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------- softmax + epilogue (warps 4..11)
    constexpr int kCols = kD / 2;       // output columns of one warpgroup
    const int wg = (warp - 4) >> 2;     // this warpgroup takes the steps gp with gp & 1 == wg
    const int sp = warp & 3;            // TMEM sub-partition: lanes [32 sp, 32 sp + 32)
    const int bar_id = 1 + sp;          // named barrier of warps w and w + 4 (same TMEM lanes)
    const int t0 = lane & 3;
    const int q4 = lane >> 2;           // row within the warp's 8-row group
    const int r0 = 16 * sp + q4, r1 = r0 + 8;  // this thread's two query rows
    const uint32_t lane_base = tmem + ((uint32_t)(sp * 32) << 16);
    const uint32_t t_s = lane_base + kColS + 128 * (uint32_t)wg;  // this warpgroup's S buffer
    const uint32_t t_p = lane_base + kColP + 64 * (uint32_t)wg;   // and P buffer
    const long ld = (long)g.heads_total * kD;
    const int col0 = kCols * wg;        // output columns this warpgroup writes
    const bool reporter = wg == 0 && sp == 0 && lane == 0;  // records list-size problems
    int active = 0;
    long nu = 0;
    long gp = 0;  // global index of the unit's first step
    bool reported = false;
    bool failed = false;  // a bounded wait gave up; carried to the pair's next barrier
    auto give_up = [&]() {  // every other wait of the CTA returns at once from here on
      failed = true;
      *abort_flag = 1;
    };
    while (true) {
      bool got = true;
      int cnt = 0;
      const int u = take_unit(s, nu, abort_flag, lim, got, cnt);
      if (!got) give_up();
      // Both warps of a pair leave together (a failed wait in either ends both).
      if (named_bar_or(bar_id, 64, failed)) {
        failed = true;
        break;
      }
      if (u < 0) break;
      const UnitInfo ui = unit_info(g, a, u, cnt);
      if (reporter && (ui.over || ui.under))
        report(a.dev_status, ui.over ? T3D_DEV_OVERFLOW : T3D_DEV_INDEX_RANGE);
      const long row0 = (long)ui.b * g.Lp + (long)ui.i * kTileElems;
      const int vci = s.vc[ui.i];
      __nv_bfloat16* out =
          static_cast<__nv_bfloat16*>(a.o) + row0 * ld + (long)(g.head0 + ui.h) * kD;
      if (ui.npairs == 0) {
        // No kept key tile: this thread's two output rows are zero (this warpgroup's columns).
        for (int c = col0 + 2 * t0; c < col0 + kCols; c += 8) {
          *reinterpret_cast<uint32_t*>(out + r0 * ld + c) = 0u;
          *reinterpret_cast<uint32_t*>(out + r1 * ld + c) = 0u;
        }
        if (a.lse != nullptr && wg == 0 && t0 == 0) {
          float* lr = a.lse + (((long)ui.b * g.heads + ui.h) * g.Lp + (long)ui.i * kTileElems);
          lr[r0] = -INFINITY;
          lr[r1] = -INFINITY;
        }
        continue;
      }
      // mw: the shift this warpgroup used at its latest step of the unit; l is relative to it.
      float mw0 = -INFINITY, mw1 = -INFINITY;
      float l0 = 0.f, l1 = 0.f;  // sums over this thread's columns of this warpgroup's steps
      const int nfirst = (int)((wg ^ (int)(gp & 1)) & 1);  // first step of the unit that is ours
      // Key tiles of our next step (prefetched one own step ahead).
      int ea = (2 * nfirst < ui.cnt) ? ui.list[2 * nfirst] : kAbsent;
      int eb = (2 * nfirst + 1 < ui.cnt) ? ui.list[2 * nfirst + 1] : kAbsent;
      for (int n = nfirst; n < ui.npairs; n += 2) {
        const long gs = gp + n;  // global step index; gs & 1 == wg
        const int ja = ea, jb = eb;
        ea = (2 * n + 4 < ui.cnt) ? ui.list[2 * n + 4] : kAbsent;
        eb = (2 * n + 5 < ui.cnt) ? ui.list[2 * n + 5] : kAbsent;
        if (!mbar_wait(&s.s_full[wg], (uint32_t)((gs >> 1) & 1), abort_flag, lim)) give_up();
        tc_fence_after();
        uint32_t v[64];
        tmem_ld_16x256b_x16(t_s, v);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s.s_empty[wg]);
        // Valid keys: tile a gives keys 0..63, tile b keys 64..127.
        const bool ina = ja >= 0 && ja < g.nT, inb = jb >= 0 && jb < g.nT;
        if (!reported && ((ja != kAbsent && !ina) || (jb != kAbsent && !inb))) {
          report(a.dev_status, T3D_DEV_INDEX_RANGE);
          reported = true;
        }
        const int ca = ina ? s.vc[ja] : 0, cb = inb ? s.vc[jb] : 0;
        if (ca < kTileElems || cb < kTileElems) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int key = 8 * j + 2 * t0 + e;  // 0..127
              const bool valid = key < 64 ? key < ca : key - 64 < cb;
              if (!valid) {
                v[4 * j + e] = __float_as_uint(-INFINITY);
                v[4 * j + 2 + e] = __float_as_uint(-INFINITY);
              }
            }
          }
        }
        // Row maxima (the 4 threads of a row hold its 128 columns), as trees of 3-input maxima.
        float x0, x1;
        {
          float r0v[32], r1v[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            r0v[2 * j] = __uint_as_float(v[4 * j]);
            r0v[2 * j + 1] = __uint_as_float(v[4 * j + 1]);
            r1v[2 * j] = __uint_as_float(v[4 * j + 2]);
            r1v[2 * j + 1] = __uint_as_float(v[4 * j + 3]);
          }
          x0 = max_of_32(r0v);
          x1 = max_of_32(r1v);
        }
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
        x0 *= sl2;  // log2 units (the scale is positive)
        x1 *= sl2;
        // The shift after the previous step (the other warpgroup's), then ours for this step.
        // Every step waits for its predecessor's, so the two barriers never run a phase apart.
        float mp0 = -INFINITY, mp1 = -INFINITY;
        if (gs > 0) {
          if (!mbar_wait(&s.m_ready[wg ^ 1], (uint32_t)(((gs - 1) >> 1) & 1), abort_flag, lim))
            give_up();
          if (n > 0) {
            mp0 = s.mrow[wg ^ 1][r0];
            mp1 = s.mrow[wg ^ 1][r1];
          }
        }
        const bool up0 = x0 > mp0 + kShiftSlack || (mp0 == -INFINITY && x0 > -INFINITY);
        const bool up1 = x1 > mp1 + kShiftSlack || (mp1 == -INFINITY && x1 > -INFINITY);
        const float n0 = up0 ? fmaxf(mp0, x0) : mp0, n1 = up1 ? fmaxf(mp1, x1) : mp1;
        if (t0 == 0) {
          s.mrow[wg][r0] = n0;
          s.mrow[wg][r1] = n1;
        }
        mbar_arrive(&s.m_ready[wg]);
        // Our running sums follow the shift (it never decreases).
        if (mw0 != n0) l0 = (mw0 == -INFINITY) ? 0.f : l0 * ex2(mw0 - n0);
        if (mw1 != n1) l1 = (mw1 == -INFINITY) ? 0.f : l1 * ex2(mw1 - n1);
        mw0 = n0;
        mw1 = n1;
        // P = exp2(x * scale - shift) as bf16 pairs, computed before any wait on the PV MMAs: keys
        // 8j + 2 t0, + 1 go to P column 4j + t0 (the layout tcgen05.st 16x128b writes).
        const float ns0 = n0 == -INFINITY ? 0.f : -n0, ns1 = n1 == -INFINITY ? 0.f : -n1;
        uint32_t pw[2][16];  // keys 0..63, 64..127
        {
          float ls0[2] = {0.f, 0.f}, ls1[2] = {0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float p00 = ex2(fmaf(__uint_as_float(v[4 * j]), sl2, ns0));
            const float p01 = ex2(fmaf(__uint_as_float(v[4 * j + 1]), sl2, ns0));
            const float p10 = ex2(fmaf(__uint_as_float(v[4 * j + 2]), sl2, ns1));
            const float p11 = ex2(fmaf(__uint_as_float(v[4 * j + 3]), sl2, ns1));
            ls0[j & 1] += p00 + p01;
            ls1[j & 1] += p10 + p11;
            __nv_bfloat162 q0 = __floats2bfloat162_rn(p00, p01);
            __nv_bfloat162 q1 = __floats2bfloat162_rn(p10, p11);
            pw[j >> 3][2 * (j & 7)] = *reinterpret_cast<uint32_t*>(&q0);
            pw[j >> 3][2 * (j & 7) + 1] = *reinterpret_cast<uint32_t*>(&q1);
          }
          l0 += ls0[0] + ls0[1];
          l1 += ls1[0] + ls1[1];
        }
        // Our P buffer is free once the PV of our previous step (two steps back) has landed.
        if (gs >= 2) {
          if (!mbar_wait(&s.pv_done[wg], (uint32_t)(((gs - 2) >> 1) & 1), abort_flag, lim))
            give_up();
          tc_fence_after();
        }
        tmem_st_16x128b_x8(t_p, pw[0]);
        tmem_st_16x128b_x8(t_p + 32, pw[1]);
        // O follows the shift too: rescale the warp's rows (factor 1 where the shift held) once the
        // previous step's PV has landed; our own PV of this step is issued only after this.
        if (n > 0 && __any_sync(0xffffffffu, up0 || up1)) {
          if (!mbar_wait(&s.pv_done[wg ^ 1], (uint32_t)(((gs - 1) >> 1) & 1), abort_flag, lim))
            give_up();
          tc_fence_after();
          const float a0 = !up0 ? 1.f : (mp0 == -INFINITY ? 0.f : ex2(mp0 - n0));
          const float a1 = !up1 ? 1.f : (mp1 == -INFINITY ? 0.f : ex2(mp1 - n1));
#pragma unroll
          for (int hc = 0; hc < kD / 64; ++hc) {
            uint32_t o[32];
            tmem_ld_16x256b_x8(lane_base + kColO + 64 * hc, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              o[4 * j] = __float_as_uint(__uint_as_float(o[4 * j]) * a0);
              o[4 * j + 1] = __float_as_uint(__uint_as_float(o[4 * j + 1]) * a0);
              o[4 * j + 2] = __float_as_uint(__uint_as_float(o[4 * j + 2]) * a1);
              o[4 * j + 3] = __float_as_uint(__uint_as_float(o[4 * j + 3]) * a1);
            }
            tmem_st_16x256b_x8(lane_base + kColO + 64 * hc, o);
          }
          tmem_wait_st();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&s.p_full[wg]);
      }
      gp += ui.npairs;
      // ---- epilogue: O / l for this thread's rows, bf16, into the tiled output
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      const int ub = active & 1;  // the swap buffers alternate by unit
      if (t0 == 0) {
        s.xsum[ub][wg][sp][q4] = l0;
        s.xsum[ub][wg][sp][q4 + 8] = l1;
        s.xm[ub][wg][sp][q4] = mw0;
        s.xm[ub][wg][sp][q4 + 8] = mw1;
      }
      if (named_bar_or(bar_id, 64, failed)) {
        failed = true;
        break;
      }
      // The two warpgroups' sums, each relative to the last shift it used, brought to the final
      // shift (the larger: the shift never decreases along the steps).
      float i0, i1;
      {
        const float om0 = s.xm[ub][wg ^ 1][sp][q4], om1 = s.xm[ub][wg ^ 1][sp][q4 + 8];
        const float ol0 = s.xsum[ub][wg ^ 1][sp][q4], ol1 = s.xsum[ub][wg ^ 1][sp][q4 + 8];
        const float mf0 = fmaxf(mw0, om0), mf1 = fmaxf(mw1, om1);
        const float s0 = (mw0 == -INFINITY ? 0.f : l0 * ex2(mw0 - mf0)) +
                         (om0 == -INFINITY ? 0.f : ol0 * ex2(om0 - mf0));
        const float s1 = (mw1 == -INFINITY ? 0.f : l1 * ex2(mw1 - mf1)) +
                         (om1 == -INFINITY ? 0.f : ol1 * ex2(om1 - mf1));
        i0 = s0 > 0.f ? 1.f / s0 : 0.f;
        i1 = s1 > 0.f ? 1.f / s1 : 0.f;
        if (a.lse != nullptr && wg == 0 && t0 == 0) {
          // log sum_c exp(scale q.k_c) = ln 2 * (final shift + log2 of the sum relative to it)
          float* lr = a.lse + (((long)ui.b * g.heads + ui.h) * g.Lp + (long)ui.i * kTileElems);
          lr[r0] = s0 > 0.f ? (mf0 + log2f(s0)) * kLn2 : -INFINITY;
          lr[r1] = s1 > 0.f ? (mf1 + log2f(s1)) * kLn2 : -INFINITY;
        }
      }
      // Pruned-query variant: the output rows that take this lane's row (row 16 sp + lane for
      // lane < 16), as a bit mask over the tile's 64 rows: a kept row takes itself, a pruned row
      // its source row (a source outside the tile falls back to the row itself).
      uint64_t takers = 0;
      const int rown = 16 * sp + (lane & 15);
      if (a.keep != nullptr) {
        const long blk = ((long)ui.b * g.heads + ui.h) * g.nT + ui.i;
        const uint4* kp = reinterpret_cast<const uint4*>(a.keep + blk * kTileElems);
        const uint4* sr = reinterpret_cast<const uint4*>(a.src_row + blk * kTileElems);
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          const uint4 kv = kp[w4], sv = sr[w4];
          const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int rr = 16 * w4 + e;
            const uint32_t kb = (kw[e >> 2] >> (8 * (e & 3))) & 0xffu;
            uint32_t sb = (sw[e >> 2] >> (8 * (e & 3))) & 0xffu;
            if (kb != 0u || sb >= (uint32_t)kTileElems) sb = (uint32_t)rr;
            if (sb == (uint32_t)rown) takers |= 1ull << rr;
          }
        }
      } else {
        takers = 1ull << rown;
      }
      if (!mbar_wait(&s.o_full, (uint32_t)(active & 1), abort_flag, lim)) give_up();
      tc_fence_after();
      failed = __any_sync(0xffffffffu, failed);  // the TMEM loads below are warp-collective
      if (!failed) {
        // O rows are read with the 32-lane shape: lane L < 16 of this warp holds row 16 sp + L
        // (the M = 64 layout), 32 columns per load, so a row goes out in 16-byte stores. Its 1 / l
        // comes from the threads that own the row in the 16x256b layout (row r0 of lanes 4L.., or
        // r1).
        const float ia = __shfl_sync(0xffffffffu, i0, 4 * (lane & 7));
        const float ib = __shfl_sync(0xffffffffu, i1, 4 * (lane & 7));
        const float inv = (lane & 15) < 8 ? ia : ib;
        // All of this warpgroup's O columns come into registers first, so O is released to the
        // next unit's first PV before the normalisation and the global stores.
        uint32_t o[kCols / 32][32];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(lane_base + kColO + col0 + 32 * c, o[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s.o_empty);
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          const int cc = col0 + 32 * c;
          if (lane < 16) {
            uint4 w4[4];
            uint32_t* w = reinterpret_cast<uint32_t*>(w4);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              __nv_bfloat162 y = __floats2bfloat162_rn(__uint_as_float(o[c][2 * e]) * inv,
                                                       __uint_as_float(o[c][2 * e + 1]) * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&y);
            }
            // Every output row that takes this row's result; rows past the tile's valid count
            // are zero.
            for (uint64_t m = takers; m != 0; m &= m - 1) {
              const int rr = __ffsll((long long)m) - 1;
              uint4* dst = reinterpret_cast<uint4*>(out + rr * ld + cc);
              const bool zero = rr >= vci;
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) dst[k4] = zero ? make_uint4(0u, 0u, 0u, 0u) : w4[k4];
            }
          }
        }
      }
      ++active;
    }
    if (failed && lane == 0) fail(s, a.dev_status);
    tc_fence_before();
    named_bar(kTeardownBar, kThreads);
  }
}

// ---------------------------------------------------------------------------------- host side

// 3D map over a [B * Lp, heads_total, D] bf16 tensor; box = 64 rows x 1 head x 64 elements, 128B
// swizzle (a unit of head h reads head coordinate head0 + h).
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

// Dynamic shared memory of a CTA: the layout plus alignment slack, and never less than half of an
// SM's 228 KB, so that no SM ever holds two CTAs (the second would wait for the first's TMEM).
template <int kD>
constexpr size_t smem_bytes() {
  return sizeof(SmemLayout<kD>) + 1024 > 120 * 1024 ? sizeof(SmemLayout<kD>) + 1024 : 120 * 1024;
}

template <int kD>
cudaError_t launch_d(const Maps& maps, const Geo& g, const AttnArgs& a, cudaStream_t s) {
  const size_t smem = smem_bytes<kD>();
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<kD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int units = g.B * g.heads * g.nT;
  const int grid = units < sm_count() ? units : sm_count();
  const float sl2 = a.scale * 1.4426950408889634f;
  attn_sm100_kernel<kD><<<grid, kThreads, smem, s>>>(maps, g, a, sl2);
  return cudaGetLastError();
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

bool encode_bf16_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_workspace_bytes(const Geo& g, int kmax) {
  (void)g;
  (void)kmax;
  return kAttnWorkspaceBytes;
}

cudaError_t launch_attn(const Geo& g, const AttnArgs& a, cudaStream_t s) {
  Maps maps;
  if (!make_map(&maps.q, a.q, g) || !make_map(&maps.k, a.k, g) || !make_map(&maps.v, a.v, g))
    return cudaErrorInvalidValue;
  // The unit queue starts at zero on every launch.
  cudaError_t e = cudaMemsetAsync(a.workspace, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  return g.D == 128 ? launch_d<128>(maps, g, a, s) : launch_d<64>(maps, g, a, s);
}

}  // namespace t3d
