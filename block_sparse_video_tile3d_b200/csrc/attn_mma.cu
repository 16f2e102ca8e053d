// Fine stage, warp-MMA version: block-sparse softmax attention over kept (query tile, key tile)
// pairs with mma.sync m16n8k16 bf16 tensor-core instructions and an online softmax.
//
// FastVideo API docs, bsa_attn page, BSAAttentionImpl.__init__ / forward: bidirectional, one KV
// head per query head, scale 1/sqrt(D), tile-ordered [B, L, heads, D] bf16 tensors; the sparse
// attention runs per kept block pair and pruned query rows are reconstructed afterwards.
//
// One CTA (4 warps) per (query tile, head, batch); warp w owns query rows 16w .. 16w + 15.
// The kept key tiles of the query tile are streamed through a double-buffered cp.async pipeline
// (K and V, 64 x D each, XOR-swizzled 16-byte chunks so ldmatrix is conflict-free). For each key
// tile: S = Q K^T (fp32), pad keys of ragged tiles masked to -inf, running max / sum in the log2
// domain with quad shuffles, P rounded to bf16 and fed straight from registers as the A operand of
// O += P V. The epilogue divides by the row sum, stages O in shared memory, writes zeros for pad
// rows and, in the pruned-query variant, copies each pruned row from its source row.
#include "kernels.h"

namespace t3d {
namespace {

constexpr int kAttnThreads = 128;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Element offset of 16-byte chunk `chunk` of row `row` in a [64][D] bf16 tile.
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * D + ((chunk ^ (row & 7)) << 3);
}

// Asynchronously copy 64 rows x D of one tile (global row stride `ld` elements) into smem.
template <int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16* dst, const __nv_bfloat16* src, long ld) {
  constexpr int kChunks = D / 8;
  for (int e = threadIdx.x; e < kTileElems * kChunks; e += kAttnThreads) {
    const int r = e / kChunks, c = e - r * kChunks;
    cp_async16(smem_addr(dst + swz<D>(r, c)), src + r * ld + c * 8);
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads) attn_mma_kernel(Geo g, AttnArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __nv_bfloat16* sq = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sk = sq + kTileElems * D;      // [2][64*D]
  __nv_bfloat16* sv = sk + 2 * kTileElems * D;  // [2][64*D]

  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long bh = (long)b * g.heads + h;
  const long ld = (long)g.heads * D;
  const long head_off = (long)h * D;
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(a.v);
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(a.o);

  int cnt = a.kv_cnt[bh * g.nT + i];
  if (cnt > a.kmax || cnt < 0) {
    if (tid == 0) report(a.dev_status, T3D_DEV_OVERFLOW);
    cnt = cnt < 0 ? 0 : a.kmax;
  }
  const int32_t* list = a.kv_idx + (bh * g.nT + i) * a.kmax;
  const long tile_rows = (long)b * g.Lp;

  auto tile_of = [&](int t, int& vcj) -> int {
    const int j = list[t];
    if (j < 0 || j >= g.nT) {
      vcj = 0;  // masked entirely
      return 0;
    }
    vcj = tile_valid_count(g, j);
    return j;
  };

  load_tile<D>(sq, Q + (tile_rows + (long)i * kTileElems) * ld + head_off, ld);
  cp_async_commit();
  int vc_next = 0;
  if (cnt > 0) {
    const int j0 = tile_of(0, vc_next);
    load_tile<D>(sk, K + (tile_rows + (long)j0 * kTileElems) * ld + head_off, ld);
    load_tile<D>(sv, V + (tile_rows + (long)j0 * kTileElems) * ld + head_off, ld);
  }
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();

  // Q fragments for this warp's 16 rows, all of D.
  uint32_t qf[D / 16][4];
  {
    const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int c = 2 * ks + (lane >> 4);
      ldsm_x4(smem_addr(sq + swz<D>(r, c)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale * 1.4426950408889634f;
  const int tq = lane & 3;

  for (int t = 0; t < cnt; ++t) {
    const int buf = t & 1;
    const int vcj = vc_next;
    if (t + 1 < cnt) {
      const int jn = tile_of(t + 1, vc_next);
      load_tile<D>(sk + (buf ^ 1) * kTileElems * D,
                   K + (tile_rows + (long)jn * kTileElems) * ld + head_off, ld);
      load_tile<D>(sv + (buf ^ 1) * kTileElems * D,
                   V + (tile_rows + (long)jn * kTileElems) * ld + head_off, ld);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (tid == 0 && vcj == 0 && (list[t] < 0 || list[t] >= g.nT))
      report(a.dev_status, T3D_DEV_INDEX_RANGE);

    const __nv_bfloat16* kb = sk + buf * kTileElems * D;
    const __nv_bfloat16* vb = sv + buf * kTileElems * D;

    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + (lane & 7) + 8 * (lane >> 4);
        const int c = 2 * ks + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_addr(kb + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
    }

    // Scale into the log2 domain and mask pad keys.
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = n * 8 + 2 * tq + e;
        const bool ok = col < vcj;
        s[n][e] = ok ? s[n][e] * sl2 : -INFINITY;
        s[n][2 + e] = ok ? s[n][2 + e] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, s[n][e]);
        mx1 = fmaxf(mx1, s[n][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = ex2(m0 - base0), al1 = ex2(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      s[n][0] = ex2(s[n][0] - base0);
      s[n][1] = ex2(s[n][1] - base0);
      s[n][2] = ex2(s[n][2] - base1);
      s[n][3] = ex2(s[n][3] - base1);
      rs0 += s[n][0] + s[n][1];
      rs1 += s[n][2] + s[n][3];
    }
    l0 = l0 * al0 + rs0;
    l1 = l1 * al1 + rs1;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= al0;
      o[n][1] *= al0;
      o[n][2] *= al1;
      o[n][3] *= al1;
    }

    // O += P V, P from registers (C layout of two adjacent n-blocks = A layout of one k-step).
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      const int r = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int nd = 0; nd < D / 16; ++nd) {
        const int c = 2 * nd + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_addr(vb + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(o[2 * nd], pa, b0, b1);
        mma_bf16(o[2 * nd + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
  const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;

  // Stage O (bf16) in this warp's own rows of the Q buffer.
  const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    *reinterpret_cast<uint32_t*>(sq + swz<D>(r0, n) + 2 * tq) =
        pack_bf16(o[n][0] * inv0, o[n][1] * inv0);
    *reinterpret_cast<uint32_t*>(sq + swz<D>(r0 + 8, n) + 2 * tq) =
        pack_bf16(o[n][2] * inv1, o[n][3] * inv1);
  }
  __syncthreads();

  const int vci = tile_valid_count(g, i);
  const uint8_t* keep = a.keep ? a.keep + (bh * g.nT + i) * kTileElems : nullptr;
  const uint8_t* srcr = a.src_row ? a.src_row + (bh * g.nT + i) * kTileElems : nullptr;
  constexpr int kChunks = D / 8;
  __nv_bfloat16* out = O + (tile_rows + (long)i * kTileElems) * ld + head_off;
  for (int e = tid; e < kTileElems * kChunks; e += kAttnThreads) {
    const int r = e / kChunks, c = e - r * kChunks;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < vci && cnt > 0) {
      int sr = r;
      if (keep != nullptr && !keep[r]) {
        sr = srcr[r];
        if (sr >= kTileElems) sr = r;
      }
      val = *reinterpret_cast<const uint4*>(sq + swz<D>(sr, c));
    }
    *reinterpret_cast<uint4*>(out + r * ld + c * 8) = val;
  }
}

template <int D>
cudaError_t launch_attn_d(const Geo& g, const AttnArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)5 * kTileElems * D * sizeof(__nv_bfloat16);
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nT, g.heads, g.B);
  attn_mma_kernel<D><<<grid, kAttnThreads, smem, s>>>(g, a);
  return cudaGetLastError();
}

}  // namespace

size_t attn_workspace_bytes(const Geo& g, int kmax) {
  (void)g;
  (void)kmax;
  return 0;
}

cudaError_t launch_attn_mma(const Geo& g, const AttnArgs& a, cudaStream_t s) {
  if (g.D == 128) return launch_attn_d<128>(g, a, s);
  return launch_attn_d<64>(g, a, s);
}

cudaError_t launch_attn(const Geo& g, const AttnArgs& a, cudaStream_t s) {
  if (g.D == 128) return launch_attn_sm100(g, a, s);
  return launch_attn_mma(g, a, s);
}

}  // namespace t3d
