// C ABI of libtile3d: argument validation, then one asynchronous launch per call.
// Declarations and the contract of each call are in include/tile3d.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include "kernels.h"
#include "tile3d_testing.h"

namespace {

thread_local char g_err[512] = "";

// Limit of each pipeline wait of the attention kernel, in clock cycles (tile3d_testing.h).
constexpr long long kDefaultWaitCycles = 4000000000LL;  // ~2 s at 2 GHz
long long g_wait_cycles = kDefaultWaitCycles;

t3d_status fail(t3d_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

t3d_status ok() {
  g_err[0] = '\0';
  return T3D_OK;
}

t3d_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(T3D_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

t3d_status check_geom(const t3d_geom* g, t3d::Geo* out) {
  if (g == nullptr) return fail(T3D_ERR_INVALID, "geometry pointer is NULL");
  if (g->B < 1 || g->T < 1 || g->H < 1 || g->W < 1 || g->heads < 1)
    return fail(T3D_ERR_INVALID, "B, T, H, W and heads must be >= 1 (got %d, %d, %d, %d, %d)", g->B,
                g->T, g->H, g->W, g->heads);
  if (g->D != 64 && g->D != 128)
    return fail(T3D_ERR_UNSUPPORTED, "head dimension D=%d is not supported (64 or 128)", g->D);
  if (g->head0 < 0 || g->heads_total < 0)
    return fail(T3D_ERR_INVALID, "head0=%d and heads_total=%d must be >= 0", g->head0,
                g->heads_total);
  if (g->heads_total == 0 && g->head0 != 0)
    return fail(T3D_ERR_INVALID, "head0=%d needs heads_total (0 means heads_total = heads)",
                g->head0);
  if (g->heads_total > 0 && g->head0 + g->heads > g->heads_total)
    return fail(T3D_ERR_INVALID, "heads %d .. %d lie outside the %d heads of a row", g->head0,
                g->head0 + g->heads - 1, g->heads_total);
  const t3d::Geo geo = t3d::make_geo(*g);
  if (geo.nT > t3d::kMaxTiles)
    return fail(T3D_ERR_UNSUPPORTED, "%d tiles exceed the supported maximum %d", geo.nT,
                t3d::kMaxTiles);
  if ((long long)g->B * geo.Lp * geo.heads_total > (1LL << 31))
    return fail(T3D_ERR_UNSUPPORTED, "B * Lp * heads_total = %lld token-head rows exceeds 2^31",
                (long long)g->B * geo.Lp * geo.heads_total);
  *out = geo;
  return T3D_OK;
}

#define T3D_CHECK(expr)            \
  do {                             \
    t3d_status _st = (expr);       \
    if (_st != T3D_OK) return _st; \
  } while (0)

t3d_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(T3D_ERR_INVALID, "%s is NULL", name);
  if (!aligned16(p)) return fail(T3D_ERR_INVALID, "%s is not 16-byte aligned", name);
  return T3D_OK;
}

t3d_status check_ptr4(const void* p, const char* name) {
  if (p == nullptr) return fail(T3D_ERR_INVALID, "%s is NULL", name);
  if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)
    return fail(T3D_ERR_INVALID, "%s is not 4-byte aligned", name);
  return T3D_OK;
}

cudaStream_t as_stream(t3d_stream s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

const char* t3d_last_error_string(void) { return g_err; }

const char* t3d_version(void) { return "0.2.0"; }

t3d_status t3d_testing_set_wait_cycles(long long cycles) {
  if (cycles < 0) return fail(T3D_ERR_INVALID, "cycles=%lld must be >= 0", cycles);
  g_wait_cycles = cycles == 0 ? kDefaultWaitCycles : cycles;
  return ok();
}

t3d_status tile3d_geometry(const t3d_geom* g, int* nT, int* Lp, int32_t* vc_host) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  if (nT) *nT = geo.nT;
  if (Lp) *Lp = geo.Lp;
  if (vc_host)
    for (int i = 0; i < geo.nT; ++i) vc_host[i] = t3d::tile_valid_count(geo, i);
  return ok();
}

t3d_status tile3d_scatter(const t3d_geom* g, const void* x, void* y, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(x, "x"));
  T3D_CHECK(check_ptr(y, "y"));
  return cuda_status(t3d::launch_scatter(geo, x, y, as_stream(stream)), "tile3d_scatter");
}

t3d_status tile3d_gather(const t3d_geom* g, const void* y, void* x, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(y, "y"));
  T3D_CHECK(check_ptr(x, "x"));
  return cuda_status(t3d::launch_gather(geo, y, x, as_stream(stream)), "tile3d_gather");
}

t3d_status tile_pool(const t3d_geom* g, const void* y, float* pooled, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(y, "y"));
  T3D_CHECK(check_ptr(pooled, "pooled"));
  return cuda_status(t3d::launch_pool(geo, y, pooled, as_stream(stream)), "tile_pool");
}

t3d_status tile3d_scatter_pool(const t3d_geom* g, const void* x, void* y, float* pooled,
                               t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(x, "x"));
  T3D_CHECK(check_ptr(y, "y"));
  T3D_CHECK(check_ptr(pooled, "pooled"));
  return cuda_status(t3d::launch_scatter_pool(geo, x, y, pooled, as_stream(stream)),
                     "tile3d_scatter_pool");
}

size_t tile_select_workspace_size(const t3d_geom* g) {
  t3d::Geo geo;
  if (check_geom(g, &geo) != T3D_OK) return 0;
  return t3d::select_workspace_bytes(geo);
}

static t3d_status check_select_workspace(const t3d::Geo& geo, const void* workspace,
                                         size_t ws_bytes) {
  const size_t need = t3d::select_workspace_bytes(geo);
  if (ws_bytes < need)
    return fail(T3D_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                ws_bytes, need);
  return check_ptr(workspace, "workspace");
}

t3d_status tile_select_topk(const t3d_geom* g, const float* pq, const float* pk, int k,
                            int32_t* kv_idx, int32_t* kv_cnt, void* workspace, size_t ws_bytes,
                            int32_t* dev_status, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(pq, "pq"));
  T3D_CHECK(check_ptr(pk, "pk"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (k < 1) return fail(T3D_ERR_INVALID, "k=%d must be >= 1", k);
  T3D_CHECK(check_select_workspace(geo, workspace, ws_bytes));
  return cuda_status(t3d::launch_select_topk(geo, pq, pk, k, kv_idx, kv_cnt, workspace, dev_status,
                                             as_stream(stream)),
                     "tile_select_topk");
}

t3d_status tile_select_mass(const t3d_geom* g, const float* pq, const float* pk, float scale,
                            float mass, int min_k, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                            void* workspace, size_t ws_bytes, int32_t* dev_status,
                            t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(pq, "pq"));
  T3D_CHECK(check_ptr(pk, "pk"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (!(scale > 0.f) || !isfinite(scale))
    return fail(T3D_ERR_INVALID, "scale=%g must be finite and > 0", (double)scale);
  if (!(mass > 0.f) || mass > 1.f)
    return fail(T3D_ERR_INVALID, "mass=%g must lie in (0, 1]", (double)mass);
  if (min_k < 1) return fail(T3D_ERR_INVALID, "min_k=%d must be >= 1", min_k);
  if (kmax < 1 || kmax > geo.nT)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [1, nT=%d]", kmax, geo.nT);
  T3D_CHECK(check_select_workspace(geo, workspace, ws_bytes));
  return cuda_status(t3d::launch_select_mass(geo, pq, pk, scale, mass, min_k, kmax, kv_idx, kv_cnt,
                                             workspace, dev_status, as_stream(stream)),
                     "tile_select_mass");
}

t3d_status tile_prune_queries(const t3d_geom* g, const void* q, float cos_thresh, uint8_t* keep,
                              uint8_t* src_row, float* pq_kept, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(q, "q"));
  T3D_CHECK(check_ptr(keep, "keep"));
  T3D_CHECK(check_ptr(src_row, "src_row"));
  T3D_CHECK(check_ptr(pq_kept, "pq_kept"));
  if (geo.L != geo.Lp)
    return fail(T3D_ERR_INVALID,
                "query pruning needs every tile full (L=%d must equal 64 * nT = %d)", geo.L, geo.Lp);
  if (isnan(cos_thresh)) return fail(T3D_ERR_INVALID, "cos_thresh is NaN");
  return cuda_status(
      t3d::launch_prune(geo, q, cos_thresh, 0, keep, src_row, pq_kept, as_stream(stream)),
      "tile_prune_queries");
}

t3d_status tile_prune_queries_ratio(const t3d_geom* g, const void* q, float keep_ratio,
                                    uint8_t* keep, uint8_t* src_row, float* pq_kept,
                                    t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_ptr(q, "q"));
  T3D_CHECK(check_ptr(keep, "keep"));
  T3D_CHECK(check_ptr(src_row, "src_row"));
  T3D_CHECK(check_ptr(pq_kept, "pq_kept"));
  if (geo.L != geo.Lp)
    return fail(T3D_ERR_INVALID,
                "query pruning needs every tile full (L=%d must equal 64 * nT = %d)", geo.L, geo.Lp);
  if (!(keep_ratio > 0.f && keep_ratio <= 1.f))
    return fail(T3D_ERR_INVALID, "keep_ratio=%g must lie in (0, 1]", (double)keep_ratio);
  // Kept rows per block, in double so that the count is the exact floor of 64 * keep_ratio.
  int keep_size = (int)floor((double)keep_ratio * t3d::kTileElems);
  keep_size = keep_size < 1 ? 1 : (keep_size > t3d::kTileElems ? t3d::kTileElems : keep_size);
  return cuda_status(
      t3d::launch_prune(geo, q, 0.f, keep_size, keep, src_row, pq_kept, as_stream(stream)),
      "tile_prune_queries_ratio");
}

t3d_status block_mask_to_index(const t3d_geom* g, const uint8_t* mask, int kmax, int32_t* kv_idx,
                               int32_t* kv_cnt, int32_t* dev_status, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  if (mask == nullptr) return fail(T3D_ERR_INVALID, "mask is NULL");
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (kmax < 1 || kmax > geo.nT)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [1, nT=%d]", kmax, geo.nT);
  return cuda_status(
      t3d::launch_mask_to_index(geo, mask, kmax, kv_idx, kv_cnt, dev_status, as_stream(stream)),
      "block_mask_to_index");
}

size_t block_sparse_attn_workspace_size(const t3d_geom* g, int kmax) {
  t3d::Geo geo;
  if (check_geom(g, &geo) != T3D_OK) return 0;
  return t3d::attn_workspace_bytes(geo, kmax);
}

t3d_status block_sparse_attn_fwd(const t3d_geom* g, const void* q, const void* k, const void* v,
                                 void* o, const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                 const uint8_t* keep, const uint8_t* src_row, float softmax_scale,
                                 int causal, int num_kv_heads, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  if (causal != 0)
    return fail(T3D_ERR_UNSUPPORTED, "the attention is bidirectional; causal=1 is unsupported");
  if (num_kv_heads != g->heads)
    return fail(T3D_ERR_UNSUPPORTED,
                "grouped-query attention is unsupported (num_kv_heads=%d, heads=%d)", num_kv_heads,
                g->heads);
  const double expected = 1.0 / sqrt((double)g->D);
  const double diff = fabs((double)softmax_scale - expected);
  if (!(diff <= fmax(1e-4 * fmax(fabs((double)softmax_scale), expected), 1e-5)))
    return fail(T3D_ERR_INVALID, "softmax_scale=%.8g must be 1/sqrt(D)=%.8g", (double)softmax_scale,
                expected);
  T3D_CHECK(check_ptr(q, "q"));
  T3D_CHECK(check_ptr(k, "k"));
  T3D_CHECK(check_ptr(v, "v"));
  T3D_CHECK(check_ptr(o, "o"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (kmax < 1 || kmax > geo.nT)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [1, nT=%d]", kmax, geo.nT);
  if ((keep == nullptr) != (src_row == nullptr))
    return fail(T3D_ERR_INVALID, "keep and src_row must both be given or both be NULL");
  if (keep != nullptr && geo.L != geo.Lp)
    return fail(T3D_ERR_INVALID, "pruned-query attention needs every tile full (L=%d, Lp=%d)",
                geo.L, geo.Lp);
  const size_t need = t3d::attn_workspace_bytes(geo, kmax);
  if (ws_bytes < need)
    return fail(T3D_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                ws_bytes, need);
  if (need > 0) T3D_CHECK(check_ptr(workspace, "workspace"));
  t3d::AttnArgs a{q, k, v, o, kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale,
                  workspace, ws_bytes, dev_status, g_wait_cycles};
  return cuda_status(t3d::launch_attn(geo, a, as_stream(stream)), "block_sparse_attn_fwd");
}

// The checks every attention entry point makes (BSAAttentionImpl.__init__ contract, pointers,
// list capacity, pruning geometry).
static t3d_status check_attn_call(const t3d_geom* g, const t3d::Geo& geo, const void* q,
                                  const void* k, const void* v, const int32_t* kv_idx,
                                  const int32_t* kv_cnt, int kmax, const uint8_t* keep,
                                  const uint8_t* src_row, float softmax_scale, int causal,
                                  int num_kv_heads) {
  if (causal != 0)
    return fail(T3D_ERR_UNSUPPORTED, "the attention is bidirectional; causal=1 is unsupported");
  if (num_kv_heads != g->heads)
    return fail(T3D_ERR_UNSUPPORTED,
                "grouped-query attention is unsupported (num_kv_heads=%d, heads=%d)", num_kv_heads,
                g->heads);
  const double expected = 1.0 / sqrt((double)g->D);
  const double diff = fabs((double)softmax_scale - expected);
  if (!(diff <= fmax(1e-4 * fmax(fabs((double)softmax_scale), expected), 1e-5)))
    return fail(T3D_ERR_INVALID, "softmax_scale=%.8g must be 1/sqrt(D)=%.8g", (double)softmax_scale,
                expected);
  T3D_CHECK(check_ptr(q, "q"));
  T3D_CHECK(check_ptr(k, "k"));
  T3D_CHECK(check_ptr(v, "v"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (kmax < 1 || kmax > geo.nT)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [1, nT=%d]", kmax, geo.nT);
  if ((keep == nullptr) != (src_row == nullptr))
    return fail(T3D_ERR_INVALID, "keep and src_row must both be given or both be NULL");
  if (keep != nullptr && geo.L != geo.Lp)
    return fail(T3D_ERR_INVALID, "pruned-query attention needs every tile full (L=%d, Lp=%d)",
                geo.L, geo.Lp);
  return T3D_OK;
}

t3d_status block_sparse_attn_fwd_lse(const t3d_geom* g, const void* q, const void* k,
                                     const void* v, void* o, float* lse, const int32_t* kv_idx,
                                     const int32_t* kv_cnt, int kmax, const uint8_t* keep,
                                     const uint8_t* src_row, float softmax_scale, int causal,
                                     int num_kv_heads, void* workspace, size_t ws_bytes,
                                     int32_t* dev_status, t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_attn_call(g, geo, q, k, v, kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale,
                            causal, num_kv_heads));
  T3D_CHECK(check_ptr(o, "o"));
  T3D_CHECK(check_ptr(lse, "lse"));
  const size_t need = t3d::attn_workspace_bytes(geo, kmax);
  if (ws_bytes < need)
    return fail(T3D_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                ws_bytes, need);
  T3D_CHECK(check_ptr(workspace, "workspace"));
  t3d::AttnArgs a{q, k, v, o, kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale,
                  workspace, ws_bytes, dev_status, g_wait_cycles, lse};
  return cuda_status(t3d::launch_attn(geo, a, as_stream(stream)), "block_sparse_attn_fwd_lse");
}

size_t block_sparse_attn_bwd_workspace_size(const t3d_geom* g, int kmax) {
  t3d::Geo geo;
  (void)kmax;
  if (check_geom(g, &geo) != T3D_OK) return 0;
  return t3d::attn_bwd_workspace_bytes(geo);
}

t3d_status block_sparse_attn_bwd(const t3d_geom* g, const void* q, const void* k, const void* v,
                                 const void* o, const void* dout, const float* lse,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                 const uint8_t* keep, const uint8_t* src_row, float softmax_scale,
                                 int causal, int num_kv_heads, void* dq, void* dk, void* dv,
                                 void* workspace, size_t ws_bytes, int32_t* dev_status,
                                 t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  T3D_CHECK(check_attn_call(g, geo, q, k, v, kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale,
                            causal, num_kv_heads));
  T3D_CHECK(check_ptr(o, "o"));
  T3D_CHECK(check_ptr(dout, "dout"));
  T3D_CHECK(check_ptr(lse, "lse"));
  T3D_CHECK(check_ptr(dq, "dq"));
  T3D_CHECK(check_ptr(dk, "dk"));
  T3D_CHECK(check_ptr(dv, "dv"));
  const size_t need = t3d::attn_bwd_workspace_bytes(geo);
  if (ws_bytes < need)
    return fail(T3D_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                ws_bytes, need);
  T3D_CHECK(check_ptr(workspace, "workspace"));
  t3d::AttnBwdArgs a{q, k, v, o, dout, lse, kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale,
                     dq, dk, dv, workspace, dev_status, g_wait_cycles};
  return cuda_status(t3d::launch_attn_bwd(geo, a, as_stream(stream)), "block_sparse_attn_bwd");
}

t3d_status block_sparse_attn_fwd_noalloc(const t3d_geom* g, const void* q, const void* k,
                                         const void* v, void* o, const int32_t* kv_idx,
                                         const int32_t* kv_cnt, int kmax, const uint8_t* keep,
                                         const uint8_t* src_row, float softmax_scale, int causal,
                                         int num_kv_heads, int32_t* dev_status,
                                         t3d_stream stream) {
  t3d::Geo geo;
  T3D_CHECK(check_geom(g, &geo));
  if (causal != 0)
    return fail(T3D_ERR_UNSUPPORTED, "the attention is bidirectional; causal=1 is unsupported");
  if (num_kv_heads != g->heads)
    return fail(T3D_ERR_UNSUPPORTED,
                "grouped-query attention is unsupported (num_kv_heads=%d, heads=%d)", num_kv_heads,
                g->heads);
  const double expected = 1.0 / sqrt((double)g->D);
  const double diff = fabs((double)softmax_scale - expected);
  if (!(diff <= fmax(1e-4 * fmax(fabs((double)softmax_scale), expected), 1e-5)))
    return fail(T3D_ERR_INVALID, "softmax_scale=%.8g must be 1/sqrt(D)=%.8g", (double)softmax_scale,
                expected);
  T3D_CHECK(check_ptr(q, "q"));
  T3D_CHECK(check_ptr(k, "k"));
  T3D_CHECK(check_ptr(v, "v"));
  T3D_CHECK(check_ptr(o, "o"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (kmax < 1 || kmax > geo.nT)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [1, nT=%d]", kmax, geo.nT);
  if ((keep == nullptr) != (src_row == nullptr))
    return fail(T3D_ERR_INVALID, "keep and src_row must both be given or both be NULL");
  if (keep != nullptr && geo.L != geo.Lp)
    return fail(T3D_ERR_INVALID, "pruned-query attention needs every tile full (L=%d, Lp=%d)",
                geo.L, geo.Lp);
  const size_t need = t3d::attn_workspace_bytes(geo, kmax);
  if (need > t3d::kNoAllocScratchBytes)
    return fail(T3D_ERR_UNSUPPORTED,
                "this problem needs %zu bytes of scratch, more than the library's fixed %zu bytes",
                need, t3d::kNoAllocScratchBytes);
  void* scratch = nullptr;
  cudaError_t e = t3d::noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_status(e, "block_sparse_attn_fwd_noalloc: scratch address");
  t3d::AttnArgs a{q, k, v, o, kv_idx, kv_cnt, kmax, keep, src_row, softmax_scale,
                  scratch, t3d::kNoAllocScratchBytes, dev_status, g_wait_cycles};
  return cuda_status(t3d::launch_attn(geo, a, as_stream(stream)), "block_sparse_attn_fwd_noalloc");
}

}  // extern "C"

// ------------------------------------------------------------------ packed multi-region sequences

static t3d_status check_packed(const t3d_packed* p, t3d::PackedGeo* out) {
  if (p == nullptr) return fail(T3D_ERR_INVALID, "packed geometry pointer is NULL");
  if (p->B < 1 || p->heads < 1 || p->n_tiles < 1 || p->rows < 1)
    return fail(T3D_ERR_INVALID, "B, heads, n_tiles and rows must be >= 1 (got %d, %d, %d, %d)",
                p->B, p->heads, p->n_tiles, p->rows);
  if (p->D != 64 && p->D != 128)
    return fail(T3D_ERR_UNSUPPORTED, "head dimension D=%d is not supported (64 or 128)", p->D);
  if (p->tile_elems != 64 && p->tile_elems != 128)
    return fail(T3D_ERR_INVALID, "tile_elems=%d must be 64 or 128", p->tile_elems);
  if (p->head0 < 0 || p->heads_total < 0 || (p->heads_total == 0 && p->head0 != 0) ||
      (p->heads_total > 0 && p->head0 + p->heads > p->heads_total))
    return fail(T3D_ERR_INVALID, "heads %d .. %d do not lie inside the %d heads of a row", p->head0,
                p->head0 + p->heads - 1, p->heads_total);
  T3D_CHECK(check_ptr4(p->slot_row, "slot_row"));
  T3D_CHECK(check_ptr4(p->vc, "vc"));
  const int ht = p->heads_total > 0 ? p->heads_total : p->heads;
  const long long slots = (long long)p->n_tiles * p->tile_elems;
  if ((long long)p->B * (slots > p->rows ? slots : p->rows) * ht > (1LL << 31))
    return fail(T3D_ERR_UNSUPPORTED, "B * rows * heads_total exceeds 2^31 token-head rows");
  t3d::PackedGeo g;
  g.B = p->B;
  g.heads = p->heads;
  g.D = p->D;
  g.heads_total = ht;
  g.head0 = p->head0;
  g.E = p->tile_elems;
  g.n_tiles = p->n_tiles;
  g.rows = p->rows;
  g.row_chunks = p->heads * p->D / 8;
  g.row_stride = ht * p->D / 8;
  g.row_off = p->head0 * p->D / 8;
  g.slot_row = p->slot_row;
  g.vc = p->vc;
  *out = g;
  return T3D_OK;
}

// Geometry of the score product of a packed buffer: n_tiles rows per head.
static t3d::Geo packed_score_geo(const t3d::PackedGeo& p) {
  t3d::Geo g = t3d::packed_attn_geo(p);
  g.nT = p.n_tiles;
  g.nw = p.n_tiles;
  g.Lp = p.n_tiles * p.E;
  g.L = g.Lp;
  return g;
}

static int keep_count(double rate, int n) {
  const int k = (int)(rate * (double)n);  // truncation, as int() of a positive value
  return k < n ? k : n;
}

static t3d_status check_spans(int n_tiles, int mode, int n_prefix, int n_regions,
                              const int32_t* spans, const double* keep_rates, t3d::SpanSpec* sp,
                              int* cap) {
  if (mode != T3D_PACKED_EXEMPT && mode != T3D_PACKED_COMPETE && mode != T3D_PACKED_DENSE)
    return fail(T3D_ERR_INVALID, "mode=%d is not a T3D_PACKED_* mode", mode);
  if (n_regions < 1 || n_regions > t3d::kMaxRegions)
    return fail(T3D_ERR_INVALID, "n_regions=%d must lie in [1, %d]", n_regions, t3d::kMaxRegions);
  if (spans == nullptr || keep_rates == nullptr)
    return fail(T3D_ERR_INVALID, "spans and keep_rates must be given");
  if (n_prefix < 0 || spans[0] != n_prefix || spans[2 * n_regions - 1] != n_tiles)
    return fail(T3D_ERR_INVALID, "the regions must run from the prefix (%d tiles) to n_tiles=%d",
                n_prefix, n_tiles);
  if (mode == T3D_PACKED_COMPETE && n_regions != 1)
    return fail(T3D_ERR_INVALID, "compete mode supports the generated-video region only (%d regions)",
                n_regions);
  sp->mode = mode;
  sp->n_prefix = n_prefix;
  sp->n_regions = n_regions;
  int sum = 0;
  for (int r = 0; r < n_regions; ++r) {
    const int lo = spans[2 * r], hi = spans[2 * r + 1];
    if (hi <= lo || (r > 0 && lo != spans[2 * r - 1]))
      return fail(T3D_ERR_INVALID, "region %d spans [%d, %d): regions must be consecutive and non-empty",
                  r, lo, hi);
    if (!(keep_rates[r] >= 0.0 && keep_rates[r] <= 1.0))
      return fail(T3D_ERR_INVALID, "keep rate %g of region %d must lie in [0, 1]", keep_rates[r], r);
    sp->lo[r] = lo;
    sp->hi[r] = hi;
    sp->k[r] = keep_count(keep_rates[r], hi - lo);
    sum += sp->k[r];
  }
  sp->k_total = keep_count(keep_rates[n_regions - 1], n_tiles);
  if (mode == T3D_PACKED_DENSE) *cap = n_tiles;
  else if (mode == T3D_PACKED_COMPETE) *cap = sp->k_total;
  else *cap = n_prefix > 0 ? n_tiles : sum;
  if (*cap < 1) *cap = 1;
  return T3D_OK;
}

extern "C" {

t3d_status t3d_packed_geometry(const t3d_segment* segs, int n_segs, int tile_t, int tile_h,
                               int tile_w, t3d_packed_layout* layout, int32_t* spans, int32_t* vc,
                               int32_t* slot_row) {
  if (segs == nullptr || n_segs < 1) return fail(T3D_ERR_INVALID, "no segments");
  if (layout == nullptr) return fail(T3D_ERR_INVALID, "layout pointer is NULL");
  if (tile_t < 1 || tile_h < 1 || tile_w < 1)
    return fail(T3D_ERR_INVALID, "tile shape %d x %d x %d must be positive", tile_t, tile_h, tile_w);
  const int E = tile_t * tile_h * tile_w;
  if (E != 64 && E != 128)
    return fail(T3D_ERR_INVALID, "tile shape %d x %d x %d holds %d tokens (64 or 128)", tile_t,
                tile_h, tile_w, E);
  auto cdiv = [](long long a, long long b) { return (a + b - 1) / b; };
  long long rows = 0, tiles = 0, prefix = 0;
  int regions = 0;
  for (int i = 0; i < n_segs; ++i) {
    const t3d_segment& g = segs[i];
    if (g.rows > 0 && g.t == 0 && g.h == 0 && g.w == 0) {
      rows += g.rows;
      prefix += cdiv(g.rows, E);
    } else if (g.rows == 0 && g.t >= 1 && g.h >= 1 && g.w >= 1) {
      rows += (long long)g.t * g.h * g.w;
      tiles += cdiv(g.t, tile_t) * cdiv(g.h, tile_h) * cdiv(g.w, tile_w);
      ++regions;
    } else {
      return fail(T3D_ERR_INVALID,
                  "segment %d (rows=%d, t=%d, h=%d, w=%d) is neither a dense run nor a region", i,
                  g.rows, g.t, g.h, g.w);
    }
  }
  tiles += prefix;
  if (regions == 0) return fail(T3D_ERR_INVALID, "a packed sequence needs at least one video region");
  if (rows > (1LL << 31) - 1 || tiles * E > (1LL << 31) - 1)
    return fail(T3D_ERR_INVALID, "%lld rows / %lld slots exceed 2^31", rows, tiles * E);
  layout->n_tiles = (int)tiles;
  layout->rows = (int)rows;
  layout->n_prefix = (int)prefix;
  layout->n_regions = regions;
  if (spans == nullptr && vc == nullptr && slot_row == nullptr) return ok();
  // Packed-order start row of every segment, then the tiles: dense runs first, then regions.
  int tile = 0, region = 0;
  long long start = 0;
  for (int pass = 0; pass < 2; ++pass) {
    start = 0;
    for (int i = 0; i < n_segs; ++i) {
      const t3d_segment& g = segs[i];
      const bool dense = g.rows > 0;
      const long long len = dense ? (long long)g.rows : (long long)g.t * g.h * g.w;
      if (dense && pass == 0) {
        for (long long a = 0; a < g.rows; a += E) {
          const int n = (int)(g.rows - a < E ? g.rows - a : E);
          if (vc) vc[tile] = n;
          if (slot_row)
            for (int s = 0; s < E; ++s) slot_row[(long long)tile * E + s] = s < n ? (int32_t)(start + a + s) : -1;
          ++tile;
        }
      } else if (!dense && pass == 1) {
        if (spans) spans[2 * region] = tile;
        const int nt = (int)cdiv(g.t, tile_t), nh = (int)cdiv(g.h, tile_h), nw = (int)cdiv(g.w, tile_w);
        for (int ta = 0; ta < nt; ++ta)
          for (int ha = 0; ha < nh; ++ha)
            for (int wa = 0; wa < nw; ++wa) {
              const int et = g.t - ta * tile_t < tile_t ? g.t - ta * tile_t : tile_t;
              const int eh = g.h - ha * tile_h < tile_h ? g.h - ha * tile_h : tile_h;
              const int ew = g.w - wa * tile_w < tile_w ? g.w - wa * tile_w : tile_w;
              const int n = et * eh * ew;
              if (vc) vc[tile] = n;
              if (slot_row) {
                int s = 0;
                for (int dt = 0; dt < et; ++dt)
                  for (int dh = 0; dh < eh; ++dh)
                    for (int dw = 0; dw < ew; ++dw, ++s)
                      slot_row[(long long)tile * E + s] =
                          (int32_t)(start + ((long long)(ta * tile_t + dt) * g.h + ha * tile_h + dh) * g.w +
                                    wa * tile_w + dw);
                for (; s < E; ++s) slot_row[(long long)tile * E + s] = -1;
              }
              ++tile;
            }
        if (spans) spans[2 * region + 1] = tile;
        ++region;
      }
      start += len;
    }
  }
  return ok();
}

t3d_status tile3d_scatter_packed(const t3d_packed* p, const void* x, void* y, t3d_stream stream) {
  t3d::PackedGeo g;
  T3D_CHECK(check_packed(p, &g));
  T3D_CHECK(check_ptr(x, "x"));
  T3D_CHECK(check_ptr(y, "y"));
  return cuda_status(t3d::launch_scatter_packed(g, x, y, as_stream(stream)), "tile3d_scatter_packed");
}

t3d_status tile3d_gather_packed(const t3d_packed* p, const void* y, void* x, t3d_stream stream) {
  t3d::PackedGeo g;
  T3D_CHECK(check_packed(p, &g));
  T3D_CHECK(check_ptr(y, "y"));
  T3D_CHECK(check_ptr(x, "x"));
  return cuda_status(t3d::launch_gather_packed(g, y, x, as_stream(stream)), "tile3d_gather_packed");
}

t3d_status tile_pool_packed(const t3d_packed* p, const void* y, float* pooled, t3d_stream stream) {
  t3d::PackedGeo g;
  T3D_CHECK(check_packed(p, &g));
  T3D_CHECK(check_ptr(y, "y"));
  T3D_CHECK(check_ptr(pooled, "pooled"));
  return cuda_status(t3d::launch_pool_packed(g, y, pooled, as_stream(stream)), "tile_pool_packed");
}

t3d_status tile3d_scatter_pool_packed(const t3d_packed* p, const void* x, void* y, float* pooled,
                                      t3d_stream stream) {
  t3d::PackedGeo g;
  T3D_CHECK(check_packed(p, &g));
  T3D_CHECK(check_ptr(x, "x"));
  T3D_CHECK(check_ptr(y, "y"));
  T3D_CHECK(check_ptr(pooled, "pooled"));
  return cuda_status(t3d::launch_scatter_pool_packed(g, x, y, pooled, as_stream(stream)),
                     "tile3d_scatter_pool_packed");
}

t3d_status tile_select_packed_capacity(int n_tiles, int mode, int n_prefix, int n_regions,
                                       const int32_t* spans, const double* keep_rates, int* kmax) {
  if (n_tiles < 1 || kmax == nullptr) return fail(T3D_ERR_INVALID, "n_tiles >= 1 and kmax needed");
  t3d::SpanSpec sp;
  T3D_CHECK(check_spans(n_tiles, mode, n_prefix, n_regions, spans, keep_rates, &sp, kmax));
  return ok();
}

size_t tile_select_packed_workspace_size(const t3d_packed* p) {
  t3d::PackedGeo g;
  if (check_packed(p, &g) != T3D_OK) return 0;
  return t3d::select_workspace_bytes(packed_score_geo(g));
}

t3d_status tile_select_packed(const t3d_packed* p, const float* pq, const float* pk, int mode,
                              int n_prefix, int n_regions, const int32_t* spans,
                              const double* keep_rates, int kmax, int32_t* kv_idx,
                              int32_t* kv_cnt, void* workspace, size_t ws_bytes,
                              int32_t* dev_status, t3d_stream stream) {
  (void)dev_status;
  t3d::PackedGeo g;
  T3D_CHECK(check_packed(p, &g));
  t3d::SpanSpec sp;
  int cap = 0;
  T3D_CHECK(check_spans(g.n_tiles, mode, n_prefix, n_regions, spans, keep_rates, &sp, &cap));
  if (kmax < cap || kmax > g.n_tiles)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [%d, n_tiles=%d]", kmax, cap, g.n_tiles);
  T3D_CHECK(check_ptr(pq, "pq"));
  T3D_CHECK(check_ptr(pk, "pk"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  const t3d::Geo sg = packed_score_geo(g);
  const size_t need = t3d::select_workspace_bytes(sg);
  if (ws_bytes < need)
    return fail(T3D_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                ws_bytes, need);
  T3D_CHECK(check_ptr(workspace, "workspace"));
  return cuda_status(t3d::launch_select_spans(sg, pq, pk, sp, kmax, kv_idx, kv_cnt, workspace,
                                              as_stream(stream)),
                     "tile_select_packed");
}

size_t block_sparse_attn_packed_workspace_size(const t3d_packed* p, int kmax) {
  t3d::PackedGeo g;
  if (check_packed(p, &g) != T3D_OK || kmax < 1) return 0;
  return t3d::attn_packed_workspace_bytes(g, kmax);
}

t3d_status block_sparse_attn_fwd_packed(const t3d_packed* p, const void* q, const void* k,
                                        const void* v, void* o, const int32_t* kv_idx,
                                        const int32_t* kv_cnt, int kmax, float softmax_scale,
                                        void* workspace, size_t ws_bytes, int32_t* dev_status,
                                        t3d_stream stream) {
  t3d::PackedGeo g;
  T3D_CHECK(check_packed(p, &g));
  const long long units = (long long)g.n_tiles * (g.E / 64);
  if (units > t3d::kMaxTiles)
    return fail(T3D_ERR_UNSUPPORTED, "%lld 64-row units exceed the supported maximum %d", units,
                t3d::kMaxTiles);
  const double expected = 1.0 / sqrt((double)g.D);
  const double diff = fabs((double)softmax_scale - expected);
  if (!(diff <= fmax(1e-4 * fmax(fabs((double)softmax_scale), expected), 1e-5)))
    return fail(T3D_ERR_INVALID, "softmax_scale=%.8g must be 1/sqrt(D)=%.8g", (double)softmax_scale,
                expected);
  T3D_CHECK(check_ptr(q, "q"));
  T3D_CHECK(check_ptr(k, "k"));
  T3D_CHECK(check_ptr(v, "v"));
  T3D_CHECK(check_ptr(o, "o"));
  T3D_CHECK(check_ptr4(kv_idx, "kv_idx"));
  T3D_CHECK(check_ptr4(kv_cnt, "kv_cnt"));
  if (kmax < 1 || kmax > g.n_tiles)
    return fail(T3D_ERR_INVALID, "kmax=%d must lie in [1, n_tiles=%d]", kmax, g.n_tiles);
  const size_t need = t3d::attn_packed_workspace_bytes(g, kmax);
  if (ws_bytes < need)
    return fail(T3D_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                ws_bytes, need);
  T3D_CHECK(check_ptr(workspace, "workspace"));
  t3d::AttnArgs a{q, k, v, o, kv_idx, kv_cnt, kmax, nullptr, nullptr, softmax_scale,
                  workspace, ws_bytes, dev_status, g_wait_cycles};
  return cuda_status(t3d::launch_attn_packed(g, a, as_stream(stream)),
                     "block_sparse_attn_fwd_packed");
}

}  // extern "C"
