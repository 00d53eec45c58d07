// sa_capi.cu -- the exported C ABI: argument validation, workspace planning, dispatch.
//
// Every entry point validates its arguments on the host before launching anything,
// never allocates and never synchronises (sa_workspace_status excepted).  The
// operations themselves are documented in include/sa.h.
#include <cudaTypedefs.h>

#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"

#define SA_EXPORT extern "C" __attribute__((visibility("default")))

namespace sa {

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

static bool is_gqa(const sa_geom& g) {
  return !g.v_aliases_k && (g.Dk == 64 || g.Dk == 128) && g.Dv == g.Dk && g.Hq % g.Hkv == 0 &&
         g.Hq / g.Hkv >= 1 && g.Hq / g.Hkv <= 8 && g.Hkv <= 32 && attend_supported(g) &&
         score_supported(g);
}

static bool is_latent(const sa_geom& g) {
  return g.v_aliases_k == 1 && g.Hkv == 1 && g.Dk == 576 && g.Dv == 512 && g.Hq == 128;
}

// basic shape sanity shared by all calls
static int check_geom(const sa_geom* g) {
  if (!g) return SA_ERR_INVALID_ARG;
  if (g->B < 1 || g->Hq < 1 || g->Hkv < 1 || g->max_pages < 1 || g->n_pool < 1)
    return SA_ERR_INVALID_ARG;
  if (g->Hq % g->Hkv) return SA_ERR_INVALID_ARG;
  if (!(g->P == 16 || g->P == 32 || g->P == 64)) return SA_ERR_UNSUPPORTED;
  if ((int64_t)g->max_pages * g->P > (int64_t)1 << 30) return SA_ERR_UNSUPPORTED;
  if ((int64_t)g->n_pool * g->Hkv * g->P >= ((int64_t)1 << 31)) return SA_ERR_UNSUPPORTED;
  if (!is_gqa(*g) && !is_latent(*g)) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

static int check_budget(const sa_geom& g, int budget, int sink, int window) {
  if (budget < g.P || budget % g.P || sink < 0 || sink % g.P || window < 0 || window % g.P)
    return SA_ERR_INVALID_ARG;
  if (sink + window > budget) return SA_ERR_INVALID_ARG;
  if (budget / g.P > 65536) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

bool make_decode_plan(const sa_geom& g, int budget, DecodePlan* plan) {
  DecodePlan p{};
  p.K = budget / g.P;
  p.G = g.Hq / g.Hkv;
  p.n_sm = sm_count();
  p.n_cta = attend_ctas(g, p.K, p.n_sm);
  p.n_score_cta = score_ctas(g, p.n_sm);
  size_t off = 256;  // status header
  p.off_scores = off;
  off += up256((size_t)g.B * g.Hkv * g.max_pages * 4);
  p.off_sel = off;
  off += up256((size_t)g.B * g.Hkv * p.K * 4);
  p.off_cnt = off;
  off += up256((size_t)g.B * g.Hkv * 4);
  p.off_phys = off;
  off += up256((size_t)g.B * g.Hkv * p.K * 4);
  p.off_pre = off;
  off += up256(((size_t)g.B * g.Hkv + 1) * 4);
  p.off_part = off;
  // split states: per warp range (GQA) or per 256-token chunk (latent)
  off += up256(is_latent(g) ? mla_attend_part_bytes(g, p.K) : attend_partial_floats(g, p.n_cta) * 4);
  p.off_qs = off;  // latent geometry: sign-split query rows for the tensor-core scoring
  if (is_latent(g)) off += up256(mla_qsplit_bytes(g));
  p.total = off;
  *plan = p;
  return true;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows][inner] (inner contiguous), box [box_rows][box_inner],
// 128-byte swizzle (box_inner * 2 must be 128).
bool encode_rows_tmap(void* tmap_out, const void* base, uint64_t inner_elems, uint64_t rows,
                      uint32_t box_inner, uint32_t box_rows) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner_elems, rows};
  cuuint64_t strides[1] = {inner_elems * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(static_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view of a [rows][128] bf16 pool as (64 channels, rows, 2 halves of a row): one box
// of {64, box_rows, 2} lands as [half][row][64] with the 128-byte swizzle, the layout of
// two 2-D boxes of {64, box_rows}.
bool encode_rows3_tmap(void* tmap_out, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {256, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(static_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

}  // namespace sa

using namespace sa;

SA_EXPORT const char* sa_status_string(int status) {
  switch (status) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported geometry";
    case SA_ERR_WORKSPACE: return "workspace missing or too small";
    case SA_ERR_CUDA: return "CUDA error";
    case SA_ERR_DEVICE_CHECK: return "device-side index check failed";
    case SA_ERR_TIMEOUT: return "bounded device wait expired";
    case SA_ERR_NO_SPACE: return "not enough free pages";
    default: return "unknown status";
  }
}

SA_EXPORT int sa_version(void) { return 10000; }

SA_EXPORT size_t sa_decode_workspace_size(const sa_geom* g, int budget) {
  if (check_geom(g) != SA_OK || budget < g->P || budget % g->P) return 0;
  DecodePlan p;
  make_decode_plan(*g, budget, &p);
  return p.total;
}

SA_EXPORT size_t sa_prune_workspace_size(const sa_geom* g) {
  if (check_geom(g) != SA_OK) return 0;
  return prune_workspace_bytes(*g);
}

SA_EXPORT int sa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) return SA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

SA_EXPORT int sa_workspace_status(void* ws, void* stream) {
  if (!ws) return SA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SA_ERR_CUDA;
  int32_t bits = 0;
  if (cudaMemcpy(&bits, ws, sizeof bits, cudaMemcpyDeviceToHost) != cudaSuccess)
    return SA_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(int32_t)) != cudaSuccess) return SA_ERR_CUDA;
  const int order[] = {SA_ERR_DEVICE_CHECK, SA_ERR_TIMEOUT, SA_ERR_NO_SPACE, SA_ERR_CUDA};
  for (int st : order)
    if (bits & (1 << -st)) return st;
  return SA_OK;
}

SA_EXPORT int sa_page_summaries(const sa_geom* g, const void* k_cache, const int32_t* page_table,
                                const int32_t* seq_lens, void* summ, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!k_cache || !page_table || !seq_lens || !summ) return SA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(summ)) return SA_ERR_INVALID_ARG;
  return cuda_status(launch_summaries(*g, k_cache, page_table, seq_lens, summ, 0,
                                      static_cast<cudaStream_t>(stream)));
}

SA_EXPORT int sa_update_summaries(const sa_geom* g, const void* k_cache, const int32_t* page_table,
                                  const int32_t* seq_lens, int n_tail_pages, void* summ,
                                  void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!k_cache || !page_table || !seq_lens || !summ || n_tail_pages < 1)
    return SA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(summ)) return SA_ERR_INVALID_ARG;
  if (n_tail_pages > g->max_pages) n_tail_pages = g->max_pages;
  return cuda_status(launch_summaries(*g, k_cache, page_table, seq_lens, summ, n_tail_pages,
                                      static_cast<cudaStream_t>(stream)));
}

// scoring + selection into (sel, cnt); shared by select and decode
static int run_select(const sa_geom& g, const DecodePlan& plan, uint8_t* w, const void* q,
                      void* summ, const void* k_cache, int n_tail, const int32_t* page_table,
                      const int32_t* seq_lens, int sink, int window, int32_t* sel, int32_t* cnt,
                      int32_t* phys, float* scores, cudaStream_t s) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(w);
  if (is_latent(g)) {
    // newest pages' summaries first, then tensor-core scoring, then the selection
    if (n_tail > 0) {
      const int st = cuda_status(launch_summaries(g, k_cache, page_table, seq_lens, summ, n_tail, s));
      if (st != SA_OK) return st;
    }
    int st = cuda_status(launch_score_mla(g, q, summ, w + plan.off_qs, page_table, seq_lens,
                                          scores, &hdr->status_bits, s));
    if (st != SA_OK) return st;
    return cuda_status(launch_select(g, page_table, seq_lens, scores, plan.K, sink / g.P,
                                     window / g.P, sel, cnt, phys, &hdr->status_bits, s));
  }
  if (!is_gqa(g)) return SA_ERR_UNSUPPORTED;
  return cuda_status(launch_score_select(
      g, q, summ, n_tail > 0 ? k_cache : nullptr, n_tail, page_table, seq_lens, scores,
      plan.n_score_cta, plan.K, sink / g.P, window / g.P, sel,
      cnt, phys, &hdr->status_bits, s));
}

static int run_attend(const sa_geom& g, const DecodePlan& plan, uint8_t* w, const void* q,
                      const void* k_cache, const void* v_cache, const int32_t* page_table,
                      const int32_t* seq_lens, const int32_t* sel, const int32_t* cnt,
                      const int32_t* sel_phys, int sel_stride, float scale, float* out,
                      float* lse, cudaStream_t s) {
  if (is_latent(g)) {
    WsHeader* h = reinterpret_cast<WsHeader*>(w);
    return cuda_status(launch_attend_mla(g, q, k_cache, page_table, seq_lens, sel, cnt, sel_phys,
                                         sel_stride, scale, reinterpret_cast<float*>(w + plan.off_part),
                                         out, lse, &h->status_bits, s));
  }
  WsHeader* hdr = reinterpret_cast<WsHeader*>(w);
  AttendCall c;
  c.q = q;
  c.k_cache = k_cache;
  c.v_cache = v_cache;
  c.page_table = page_table;
  c.seq_lens = seq_lens;
  c.sel = sel;
  c.sel_count = cnt;
  c.sel_phys = sel_phys;
  c.sel_stride = sel_stride;
  c.scale = scale;
  c.part = reinterpret_cast<float*>(w + plan.off_part);
  c.pre = reinterpret_cast<int32_t*>(w + plan.off_pre);
  c.out = out;
  c.lse = lse;
  c.status = &hdr->status_bits;
  c.n_cta = plan.n_cta;
  c.counts_from_lens = sel_phys != nullptr;
  return cuda_status(launch_attend(g, c, s));
}

SA_EXPORT int sa_page_scores(const sa_geom* g, const void* q, const void* summ,
                             const int32_t* page_table, const int32_t* seq_lens, float* scores,
                             void* ws, size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!q || !summ || !page_table || !seq_lens || !scores) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(summ)) return SA_ERR_INVALID_ARG;
  if (is_latent(*g)) {
    if (!ws || ws_bytes < 256 + mla_qsplit_bytes(*g) || !aligned16(ws)) return SA_ERR_WORKSPACE;
    WsHeader* hdr = static_cast<WsHeader*>(ws);
    return cuda_status(launch_score_mla(*g, q, summ, static_cast<uint8_t*>(ws) + 256, page_table,
                                        seq_lens, scores, &hdr->status_bits,
                                        static_cast<cudaStream_t>(stream)));
  }
  if (!is_gqa(*g)) return SA_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < 256 || !aligned16(ws)) return SA_ERR_WORKSPACE;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  return cuda_status(launch_score(*g, q, summ, page_table, seq_lens, scores,
                                  score_ctas(*g, sm_count()), &hdr->status_bits,
                                  static_cast<cudaStream_t>(stream)));
}

SA_EXPORT int sa_select_pages(const sa_geom* g, const void* q, void* summ,
                              const int32_t* page_table, const int32_t* seq_lens, int budget,
                              int sink, int window, const void* k_cache, int n_tail_refresh,
                              int32_t* sel, int32_t* sel_count, int32_t* sel_phys,
                              float* scores, void* ws, size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if ((st = check_budget(*g, budget, sink, window)) != SA_OK) return st;
  if (!q || !summ || !page_table || !seq_lens || !sel || !sel_count) return SA_ERR_INVALID_ARG;
  if (n_tail_refresh < 0 || n_tail_refresh > 16 || (n_tail_refresh > 0 && !k_cache))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(summ) || (k_cache && !aligned16(k_cache)))
    return SA_ERR_INVALID_ARG;
  if ((size_t)g->max_pages * 4 > 200 * 1024) return SA_ERR_UNSUPPORTED;
  if (!is_gqa(*g) && !is_latent(*g)) return SA_ERR_UNSUPPORTED;
  DecodePlan plan;
  make_decode_plan(*g, budget, &plan);
  if (!ws || ws_bytes < plan.total || !aligned16(ws)) return SA_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* sc = scores ? scores : reinterpret_cast<float*>(w + plan.off_scores);
  int32_t* ph = sel_phys ? sel_phys : reinterpret_cast<int32_t*>(w + plan.off_phys);
  return run_select(*g, plan, w, q, summ, k_cache, n_tail_refresh, page_table, seq_lens, sink,
                    window, sel, sel_count, ph, sc, static_cast<cudaStream_t>(stream));
}

SA_EXPORT int sa_attend_selected(const sa_geom* g, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* page_table,
                                 const int32_t* seq_lens, const int32_t* sel,
                                 const int32_t* sel_count, const int32_t* sel_phys,
                                 int sel_stride, float scale, float* out, float* lse, void* ws,
                                 size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!is_gqa(*g) && !is_latent(*g)) return SA_ERR_UNSUPPORTED;
  if (sel_stride < 1 || sel_stride > 65536) return SA_ERR_INVALID_ARG;
  if (is_latent(*g) && !aligned16(out)) return SA_ERR_INVALID_ARG;
  if (!q || !k_cache || !page_table || !seq_lens || !sel || !sel_count || !out || !lse)
    return SA_ERR_INVALID_ARG;
  if (!g->v_aliases_k && !v_cache) return SA_ERR_INVALID_ARG;
  const void* vc = g->v_aliases_k ? k_cache : v_cache;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(vc)) return SA_ERR_INVALID_ARG;
  DecodePlan plan;
  make_decode_plan(*g, sel_stride * g->P, &plan);
  if (!ws || ws_bytes < plan.total || !aligned16(ws)) return SA_ERR_WORKSPACE;
  return run_attend(*g, plan, static_cast<uint8_t*>(ws), q, k_cache, vc, page_table, seq_lens,
                    sel, sel_count, sel_phys, sel_stride, scale, out, lse,
                    static_cast<cudaStream_t>(stream));
}

SA_EXPORT int sa_sparse_decode(const sa_geom* g, const void* q, const void* k_cache,
                               const void* v_cache, void* summ, const int32_t* page_table,
                               const int32_t* seq_lens, int budget, int sink, int window,
                               int n_tail_refresh, float scale, float* out, float* lse,
                               int32_t* sel_out, int32_t* sel_count_out, void* ws,
                               size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if ((st = check_budget(*g, budget, sink, window)) != SA_OK) return st;
  if (!q || !k_cache || !summ || !page_table || !seq_lens || !out || !lse)
    return SA_ERR_INVALID_ARG;
  if (n_tail_refresh < 0 || n_tail_refresh > 16) return SA_ERR_INVALID_ARG;
  if (!g->v_aliases_k && !v_cache) return SA_ERR_INVALID_ARG;
  const void* vc = g->v_aliases_k ? k_cache : v_cache;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(vc) || !aligned16(summ))
    return SA_ERR_INVALID_ARG;
  if ((size_t)g->max_pages * 4 > 200 * 1024) return SA_ERR_UNSUPPORTED;
  if (!is_gqa(*g) && !is_latent(*g)) return SA_ERR_UNSUPPORTED;
  if (is_latent(*g) && !aligned16(out)) return SA_ERR_INVALID_ARG;
  DecodePlan plan;
  make_decode_plan(*g, budget, &plan);
  if (!ws || ws_bytes < plan.total || !aligned16(ws)) return SA_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + plan.off_sel);
  int32_t* cnt = sel_count_out ? sel_count_out : reinterpret_cast<int32_t*>(w + plan.off_cnt);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = run_select(*g, plan, w, q, summ, k_cache, n_tail_refresh, page_table, seq_lens, sink,
                  window, sel, cnt, reinterpret_cast<int32_t*>(w + plan.off_phys),
                  reinterpret_cast<float*>(w + plan.off_scores), s);
  if (st != SA_OK) return st;
  return run_attend(*g, plan, w, q, k_cache, vc, page_table, seq_lens, sel, cnt,
                    reinterpret_cast<int32_t*>(w + plan.off_phys), plan.K, scale, out, lse, s);
}
SA_EXPORT int sa_sparse_decode_fused(const sa_geom* g, const void* q, const void* k_cache,
                                     const void* v_cache, void* summ, const int32_t* page_table,
                                     const int32_t* seq_lens, int budget, int sink, int window,
                                     int n_tail_refresh, float scale, float* out, float* lse,
                                     int32_t* sel_out, int32_t* sel_count_out, void* ws,
                                     size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if ((st = check_budget(*g, budget, sink, window)) != SA_OK) return st;
  if (!q || !k_cache || !v_cache || !summ || !page_table || !seq_lens || !out || !lse)
    return SA_ERR_INVALID_ARG;
  if (n_tail_refresh < 0 || n_tail_refresh > 16) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(summ))
    return SA_ERR_INVALID_ARG;
  if ((size_t)g->max_pages * 4 > 200 * 1024) return SA_ERR_UNSUPPORTED;
  if (!is_gqa(*g) || g->v_aliases_k) return SA_ERR_UNSUPPORTED;
  DecodePlan plan;
  make_decode_plan(*g, budget, &plan);
  if (!ws || ws_bytes < plan.total || !aligned16(ws)) return SA_ERR_WORKSPACE;
  if (!fused_supported(*g, plan.K, plan.n_sm)) return SA_ERR_UNSUPPORTED;
  uint8_t* w = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(w);
  FusedCall f;
  f.q = q;
  f.k_cache = k_cache;
  f.v_cache = v_cache;
  f.summ = summ;
  f.page_table = page_table;
  f.seq_lens = seq_lens;
  f.K = plan.K;
  f.s_pages = sink / g->P;
  f.w_pages = window / g->P;
  f.n_tail = n_tail_refresh;
  f.scale = scale;
  f.scores = reinterpret_cast<float*>(w + plan.off_scores);
  f.sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + plan.off_sel);
  f.sel_count = sel_count_out ? sel_count_out : reinterpret_cast<int32_t*>(w + plan.off_cnt);
  f.sel_phys = reinterpret_cast<int32_t*>(w + plan.off_phys);
  f.part = reinterpret_cast<float*>(w + plan.off_part);
  f.pre = reinterpret_cast<int32_t*>(w + plan.off_pre);
  f.out = out;
  f.lse = lse;
  f.status = &hdr->status_bits;
  f.counter = &hdr->pad[0];
  f.n_cta = plan.n_sm;
  f.n_sm = plan.n_sm;
  const cudaError_t e = launch_fused(*g, f, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorInvalidConfiguration)
    return SA_ERR_UNSUPPORTED;
  return cuda_status(e);
}

#ifdef SA_TRACE
SA_EXPORT int sa_trace_set(void* device_buf) {
  trace_set_score(device_buf);
  trace_set_attend(device_buf);
  return cuda_status(cudaGetLastError());
}
#endif

// ---- fp8 summaries rounded outward (grouped-query geometry) ---------------------------

SA_EXPORT size_t sa_summary_fp8_record_bytes(const sa_geom* g) {
  if (check_geom(g) != SA_OK || !is_gqa(*g) || !score_supported_fp8(*g)) return 0;
  return 2 * (size_t)g->Dk + 16;
}

SA_EXPORT int sa_page_summaries_fp8(const sa_geom* g, const void* k_cache,
                                    const int32_t* page_table, const int32_t* seq_lens,
                                    void* summ8, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!is_gqa(*g) || !score_supported_fp8(*g)) return SA_ERR_UNSUPPORTED;
  if (!k_cache || !page_table || !seq_lens || !summ8) return SA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(summ8)) return SA_ERR_INVALID_ARG;
  return cuda_status(launch_summaries_fp8(*g, k_cache, page_table, seq_lens, summ8, 0,
                                          static_cast<cudaStream_t>(stream)));
}

SA_EXPORT int sa_update_summaries_fp8(const sa_geom* g, const void* k_cache,
                                      const int32_t* page_table, const int32_t* seq_lens,
                                      int n_tail_pages, void* summ8, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!is_gqa(*g) || !score_supported_fp8(*g)) return SA_ERR_UNSUPPORTED;
  if (!k_cache || !page_table || !seq_lens || !summ8 || n_tail_pages < 1)
    return SA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(summ8)) return SA_ERR_INVALID_ARG;
  if (n_tail_pages > g->max_pages) n_tail_pages = g->max_pages;
  return cuda_status(launch_summaries_fp8(*g, k_cache, page_table, seq_lens, summ8,
                                          n_tail_pages, static_cast<cudaStream_t>(stream)));
}

SA_EXPORT int sa_page_scores_fp8(const sa_geom* g, const void* q, const void* summ8,
                                 const int32_t* page_table, const int32_t* seq_lens,
                                 float* scores, void* ws, size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!is_gqa(*g) || !score_supported_fp8(*g)) return SA_ERR_UNSUPPORTED;
  if (!q || !summ8 || !page_table || !seq_lens || !scores) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(summ8)) return SA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256 || !aligned16(ws)) return SA_ERR_WORKSPACE;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  return cuda_status(launch_score(*g, q, summ8, page_table, seq_lens, scores,
                                  score_ctas(*g, sm_count()), &hdr->status_bits,
                                  static_cast<cudaStream_t>(stream), true));
}

SA_EXPORT int sa_sparse_decode_fp8(const sa_geom* g, const void* q, const void* k_cache,
                                   const void* v_cache, void* summ8, const int32_t* page_table,
                                   const int32_t* seq_lens, int budget, int sink, int window,
                                   int n_tail_refresh, float scale, float* out, float* lse,
                                   int32_t* sel_out, int32_t* sel_count_out, void* ws,
                                   size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!is_gqa(*g) || !score_supported_fp8(*g)) return SA_ERR_UNSUPPORTED;
  if ((st = check_budget(*g, budget, sink, window)) != SA_OK) return st;
  if (!q || !k_cache || !v_cache || !summ8 || !page_table || !seq_lens || !out || !lse)
    return SA_ERR_INVALID_ARG;
  if (n_tail_refresh < 0 || n_tail_refresh > 16) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(summ8))
    return SA_ERR_INVALID_ARG;
  if ((size_t)g->max_pages * 4 > 200 * 1024) return SA_ERR_UNSUPPORTED;
  DecodePlan plan;
  make_decode_plan(*g, budget, &plan);
  if (!ws || ws_bytes < plan.total || !aligned16(ws)) return SA_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* status = &reinterpret_cast<WsHeader*>(w)->status_bits;
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + plan.off_sel);
  int32_t* cnt = sel_count_out ? sel_count_out : reinterpret_cast<int32_t*>(w + plan.off_cnt);
  int32_t* phys = reinterpret_cast<int32_t*>(w + plan.off_phys);
  float* scores = reinterpret_cast<float*>(w + plan.off_scores);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // fp8 scoring (which first re-encodes the newest pages' records from K), the selection
  // and the attention over bf16 K and V
  if ((st = cuda_status(launch_score(*g, q, summ8, page_table, seq_lens, scores,
                                     plan.n_score_cta, status, s, true,
                                     n_tail_refresh > 0 ? k_cache : nullptr,
                                     n_tail_refresh))) != SA_OK)
    return st;
  if ((st = cuda_status(launch_select(*g, page_table, seq_lens, scores, plan.K, sink / g->P,
                                      window / g->P, sel, cnt, phys, status, s))) != SA_OK)
    return st;
  return run_attend(*g, plan, w, q, k_cache, v_cache, page_table, seq_lens, sel, cnt, phys,
                    plan.K, scale, out, lse, s);
}

namespace sa {
// Scratch of sa_sparse_decode_noalloc: a static device variable, one per device.
static __device__ __align__(256) uint8_t g_static_scratch[SA_STATIC_SCRATCH_BYTES];
constexpr int kMaxDevices = 64;
static void* g_scratch_addr[kMaxDevices];
static std::mutex g_scratch_mu;

// Device address of the current device's scratch, looked up on the first call for that
// device.  The module's load zero-fills the array, so no clearing is needed here.
static int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return SA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SA_OK;
}
}  // namespace sa

SA_EXPORT int sa_sparse_decode_noalloc(const sa_geom* g, const void* q, const void* k_cache,
                                       const void* v_cache, void* summ,
                                       const int32_t* page_table, const int32_t* seq_lens,
                                       int budget, int sink, int window, int n_tail_refresh,
                                       float scale, float* out, float* lse, int32_t* sel_out,
                                       int32_t* sel_count_out, int32_t* status_out,
                                       void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if ((st = check_budget(*g, budget, sink, window)) != SA_OK) return st;
  if (sa_decode_workspace_size(g, budget) > SA_STATIC_SCRATCH_BYTES) return SA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = static_scratch(&scratch)) != SA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // a fresh status word (and abort flag) for this call, before its first launch, so that a
  // call that failed half-way leaves nothing behind for the next one
  if (cudaMemsetAsync(scratch, 0, 2 * sizeof(int32_t), s) != cudaSuccess) return SA_ERR_CUDA;
  st = sa_sparse_decode(g, q, k_cache, v_cache, summ, page_table, seq_lens, budget, sink, window,
                        n_tail_refresh, scale, out, lse, sel_out, sel_count_out, scratch,
                        SA_STATIC_SCRATCH_BYTES, stream);
  if (st != SA_OK) return st;
  if (status_out &&
      cudaMemcpyAsync(status_out, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return SA_ERR_CUDA;
  return SA_OK;
}

SA_EXPORT int sa_prune_compact(const sa_geom* g, const void* k_cache, const void* v_cache,
                               const int32_t* page_table, const int32_t* seq_lens,
                               const uint8_t* keep, const int32_t* free_pages, int64_t n_free,
                               void* k_dst, void* v_dst, void* summ, int32_t* new_page_table,
                               int32_t* new_seq_lens, int32_t* pos_map, int32_t* logical_len,
                               void* ws, size_t ws_bytes, void* stream) {
  int st = check_geom(g);
  if (st != SA_OK) return st;
  if (!k_cache || !page_table || !seq_lens || !keep || !k_dst || !summ || !new_page_table ||
      !new_seq_lens || !pos_map || !logical_len)
    return SA_ERR_INVALID_ARG;
  if (n_free < 0 || (n_free > 0 && !free_pages)) return SA_ERR_INVALID_ARG;
  if (!g->v_aliases_k && (!v_cache || !v_dst)) return SA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(k_dst) || !aligned16(summ) || !aligned16(keep))
    return SA_ERR_INVALID_ARG;
  if (!g->v_aliases_k && (!aligned16(v_cache) || !aligned16(v_dst))) return SA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < prune_workspace_bytes(*g) || !aligned16(ws)) return SA_ERR_WORKSPACE;
  return cuda_status(launch_prune(*g, k_cache, v_cache, page_table, seq_lens, keep, free_pages,
                                  n_free, k_dst, v_dst, summ, new_page_table, new_seq_lens,
                                  pos_map, logical_len, ws, static_cast<cudaStream_t>(stream)));
}
