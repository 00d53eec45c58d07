// sa_internal.h -- host-side launchers shared by the C-ABI layer (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sa.h"

namespace sa {

// ---- workspace carving for the decode calls ------------------------------------------
struct DecodePlan {
  int K;      // pages per (sequence, KV head) = budget / P
  int G;      // query heads per KV head
  int n_cta;        // attention CTAs (one per SM, more for very large selections)
  int n_score_cta;  // scoring CTAs (one per SM, more for very long sequences)
  int n_sm;         // streaming multiprocessors of the device
  size_t off_scores, off_sel, off_cnt, off_phys, off_pre, off_part, off_qs, total;
};

bool make_decode_plan(const sa_geom& g, int budget, DecodePlan* plan);

#ifdef SA_TRACE
// the traced build: install the timeline buffer in each translation unit with trace points
void trace_set_score(void* buf);
void trace_set_attend(void* buf);
#endif

// ---- launchers (return the CUDA error of the launch) ----------------------------------
cudaError_t launch_summaries(const sa_geom& g, const void* k_cache, const int32_t* page_table,
                             const int32_t* seq_lens, void* summ, int n_tail,
                             cudaStream_t stream);

// fp8 records [n_pool][Hkv][2 * Dk + 16] (grouped-query head dims 64 and 128)
cudaError_t launch_summaries_fp8(const sa_geom& g, const void* k_cache,
                                 const int32_t* page_table, const int32_t* seq_lens, void* summ8,
                                 int n_tail, cudaStream_t stream);

cudaError_t launch_score_select(const sa_geom& g, const void* q, void* summ, const void* k_cache,
                                int n_tail, const int32_t* page_table, const int32_t* seq_lens,
                                float* scores, int n_cta, int K, int sink_pages,
                                int window_pages, int32_t* sel, int32_t* sel_count,
                                int32_t* sel_phys, int32_t* status, cudaStream_t stream);

// fp8: summ holds fp8 records (2 * Dk + 16 bytes per page and KV head)
cudaError_t launch_score(const sa_geom& g, const void* q, const void* summ,
                         const int32_t* page_table, const int32_t* seq_lens, float* scores,
                         int n_cta, int32_t* status, cudaStream_t stream, bool fp8 = false,
                         const void* k_cache = nullptr, int n_tail = 0);
cudaError_t launch_select(const sa_geom& g, const int32_t* page_table, const int32_t* seq_lens,
                          float* scores, int K, int sink_pages, int window_pages, int32_t* sel,
                          int32_t* sel_count, int32_t* sel_phys, int32_t* status,
                          cudaStream_t stream);

// Latent (MLA) geometry: sign-split queries (workspace, mla_qsplit_bytes) then scoring on
// the tcgen05 tensor cores.
size_t mla_qsplit_bytes(const sa_geom& g);
cudaError_t launch_score_mla(const sa_geom& g, const void* q, const void* summ, void* qs,
                             const int32_t* page_table, const int32_t* seq_lens, float* scores,
                             int32_t* status, cudaStream_t stream);

size_t mla_attend_part_bytes(const sa_geom& g, int sel_stride);
cudaError_t launch_attend_mla(const sa_geom& g, const void* q, const void* kv,
                              const int32_t* page_table, const int32_t* seq_lens,
                              const int32_t* sel, const int32_t* sel_count,
                              const int32_t* sel_phys, int sel_stride, float scale, float* part,
                              float* out, float* lse, int32_t* status, cudaStream_t stream);

int score_ctas(const sa_geom& g, int sms);
bool score_supported(const sa_geom& g);
bool score_supported_fp8(const sa_geom& g);

struct AttendCall {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* sel;
  const int32_t* sel_count;
  const int32_t* sel_phys;  // physical pages of sel (nullable: looked up in page_table)
  int sel_stride;
  float scale;
  float* part;     // states of pairs cut by warp-range boundaries
  int32_t* pre;    // [B*Hkv + 1] pair prefix of units, for the merge kernel
  float* out;
  float* lse;
  int32_t* status;
  int n_cta;
  int counts_from_lens;  // the selection came from this library for these seq_lens
};

// the whole grouped-query decode step in one persistent launch
struct FusedCall {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  void* summ;
  const int32_t* page_table;
  const int32_t* seq_lens;
  int K, s_pages, w_pages, n_tail;
  float scale;
  float* scores;
  int32_t* sel;
  int32_t* sel_count;
  int32_t* sel_phys;
  float* part;
  int32_t* pre;
  float* out;
  float* lse;
  int32_t* status;
  int32_t* counter;  // grid-barrier counter (zeroed on the stream before the launch)
  int n_cta, n_sm;
};

bool fused_supported(const sa_geom& g, int K, int n_sm);
cudaError_t launch_fused(const sa_geom& g, const FusedCall& f, cudaStream_t stream);

int attend_ctas(const sa_geom& g, int K, int sms);
size_t attend_partial_floats(const sa_geom& g, int n_cta);
bool attend_supported(const sa_geom& g);

cudaError_t launch_attend(const sa_geom& g, const AttendCall& c, cudaStream_t stream);

cudaError_t launch_prune(const sa_geom& g, const void* k_cache, const void* v_cache,
                         const int32_t* page_table, const int32_t* seq_lens, const uint8_t* keep,
                         const int32_t* free_pages, int64_t n_free, void* k_dst, void* v_dst,
                         void* summ, int32_t* new_page_table, int32_t* new_seq_lens,
                         int32_t* pos_map, int32_t* logical_len, void* ws, cudaStream_t stream);

size_t prune_workspace_bytes(const sa_geom& g);

// TMA descriptor encoder from the driver (resolved once through the runtime).
bool encode_rows_tmap(void* tmap_out, const void* base, uint64_t inner_elems, uint64_t rows,
                      uint32_t box_inner, uint32_t box_rows);
// 3-D descriptor of a [rows][128] bf16 pool: one box = box_rows rows, both 128-byte halves.
bool encode_rows3_tmap(void* tmap_out, const void* base, uint64_t rows, uint32_t box_rows);

}  // namespace sa
