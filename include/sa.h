/*
 * sa.h -- C ABI of the page-sparse decode library (sm_100a, one GPU).
 *
 * Query-aware top-k page-sparse decode attention over a paged KV cache, plus
 * keep-mask prefix-cache pruning.  The sources describing the method:
 *   [SE]  "SparseEngine" blog post (blog.ontle.kr/blog/332): hook-point paragraph
 *         (Quest chooses, at each decode step, which pages to read from the
 *         current query; OmniKV/DeltaKV reuse one layer's indices at later layers),
 *         physical-vs-logical paragraph (freeing storage vs reading less), and the
 *         Prefix-Cache Pruning paragraph (the kept part stays, the rest is freed,
 *         the conversation-position marker is untouched).
 *   [VX]  "Vortex" summary (gist.science/ja/paper/2606.06453), section 1: KV in
 *         non-contiguous paged boxes; a map hands back "the top pages" without the
 *         caller knowing where they live.
 *   [SC]  SCBench notes (notes.yuuk.io), Tri-shape section: A-shape = attention-sink
 *         tokens + local window; method table: Quest loads part of the KV per step.
 *   [SSA] SubQ/SSA article (news.neo-ai.one/ja/article/2719), SSA section: exact
 *         attention over the chosen positions; FlashAttention paragraph: no
 *         materialised score matrix.
 * The pages never print the formulas.  This library computes the plain method:
 * channel-wise min/max key summaries per page; page score
 * S(b,h,p) = max_{g in group(h)} sum_c max(q_gc*kmax_c, q_gc*kmin_c) in fp32; the
 * budget/P best pages with sink and window pages forced in (ties -> lower page
 * index); exact softmax attention over the selected tokens with split-KV online
 * softmax merged by log-sum-exp.
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises (except sa_workspace_status, which
 *    says so).  bf16 tensors are passed as `const void*` (16-bit bf16 elements).
 *  - Every tensor must be 16-byte aligned and densely packed in the layout given.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued asynchronously on it; calls are capturable in a CUDA graph.
 *  - Argument errors are detected on the host before anything is launched and
 *    returned as a negative sa_status.  Errors only the device can see (an index
 *    out of range, a bounded wait that expired, too few free pages) are OR-ed into
 *    the workspace status word and read with sa_workspace_status().
 *  - Layouts (row-major, last index fastest):
 *      q           [B][Hq][Dk]            bf16
 *      k_cache     [n_pool][Hkv][P][Dk]   bf16   (each (page, head) block contiguous)
 *      v_cache     [n_pool][Hkv][P][Dv]   bf16   (ignored when v_aliases_k: V is then
 *                                                 the first Dv channels of each K row)
 *      summ        [n_pool][Hkv][2][Dk]   bf16   row 0 = min, row 1 = max, indexed by
 *                                                 PHYSICAL page
 *      page_table  [B][max_pages]         int32  logical page -> physical page
 *      seq_lens    [B]                    int32  valid tokens; logical page lp holds
 *                                                 tokens [lp*P, lp*P+P)
 *      sel         [B][Hkv][budget/P]     int32  ascending logical pages, -1 padded
 *      sel_count   [B][Hkv]               int32
 *      out         [B][Hq][Dv]            fp32   lse [B][Hq] fp32 (natural log)
 *  - Supported geometries: grouped-query (v_aliases_k = 0): Dk = Dv in {64, 128},
 *    G = Hq/Hkv in 1..8, Hkv <= 32; latent (v_aliases_k = 1): Hkv = 1, Dk = 576,
 *    Dv = 512, Hq = 128 (its scores and attention are dense contractions and run on
 *    the tcgen05 tensor cores).  P in {16, 32, 64}.  budget, sink, window are token counts,
 *    multiples of P, with sink + window <= budget.  Preconditions not checked on the
 *    device: no NaN/Inf in valid K, V, q; page_table entries of valid pages lie in
 *    [0, n_pool).
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = -1,   /* bad pointer, size, alignment or budget/sink/window */
  SA_ERR_UNSUPPORTED = -2,   /* geometry outside the supported set */
  SA_ERR_WORKSPACE = -3,     /* workspace missing or smaller than the *_workspace_size */
  SA_ERR_CUDA = -4,          /* a CUDA runtime call or a launch failed */
  SA_ERR_DEVICE_CHECK = -5,  /* device saw an out-of-range index (status word only) */
  SA_ERR_TIMEOUT = -6,       /* a bounded device wait expired (status word only) */
  SA_ERR_NO_SPACE = -7       /* prune: fewer free pages than kept pages (status word) */
} sa_status;

/* Problem geometry.  n_pool = number of physical pages in k_cache/v_cache/summ. */
typedef struct {
  int32_t B, Hq, Hkv, Dk, Dv, P, max_pages, n_pool, v_aliases_k;
} sa_geom;

/* Human-readable name of a status code (static string, never NULL). */
const char* sa_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int sa_version(void);

/* ---------------------------------------------------------------------------------
 * Workspace.  Zero it once before first use (sa_workspace_init).  Its first 256 bytes
 * hold the status word, the only part that must start at zero; the rest is scratch that
 * each call writes before it reads it (scores, the selection and its physical pages, the
 * split-KV partial states), so no state carries from one call to the next.  One
 * workspace therefore serves any geometry and budget whose sa_decode_workspace_size it
 * covers.  Calls that use one workspace must not overlap in time (use one per stream, or
 * order the streams).
 * ------------------------------------------------------------------------------ */

/* Bytes needed by sa_select_pages / sa_sparse_decode / sa_attend_selected for this
 * geometry and budget (0 on invalid arguments). */
size_t sa_decode_workspace_size(const sa_geom* g, int budget);

/* Bytes needed by sa_prune_compact (0 on invalid arguments). */
size_t sa_prune_workspace_size(const sa_geom* g);

/* Zero `ws_bytes` bytes of workspace on `stream` (cudaMemsetAsync). */
int sa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns the workspace status word (SA_OK or the first
 * device-detected error) and clears it.  The only call that blocks the host. */
int sa_workspace_status(void* ws, void* stream);

/* ---------------------------------------------------------------------------------
 * (1) Per-page key summaries  [SE hook-point paragraph; VX section 1].
 * For every valid logical page lp < ceil(seq_lens[b]/P) of every sequence, every KV
 * head h and channel c: summ[page_table[b][lp]][h][0][c] = min over the page's
 * valid tokens (t < seq_lens[b]) of K[t][h][c], row 1 = max.  Signed zeros order
 * -0 < +0.  Pages referenced by no sequence are not written.  Bit-exact.
 * ------------------------------------------------------------------------------ */
int sa_page_summaries(const sa_geom* g, const void* k_cache, const int32_t* page_table,
                      const int32_t* seq_lens, void* summ, void* stream);

/* Same as sa_page_summaries restricted to the last `n_tail_pages` valid pages of
 * each sequence: the decode-time update after new tokens were appended (one new
 * token per step -> n_tail_pages = 1).  n_tail_pages >= 1. */
int sa_update_summaries(const sa_geom* g, const void* k_cache, const int32_t* page_table,
                        const int32_t* seq_lens, int n_tail_pages, void* summ, void* stream);

/* ---------------------------------------------------------------------------------
 * (2) Page scoring alone  [SE hook-point paragraph (Quest): the query-aware page
 * bound].  scores[b][h][p] = max over the G query heads g of KV head h of
 * sum_c max(q[b][h*G+g][c] * kmax_c, q[b][h*G+g][c] * kmin_c) for p < n_b, with
 * (kmin, kmax) = summ[page_table[b][p]][h]; -inf for n_b <= p < max_pages.  fp32,
 * summation order unspecified.  q: [B][Hq][Dk] bf16, 16-byte aligned; summ as written
 * by sa_page_summaries; scores: [B][Hkv][max_pages] fp32, caller-owned.  ws: for the
 * grouped-query geometries any workspace of at least 256 bytes (only its status word is
 * used: page-table entries outside [0, n_pool) set SA_ERR_DEVICE_CHECK there and score
 * as 0); for the latent geometry at least sa_decode_workspace_size(g, any budget) bytes
 * (it also holds the sign-split query rows the tensor cores read).  Asynchronous on
 * `stream`; argument errors are returned before any launch.
 * ------------------------------------------------------------------------------ */
int sa_page_scores(const sa_geom* g, const void* q, const void* summ,
                   const int32_t* page_table, const int32_t* seq_lens, float* scores, void* ws,
                   size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (2)+(3) Page scoring and top-k selection  [SE hook-point paragraph (Quest);
 * VX section 1 ("top pages"); SC Tri-shape section (sink + local window)].
 * K = budget/P pages per (sequence, KV head).  If n_b = ceil(seq_lens[b]/P) <= K
 * all n_b pages are selected.  Otherwise pages [0, sink/P) and [n_b - window/P, n_b)
 * are forced in and the K - sink/P - window/P highest-scoring other pages join them
 * (equal fp32 scores -> lower page index).  sel gets the ascending page list, -1
 * after sel_count entries.  `scores` (nullable, [B][Hkv][max_pages] fp32) receives
 * S for p < n_b and -inf beyond.  Selection is deterministic.
 * Decode-time refresh: with n_tail_refresh in 1..16 (k_cache then required), the
 * summaries of the last n_tail_refresh pages of every sequence are first recomputed
 * from k_cache -- the pages that just received appended tokens -- and written to
 * summ, exactly as sa_update_summaries would; 0 leaves summ untouched.
 * sel_phys (nullable, [B][Hkv][budget/P] int32) receives page_table[b][sel[b][h][i]]
 * for each selected entry (-1 after sel_count): handing it to sa_attend_selected
 * saves that call one dependent page-table lookup.
 * ------------------------------------------------------------------------------ */
int sa_select_pages(const sa_geom* g, const void* q, void* summ, const int32_t* page_table,
                    const int32_t* seq_lens, int budget, int sink, int window,
                    const void* k_cache, int n_tail_refresh, int32_t* sel, int32_t* sel_count,
                    int32_t* sel_phys, float* scores, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (4) Sparse decode: selection as above, then exact attention over the tokens of
 * the selected pages gathered through the page table  [VX section 1; SSA section;
 * FlashAttention paragraph]:
 *   x_t = scale * q . k_t over valid tokens t of the selected pages of KV head
 *   hq / G;  out[b][hq] = sum_t softmax(x)_t v_t;  lse[b][hq] = log sum_t exp(x_t).
 * A sequence with seq_len 0 gives out = 0, lse = -inf.  bf16 inputs, fp32
 * accumulation.  sel_out / sel_count_out (nullable) receive the selection;
 * n_tail_refresh as in sa_select_pages (a refreshed page must not be shared with another
 * sequence of the same call: that sequence's scoring may read either version of its
 * summary).
 * ------------------------------------------------------------------------------ */
int sa_sparse_decode(const sa_geom* g, const void* q, const void* k_cache, const void* v_cache,
                     void* summ, const int32_t* page_table, const int32_t* seq_lens, int budget,
                     int sink, int window, int n_tail_refresh, float scale, float* out,
                     float* lse, int32_t* sel_out, int32_t* sel_count_out, void* ws,
                     size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * sa_sparse_decode_fused: the same outputs as sa_sparse_decode (grouped-query geometry,
 * V not aliasing K) from one persistent launch instead of four kernels: page scoring
 * with the n_tail_refresh refresh, the selection, the gathered attention and the merge
 * run as phases of one grid of one CTA per SM, all resident (cooperative launch), handed
 * over by grid barriers on a counter in the workspace header (zeroed on `stream` before
 * the launch; a barrier that waits longer than 2 s sets SA_ERR_TIMEOUT).  The selection
 * is bit-identical to sa_sparse_decode's; the attention is the same computation with the
 * same work split.  SA_ERR_UNSUPPORTED where one CTA per SM cannot cover the geometry
 * or the phases' shared memory does not fit.  Arguments and workspace as for
 * sa_sparse_decode.  [VX section 1; SSA section; FlashAttention paragraph: the method
 * of (4), in one launch.]
 * ------------------------------------------------------------------------------ */
int sa_sparse_decode_fused(const sa_geom* g, const void* q, const void* k_cache,
                           const void* v_cache, void* summ, const int32_t* page_table,
                           const int32_t* seq_lens, int budget, int sink, int window,
                           int n_tail_refresh, float scale, float* out, float* lse,
                           int32_t* sel_out, int32_t* sel_count_out, void* ws, size_t ws_bytes,
                           void* stream);

/* ---------------------------------------------------------------------------------
 * fp8 summaries rounded outward (grouped-query geometry only; others return
 * SA_ERR_UNSUPPORTED)  [SE hook-point paragraph: quantised KV (KIVI) listed next to
 * Quest; the pages give no format].  Per (physical page, KV head) a record of
 * 2*Dk + 16 bytes replaces the 4*Dk bytes of bf16 min/max:
 *   summ8 [n_pool][Hkv][2*Dk + 16] uint8 = [Dk codes of min][Dk codes of max][int8 e]
 *   [15 zero bytes].
 * Codes are OCP FP8 E4M3 ("fn": bias 7, max finite 448, 0x7F/0xFF NaN never written):
 * the min row rounded toward -inf and the max row toward +inf, of the bf16 min/max of
 * sa_page_summaries scaled by 2^-e, where e is the smallest integer with
 * max|value| * 2^-e <= 448 (e = 0 for an all-zero record).  Zero is the code 0x00.
 * Decoded, code * 2^e <= kmin and >= kmax, so the page bound over the records is still
 * an upper bound of every q.k on the page (never below the bf16 bound; equal to it
 * when every scaled min/max is an exact code).  Bit-exact.
 * sa_summary_fp8_record_bytes: 2*Dk + 16 for a supported geometry, else 0.
 * sa_page_scores_fp8: the bound S of (2) over decoded records, fp32 (codes widened to
 * bf16 exactly; products exact; fp32 accumulation), -inf beyond each sequence.
 * sa_sparse_decode_fp8: sa_sparse_decode with the selection scored over fp8 records;
 * attention still reads the bf16 K and V.  n_tail_refresh (0..16) re-encodes the
 * newest pages' records from k_cache first, exactly as sa_update_summaries_fp8 would
 * (inside the scoring kernel; a refreshed page must not be shared with another sequence
 * of the call).  Argument rules and workspace as for sa_sparse_decode (summ8 16-byte
 * aligned).
 * ------------------------------------------------------------------------------ */
size_t sa_summary_fp8_record_bytes(const sa_geom* g);
int sa_page_summaries_fp8(const sa_geom* g, const void* k_cache, const int32_t* page_table,
                          const int32_t* seq_lens, void* summ8, void* stream);
int sa_update_summaries_fp8(const sa_geom* g, const void* k_cache, const int32_t* page_table,
                            const int32_t* seq_lens, int n_tail_pages, void* summ8,
                            void* stream);
int sa_page_scores_fp8(const sa_geom* g, const void* q, const void* summ8,
                       const int32_t* page_table, const int32_t* seq_lens, float* scores,
                       void* ws, size_t ws_bytes, void* stream);
int sa_sparse_decode_fp8(const sa_geom* g, const void* q, const void* k_cache,
                         const void* v_cache, void* summ8, const int32_t* page_table,
                         const int32_t* seq_lens, int budget, int sink, int window,
                         int n_tail_refresh, float scale, float* out, float* lse,
                         int32_t* sel_out, int32_t* sel_count_out, void* ws, size_t ws_bytes,
                         void* stream);

/* ---------------------------------------------------------------------------------
 * Allocation-free sparse decode.  The pages have no counterpart to this call: it is an
 * engineering variant of sa_sparse_decode for callers that cannot hand the library a
 * workspace.  Arguments, results and argument errors are those of sa_sparse_decode
 * without (ws, ws_bytes); the workspace is instead a scratch array inside the library,
 * a static device variable of SA_STATIC_SCRATCH_BYTES bytes per device, so nothing is
 * allocated at run time (no cudaMalloc, no allocating library routine).
 *  - Limit: a geometry and budget whose sa_decode_workspace_size exceeds
 *    SA_STATIC_SCRATCH_BYTES is rejected with SA_ERR_WORKSPACE before any launch
 *    (Llama-3.1-8B geometry, batch 8, 128K tokens, budget 2048 needs about 8 MB).
 *    The latent geometry at 16 sequences of 64K tokens with budget 2048 needs about
 *    38 MB and is therefore refused; 8 such sequences fit.
 *  - Setup: the first call on a device, with that device current, looks the scratch up
 *    with cudaGetSymbolAddress (a host-side lookup, no device work); make that first
 *    call before any stream capture.  The address is cached per device for the life of
 *    the process: resetting a device (cudaDeviceReset) is not supported afterwards.
 *  - Zeroing: the module's load zero-fills the scratch.  Every call clears the status
 *    word on `stream` before its first launch; the rest of the scratch is written by
 *    each call before it is read, as in a workspace, so nothing else carries over.
 *  - status_out (nullable, device int32): receives, on `stream`, the bit-OR of the
 *    device-detected errors of this call ((1 << -status) per error, 0 when none).  With
 *    status_out NULL those errors are dropped: the next call clears the word, and no
 *    other call reads the scratch's status.
 *  - Concurrency: the scratch is shared by all calls on a device.  Calls that can
 *    overlap in time (other streams, other host threads) race on it; the caller must
 *    serialise them.
 * ------------------------------------------------------------------------------ */
#define SA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
int sa_sparse_decode_noalloc(const sa_geom* g, const void* q, const void* k_cache,
                             const void* v_cache, void* summ, const int32_t* page_table,
                             const int32_t* seq_lens, int budget, int sink, int window,
                             int n_tail_refresh, float scale, float* out, float* lse,
                             int32_t* sel_out, int32_t* sel_count_out, int32_t* status_out,
                             void* stream);

/* Attention over a given selection (sel [B][Hkv][sel_stride], ascending logical
 * pages, sel_count [B][Hkv] <= sel_stride): the reuse of one layer's selected
 * indices at later layers [SE hook-point paragraph, OmniKV/DeltaKV].  `budget` for
 * the workspace size is sel_stride * P.  sel_phys (nullable) holds the physical page
 * of each entry as written by sa_select_pages; passing it also states that the
 * selection was made by sa_select_pages for these seq_lens with budget
 * sel_stride * P, so that sel_count[b][h] == min(ceil(seq_lens[b] / P), sel_stride)
 * (the kernel then derives the counts from seq_lens and starts earlier; it reads
 * seq_lens before the previous kernel of the stream has finished, so seq_lens must be
 * unchanged since that selection).  Without sel_phys the page table and sel_count
 * are read. */
int sa_attend_selected(const sa_geom* g, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* page_table, const int32_t* seq_lens, const int32_t* sel,
                       const int32_t* sel_count, const int32_t* sel_phys, int sel_stride,
                       float scale, float* out, float* lse, void* ws, size_t ws_bytes,
                       void* stream);

/* ---------------------------------------------------------------------------------
 * (5) Prefix-cache pruning  [SE physical-vs-logical and Prefix-Cache Pruning
 * paragraphs]: physical removal of the tokens keep[b][t] == 0.
 * For each session b in order, the kept valid tokens (t < seq_lens[b], increasing t)
 * are numbered i = 0.. L'_b - 1 and kept token i (K and V rows of every KV head) is
 * copied to page free_pages[off_b + i/P], slot i % P, with off_b = sum over b' < b
 * of ceil(L'_b'/P).  Outputs: new_page_table[b][j] = free_pages[off_b + j] for
 * j < ceil(L'_b/P), else -1; new_seq_lens[b] = L'_b; logical_len[b] = seq_lens[b]
 * (the position marker is kept); pos_map[b][i] = original position of kept token
 * i, -1 for i >= L'_b; summ of every new page; padding slots of a partial last page
 * are zero.  Old pages are read, never written: the caller returns them to its
 * allocator.  keep [B][max_pages*P] uint8, pos_map [B][max_pages*P] int32.
 * k_dst/v_dst may be k_cache/v_cache; free pages must not be referenced by
 * page_table.  If n_free < sum_b ceil(L'_b/P) nothing is written and the status
 * word reports SA_ERR_NO_SPACE.  Bit-exact.
 * ------------------------------------------------------------------------------ */
int sa_prune_compact(const sa_geom* g, const void* k_cache, const void* v_cache,
                     const int32_t* page_table, const int32_t* seq_lens, const uint8_t* keep,
                     const int32_t* free_pages, int64_t n_free, void* k_dst, void* v_dst,
                     void* summ, int32_t* new_page_table, int32_t* new_seq_lens,
                     int32_t* pos_map, int32_t* logical_len, void* ws, size_t ws_bytes,
                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
