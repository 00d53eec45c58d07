/*
 * sa_oracle.c -- plain, slow, obviously-correct CPU oracle for query-aware
 * page-sparse decode over a paged KV cache, and for prefix-cache pruning.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may call this code.  It shares nothing with the CUDA library
 * (no headers, helpers, tables or kernels) and it never calls it.
 *
 * What each function follows (sources are the pages on the method; where they
 * stay silent, the reading taken is written next to the code):
 *   - "SparseEngine" blog (blog.ontle.kr/blog/332), hook-point paragraph: Quest
 *     picks, at each decode step, the pages to read from the current query; the
 *     same page distinguishes physical removal (frees storage) from logical
 *     selection (reads less), and its Prefix-Cache Pruning paragraph says the
 *     dropped part is freed while the conversation-position marker stays.
 *   - "Vortex" summary (gist.science/ja/paper/2606.06453), section 1: KV lives in
 *     non-contiguous paged boxes and a map hands back the top pages.
 *   - SCBench notes (notes.yuuk.io), Tri-shape section: A-shape = sink tokens +
 *     local window, the pattern forced into every selection here.
 *   - The pages never write the formulas out; this oracle takes the method's
 *     plain definition: channel-wise min/max key summaries per page; page bound
 *     sum_c max(q_c*kmax_c, q_c*kmin_c) per KV head with the GQA query heads
 *     max-reduced; top-k under a token budget with forced sink/window pages and
 *     lowest-page-index tie-break; exact softmax attention over the selected
 *     tokens; keep-mask compaction into fresh pages keeping the logical length.
 *
 * Parity status: every function here is pinned by the CPU tests against closed
 * forms, library routines, invariants or brute force (see tests/test_oracle_pins.py).
 *
 * Conventions:
 *   bf16 values are passed as uint16 bit patterns; every arithmetic step is done
 *   in double (a bf16 value converts to double exactly, and so does the product
 *   of two of them).
 *   k_cache [n_pool][Hkv][P][Dk], v_cache [n_pool][Hkv][P][Dv] (V may alias the
 *   first Dv channels of K), summ [n_pool][Hkv][2][Dk] with row 0 = min, row 1 = max,
 *   page_table [B][max_pages], seq_lens [B], q [B][Hq][Dk].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

typedef struct {
    int32_t B, Hq, Hkv, Dk, Dv, P, max_pages, n_pool, v_aliases_k;
} oracle_geom;

static double bf(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Strict "a < b" on bf16 values, with -0 ordered before +0 so that min and max
 * have one well-defined bit pattern (reading: the pages give no rule for signed
 * zeros; the summary stores one of the page's own values, and -0 < +0 picks it). */
static int bf_less(uint16_t a, uint16_t b) {
    double da = bf(a), db = bf(b);
    if (da < db) return 1;
    if (da > db) return 0;
    return (a & 0x8000u) && !(b & 0x8000u);
}

static int64_t n_pages_of(int32_t len, int32_t P) { return ((int64_t)len + P - 1) / P; }

static const uint16_t* k_row(const oracle_geom* g, const uint16_t* k_cache, int64_t phys,
                             int h, int t) {
    return k_cache + (((phys * g->Hkv + h) * g->P + t) * (int64_t)g->Dk);
}

static const uint16_t* v_row(const oracle_geom* g, const uint16_t* k_cache,
                             const uint16_t* v_cache, int64_t phys, int h, int t) {
    if (g->v_aliases_k) return k_row(g, k_cache, phys, h, t);
    return v_cache + (((phys * g->Hkv + h) * g->P + t) * (int64_t)g->Dv);
}

/* (1) Per-page key summaries: for every page a sequence uses, every KV head and
 * channel, the min and the max of K over the page's valid tokens (t < seq_len).
 * Pages no sequence references are left untouched. */
ORACLE_API void oracle_page_summaries(const oracle_geom* g, const uint16_t* k_cache,
                                      const int32_t* page_table, const int32_t* seq_lens,
                                      uint16_t* summ) {
    for (int b = 0; b < g->B; ++b) {
        int32_t L = seq_lens[b];
        int64_t nb = n_pages_of(L, g->P);
        for (int64_t lp = 0; lp < nb; ++lp) {
            int64_t phys = page_table[(int64_t)b * g->max_pages + lp];
            int valid = (int)((L - lp * g->P) < g->P ? (L - lp * g->P) : g->P);
            for (int h = 0; h < g->Hkv; ++h) {
                uint16_t* out = summ + ((phys * g->Hkv + h) * 2) * (int64_t)g->Dk;
                for (int c = 0; c < g->Dk; ++c) {
                    uint16_t mn = k_row(g, k_cache, phys, h, 0)[c];
                    uint16_t mx = mn;
                    for (int t = 1; t < valid; ++t) {
                        uint16_t x = k_row(g, k_cache, phys, h, t)[c];
                        if (bf_less(x, mn)) mn = x;
                        if (bf_less(mx, x)) mx = x;
                    }
                    out[c] = mn;
                    out[g->Dk + c] = mx;
                }
            }
        }
    }
}

/* (2) Page scores: u_g(p) = sum_c max(q_gc * kmax_c, q_gc * kmin_c) for every query
 * head g of KV head h's group, S(b,h,p) = max_g u_g(p); in double, over the
 * sequence's n_b logical pages, -inf beyond them.  Group of KV head h = query
 * heads [h*G, (h+1)*G). */
ORACLE_API void oracle_page_scores(const oracle_geom* g, const uint16_t* q,
                                   const uint16_t* summ, const int32_t* page_table,
                                   const int32_t* seq_lens, double* scores) {
    int G = g->Hq / g->Hkv;
    for (int b = 0; b < g->B; ++b) {
        int64_t nb = n_pages_of(seq_lens[b], g->P);
        for (int h = 0; h < g->Hkv; ++h) {
            double* srow = scores + ((int64_t)b * g->Hkv + h) * g->max_pages;
            for (int64_t lp = 0; lp < g->max_pages; ++lp) {
                if (lp >= nb) { srow[lp] = -INFINITY; continue; }
                int64_t phys = page_table[(int64_t)b * g->max_pages + lp];
                const uint16_t* kmin = summ + ((phys * g->Hkv + h) * 2) * (int64_t)g->Dk;
                const uint16_t* kmax = kmin + g->Dk;
                double best = -INFINITY;
                for (int gi = 0; gi < G; ++gi) {
                    const uint16_t* qg = q + ((int64_t)b * g->Hq + h * G + gi) * g->Dk;
                    double u = 0.0;
                    for (int c = 0; c < g->Dk; ++c) {
                        double a = bf(qg[c]) * bf(kmax[c]);
                        double d = bf(qg[c]) * bf(kmin[c]);
                        u += (a > d) ? a : d;
                    }
                    if (u > best) best = u;
                }
                srow[lp] = best;
            }
        }
    }
}

/* (2') fp8 summaries rounded outward, and the page bound over them.  The SparseEngine
 * blog's hook-point paragraph lists quantised KV (KIVI) next to Quest; the pages give
 * no format.  Reading taken: OCP FP8 E4M3 ("fn": bias 7, no infinities, 0x7F/0xFF
 * NaN) codes of the min row rounded toward -inf and of the max row rounded toward
 * +inf, after scaling the (page, KV head) record by 2^-e, e the smallest integer with
 * max|value| * 2^-e <= 448 (the largest finite code).  The decoded record then still
 * brackets every key of the page, so the bound stays an upper bound.
 * Record: [Dk codes of min][Dk codes of max][int8 e][15 zero bytes]. */

/* Value of an E4M3 code from the format's definition. */
static double e4m3_value(int code) {
    int s = (code >> 7) & 1, E = (code >> 3) & 15, m = code & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0)
        v = ldexp((double)m, -9);          /* subnormal: (m/8) * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, E - 7);
    return s ? -v : v;
}

ORACLE_API void oracle_e4m3_values(double* out) {
    for (int c = 0; c < 256; ++c) out[c] = e4m3_value(c);
}

/* The tightest finite code >= x (up) or <= x (down), found by trying all of them; a
 * zero result is the code 0x00.  0x7F (NaN) when no finite code qualifies. */
static uint8_t e4m3_outward(double x, int up) {
    int best = -1;
    double bv = 0.0;
    for (int c = 0; c < 256; ++c) {
        double v = e4m3_value(c);
        if (isnan(v)) continue;
        if (up ? !(v >= x) : !(v <= x)) continue;
        if (best < 0 || (up ? v < bv : v > bv)) {
            best = c;
            bv = v;
        }
    }
    if (best < 0) return 0x7F;
    return bv == 0.0 ? 0x00 : (uint8_t)best;
}

ORACLE_API uint8_t oracle_e4m3_outward(double x, int up) { return e4m3_outward(x, up); }

/* smallest integer e with A * 2^-e <= 448; 0 when A == 0 */
static int fp8_exponent(double A) {
    if (A == 0.0) return 0;
    int e = -400;
    while (ldexp(A, -e) > 448.0) ++e;
    return e;
}

/* Encode the bf16 summaries of every page a sequence uses into fp8 records. */
ORACLE_API void oracle_encode_fp8(const oracle_geom* g, const uint16_t* summ,
                                  const int32_t* page_table, const int32_t* seq_lens,
                                  uint8_t* summ8) {
    const int64_t rec = 2 * (int64_t)g->Dk + 16;
    for (int b = 0; b < g->B; ++b) {
        int64_t nb = n_pages_of(seq_lens[b], g->P);
        for (int64_t lp = 0; lp < nb; ++lp) {
            int64_t phys = page_table[(int64_t)b * g->max_pages + lp];
            for (int h = 0; h < g->Hkv; ++h) {
                const uint16_t* kmin = summ + ((phys * g->Hkv + h) * 2) * (int64_t)g->Dk;
                const uint16_t* kmax = kmin + g->Dk;
                uint8_t* out = summ8 + (phys * g->Hkv + h) * rec;
                double A = 0.0;
                for (int c = 0; c < g->Dk; ++c) {
                    if (fabs(bf(kmin[c])) > A) A = fabs(bf(kmin[c]));
                    if (fabs(bf(kmax[c])) > A) A = fabs(bf(kmax[c]));
                }
                int e = fp8_exponent(A);
                for (int c = 0; c < g->Dk; ++c) {
                    out[c] = e4m3_outward(ldexp(bf(kmin[c]), -e), 0);
                    out[g->Dk + c] = e4m3_outward(ldexp(bf(kmax[c]), -e), 1);
                }
                memset(out + 2 * g->Dk, 0, 16);
                out[2 * g->Dk] = (uint8_t)(int8_t)e;
            }
        }
    }
}

/* The page bound of (2) over decoded fp8 records: kmin_c = value(code) * 2^e, the same
 * for kmax; in double (exact: a bf16 times a 4-bit-significand value scaled by 2^e). */
ORACLE_API void oracle_page_scores_fp8(const oracle_geom* g, const uint16_t* q,
                                       const uint8_t* summ8, const int32_t* page_table,
                                       const int32_t* seq_lens, double* scores) {
    int G = g->Hq / g->Hkv;
    const int64_t rec = 2 * (int64_t)g->Dk + 16;
    for (int b = 0; b < g->B; ++b) {
        int64_t nb = n_pages_of(seq_lens[b], g->P);
        for (int h = 0; h < g->Hkv; ++h) {
            double* srow = scores + ((int64_t)b * g->Hkv + h) * g->max_pages;
            for (int64_t lp = 0; lp < g->max_pages; ++lp) {
                if (lp >= nb) { srow[lp] = -INFINITY; continue; }
                int64_t phys = page_table[(int64_t)b * g->max_pages + lp];
                const uint8_t* r = summ8 + (phys * g->Hkv + h) * rec;
                int e = (int8_t)r[2 * g->Dk];
                double best = -INFINITY;
                for (int gi = 0; gi < G; ++gi) {
                    const uint16_t* qg = q + ((int64_t)b * g->Hq + h * G + gi) * g->Dk;
                    double u = 0.0;
                    for (int c = 0; c < g->Dk; ++c) {
                        double lo = ldexp(e4m3_value(r[c]), e);
                        double hi = ldexp(e4m3_value(r[g->Dk + c]), e);
                        double a = bf(qg[c]) * hi;
                        double d = bf(qg[c]) * lo;
                        u += (a > d) ? a : d;
                    }
                    if (u > best) best = u;
                }
                srow[lp] = best;
            }
        }
    }
}

typedef struct { double s; int32_t p; } cand;

/* higher score first; equal scores -> lower logical page index first */
static int cand_cmp(const void* x, const void* y) {
    const cand* a = (const cand*)x;
    const cand* b = (const cand*)y;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->p < b->p) ? -1 : (a->p > b->p);
}

/* (3) Top-k page selection with forced pages.  K = budget/P pages per (sequence,
 * KV head).  If n_b <= K every page is selected.  Otherwise the sink pages
 * [0, sink/P) and the window pages [n_b - window/P, n_b) are always selected and
 * the k_top = K - sink/P - window/P best remaining pages join them (ties ->
 * lower page index).  Output: ascending logical page ids in sel[b][h][0..count),
 * -1 after them.  Returns 0, or -1 on invalid arguments. */
ORACLE_API int oracle_select_pages(const oracle_geom* g, const double* scores,
                                   const int32_t* seq_lens, int budget, int sink, int window,
                                   int32_t* sel, int32_t* sel_count) {
    if (budget % g->P || sink % g->P || window % g->P || sink + window > budget) return -1;
    int K = budget / g->P, s = sink / g->P, w = window / g->P, k_top = K - s - w;
    unsigned char* chosen = (unsigned char*)calloc((size_t)g->max_pages, 1);
    cand* cs = (cand*)malloc(sizeof(cand) * (size_t)(g->max_pages > 0 ? g->max_pages : 1));
    for (int b = 0; b < g->B; ++b) {
        int64_t nb = n_pages_of(seq_lens[b], g->P);
        for (int h = 0; h < g->Hkv; ++h) {
            const double* srow = scores + ((int64_t)b * g->Hkv + h) * g->max_pages;
            int32_t* out = sel + ((int64_t)b * g->Hkv + h) * K;
            memset(chosen, 0, (size_t)g->max_pages);
            if (nb <= K) {
                for (int64_t p = 0; p < nb; ++p) chosen[p] = 1;
            } else {
                int nc = 0;
                for (int64_t p = 0; p < nb; ++p) {
                    if (p < s || p >= nb - w) chosen[p] = 1;
                    else { cs[nc].s = srow[p]; cs[nc].p = (int32_t)p; ++nc; }
                }
                qsort(cs, (size_t)nc, sizeof(cand), cand_cmp);
                for (int i = 0; i < k_top && i < nc; ++i) chosen[cs[i].p] = 1;
            }
            int cnt = 0;
            for (int64_t p = 0; p < nb; ++p)
                if (chosen[p]) out[cnt++] = (int32_t)p;
            sel_count[(int64_t)b * g->Hkv + h] = cnt;
            for (int i = cnt; i < K; ++i) out[i] = -1;
        }
    }
    free(chosen);
    free(cs);
    return 0;
}

/* (4) Exact attention over the selected tokens: for query head hq of sequence b
 * (KV head h = hq / G), logits x_t = scale * sum_c q_c k_tc over the valid tokens of
 * the selected pages, o = sum_t softmax(x)_t v_t, lse = log sum_t exp(x_t).  A
 * sequence with no token gives o = 0 and lse = -inf.  All in double. */
ORACLE_API void oracle_attend(const oracle_geom* g, const uint16_t* q, const uint16_t* k_cache,
                              const uint16_t* v_cache, const int32_t* page_table,
                              const int32_t* seq_lens, const int32_t* sel,
                              const int32_t* sel_count, int K, double scale,
                              double* out, double* lse) {
    int G = g->Hq / g->Hkv;
    int64_t max_tok = (int64_t)K * g->P;
    double* x = (double*)malloc(sizeof(double) * (size_t)(max_tok > 0 ? max_tok : 1));
    int64_t* tp = (int64_t*)malloc(sizeof(int64_t) * (size_t)(max_tok > 0 ? max_tok : 1));
    int* tt = (int*)malloc(sizeof(int) * (size_t)(max_tok > 0 ? max_tok : 1));
    for (int b = 0; b < g->B; ++b) {
        int32_t L = seq_lens[b];
        for (int hq = 0; hq < g->Hq; ++hq) {
            int h = hq / G;
            const uint16_t* qv = q + ((int64_t)b * g->Hq + hq) * g->Dk;
            const int32_t* sl = sel + ((int64_t)b * g->Hkv + h) * K;
            int cnt = sel_count[(int64_t)b * g->Hkv + h];
            int64_t n = 0;
            for (int i = 0; i < cnt; ++i) {
                int64_t lp = sl[i];
                int64_t phys = page_table[(int64_t)b * g->max_pages + lp];
                for (int t = 0; t < g->P && lp * g->P + t < L; ++t) {
                    const uint16_t* kr = k_row(g, k_cache, phys, h, t);
                    double acc = 0.0;
                    for (int c = 0; c < g->Dk; ++c) acc += bf(qv[c]) * bf(kr[c]);
                    x[n] = scale * acc;
                    tp[n] = phys;
                    tt[n] = t;
                    ++n;
                }
            }
            double* o = out + ((int64_t)b * g->Hq + hq) * g->Dv;
            for (int c = 0; c < g->Dv; ++c) o[c] = 0.0;
            if (n == 0) { lse[(int64_t)b * g->Hq + hq] = -INFINITY; continue; }
            double m = x[0];
            for (int64_t i = 1; i < n; ++i) if (x[i] > m) m = x[i];
            double sum = 0.0;
            for (int64_t i = 0; i < n; ++i) sum += exp(x[i] - m);
            for (int64_t i = 0; i < n; ++i) {
                double p = exp(x[i] - m) / sum;
                const uint16_t* vr = v_row(g, k_cache, v_cache, tp[i], h, tt[i]);
                for (int c = 0; c < g->Dv; ++c) o[c] += p * bf(vr[c]);
            }
            lse[(int64_t)b * g->Hq + hq] = m + log(sum);
        }
    }
    free(x);
    free(tp);
    free(tt);
}

/* Dense softmax attention over a contiguous token array (no pages): q [G][Dk],
 * k [L][Dk], v [L][Dv].  Used only to pin oracle_attend at budget = all pages. */
ORACLE_API void oracle_dense_attend(int L, int Dk, int Dv, int G, const uint16_t* q,
                                    const uint16_t* k, const uint16_t* v, double scale,
                                    double* out, double* lse) {
    double* x = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int gi = 0; gi < G; ++gi) {
        double* o = out + (int64_t)gi * Dv;
        for (int c = 0; c < Dv; ++c) o[c] = 0.0;
        if (L == 0) { lse[gi] = -INFINITY; continue; }
        for (int t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int c = 0; c < Dk; ++c) acc += bf(q[(int64_t)gi * Dk + c]) * bf(k[(int64_t)t * Dk + c]);
            x[t] = scale * acc;
        }
        double m = x[0];
        for (int t = 1; t < L; ++t) if (x[t] > m) m = x[t];
        double sum = 0.0;
        for (int t = 0; t < L; ++t) sum += exp(x[t] - m);
        for (int t = 0; t < L; ++t) {
            double p = exp(x[t] - m) / sum;
            for (int c = 0; c < Dv; ++c) o[c] += p * bf(v[(int64_t)t * Dv + c]);
        }
        lse[gi] = m + log(sum);
    }
    free(x);
}

/* (5) Prefix-cache pruning by keep-mask compaction.
 * For each session b in order: the kept tokens t < L_b (keep[b][t] != 0), in
 * increasing t, are numbered i = 0, 1, ...; kept token i moves (all KV heads, K and
 * V) to fresh page free_pages[off_b + i / P], slot i % P, where off_b is the number of
 * fresh pages sessions 0..b-1 used (ceil(L'_b' / P) each).  Outputs:
 *   new_page_table[b][j] = free_pages[off_b + j] for j < ceil(L'_b/P), else -1
 *   new_seq_lens[b] = L'_b,  logical_len[b] = L_b (the position marker is kept)
 *   pos_map[b][i] = original position of kept token i, -1 for i >= L'_b
 *   summ[...] of every new page (min/max over its L' valid tokens)
 *   padding slots of a partial last page are written as zero.
 * The old pages are not touched (the caller frees them).  keep and pos_map rows
 * hold max_pages * P entries.  Returns the number of fresh pages used, or -1 when
 * n_free is too small (nothing is written then). */
ORACLE_API int64_t oracle_prune_compact(const oracle_geom* g, const uint16_t* k_cache,
                                        const uint16_t* v_cache, const int32_t* page_table,
                                        const int32_t* seq_lens, const uint8_t* keep,
                                        const int32_t* free_pages, int64_t n_free,
                                        uint16_t* k_dst, uint16_t* v_dst, uint16_t* summ,
                                        int32_t* new_page_table, int32_t* new_seq_lens,
                                        int32_t* pos_map, int32_t* logical_len) {
    int64_t width = (int64_t)g->max_pages * g->P;
    int64_t need = 0;
    for (int b = 0; b < g->B; ++b) {
        int64_t kept = 0;
        for (int64_t t = 0; t < seq_lens[b]; ++t) kept += keep[b * width + t] ? 1 : 0;
        need += n_pages_of((int32_t)kept, g->P);
    }
    if (need > n_free) return -1;

    int64_t off = 0;
    for (int b = 0; b < g->B; ++b) {
        int32_t L = seq_lens[b];
        int64_t i = 0;
        for (int64_t t = 0; t < L; ++t) {
            if (!keep[b * width + t]) continue;
            int64_t lp = t / g->P;
            int st = (int)(t % g->P);
            int64_t src = page_table[(int64_t)b * g->max_pages + lp];
            int64_t dst = free_pages[off + i / g->P];
            int dt = (int)(i % g->P);
            for (int h = 0; h < g->Hkv; ++h) {
                memcpy(k_dst + ((dst * g->Hkv + h) * g->P + dt) * (int64_t)g->Dk,
                       k_row(g, k_cache, src, h, st), sizeof(uint16_t) * (size_t)g->Dk);
                if (!g->v_aliases_k)
                    memcpy(v_dst + ((dst * g->Hkv + h) * g->P + dt) * (int64_t)g->Dv,
                           v_cache + ((src * g->Hkv + h) * g->P + st) * (int64_t)g->Dv,
                           sizeof(uint16_t) * (size_t)g->Dv);
            }
            pos_map[b * width + i] = (int32_t)t;
            ++i;
        }
        int64_t kept = i;
        int64_t np = n_pages_of((int32_t)kept, g->P);
        for (int64_t j = i; j < width; ++j) pos_map[b * width + j] = -1;
        for (int64_t j = 0; j < g->max_pages; ++j)
            new_page_table[(int64_t)b * g->max_pages + j] = (j < np) ? free_pages[off + j] : -1;
        /* zero the padding slots of a partial last page */
        if (kept % g->P) {
            int64_t dst = free_pages[off + np - 1];
            for (int h = 0; h < g->Hkv; ++h)
                for (int t = (int)(kept % g->P); t < g->P; ++t) {
                    memset(k_dst + ((dst * g->Hkv + h) * g->P + t) * (int64_t)g->Dk, 0,
                           sizeof(uint16_t) * (size_t)g->Dk);
                    if (!g->v_aliases_k)
                        memset(v_dst + ((dst * g->Hkv + h) * g->P + t) * (int64_t)g->Dv, 0,
                               sizeof(uint16_t) * (size_t)g->Dv);
                }
        }
        new_seq_lens[b] = (int32_t)kept;
        logical_len[b] = L;
        off += np;
    }
    /* summaries of the new pages, from the compacted pool */
    oracle_page_summaries(g, k_dst, new_page_table, new_seq_lens, summ);
    return need;
}
