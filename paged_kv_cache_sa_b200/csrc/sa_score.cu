// sa_score.cu -- page scoring (the query-aware page bound) fused with top-k selection.
//
// Method ("SparseEngine" blog, hook-point paragraph: Quest chooses the pages to read at
// each decode step from the current query; Vortex summary, section 1: hand back the
// top pages; SCBench notes, Tri-shape section: sink tokens + local window always kept):
//   S(b,h,p) = max over the query heads g of KV head h of
//   u_g(p)   = sum_c max(q_gc * kmax_c, q_gc * kmin_c),
// then per (sequence, KV head) the sink and window pages plus the best remaining pages
// up to budget/P (equal scores -> lower page index), as an ascending list.
//
// Scoring.  Because kmax >= kmin, max(q*kmax, q*kmin) = max(q,0)*kmax + min(q,0)*kmin
// exactly, so u = [kmin | kmax] . [min(q,0) | max(q,0)], a contraction of length 2*Dk.
// Every bf16 x bf16 product is exact in fp32; accumulation is fp32.  The G <= 8 query
// heads are the N=8 side of an m16n8k16 tensor-core tile and 16 pages its M side.
// A fragments come straight from HBM: each lane reads 16-byte vectors of two summary
// rows and the contraction's channel order is permuted so that each vector lands in
// the fragment slots of the lane that loaded it (the query side uses the same order,
// so the sum is unchanged).  One load instruction covers 64 contiguous bytes of 8 rows,
// so every sector fetched is used.  The GQA max is a register max + two shuffles.
//
// Decode-time summary refresh.  When asked, the warp whose 16-page tile holds a
// sequence's newest page first recomputes that page's min/max from K (the page that
// received the appended token) and scores the fresh summary.
//
// Selection.  Each CTA scores 128 pages of one (sequence, KV head); the last CTA to
// finish for that pair (an atomic arrival counter, no waiting) turns the scores into
// order-preserving 32-bit keys in shared memory (forced pages get key 0, below every
// real score) and runs an MSB-first 8-bit radix select (4 passes, warp-aggregated
// shared-memory histograms, one warp scans the 256 bins).  That gives the exact key T
// of the k-th best candidate and how many keys equal to T are needed; a final pass
// marks forced pages, keys > T and the lowest-index keys == T, and two block scans
// write the ascending list.  Deterministic.  HBM-bound: bytes per (page, KV head) =
// 2 * Dk * 2 (summary) + 4 (page-table entry).
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kPagesPerCta = 16 * kScoreWarps;

template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < NT / 32 ? warp_tot[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += u;
    }
    if (lane < NT / 32) warp_tot[lane] = wi - wv;  // exclusive warp offsets
    if (lane == 31) warp_tot[NT / 32] = wi;        // block total
  }
  __syncthreads();
  const int res = warp_tot[warp] + incl - v;
  *total = warp_tot[NT / 32];
  __syncthreads();
  return res;
}

// Radix select of one (sequence, KV head) by the whole CTA; see the file comment.
template <int NT>
__device__ void block_select(const float* srow, int nb, int K, int s_pages, int w_pages,
                             uint32_t* keys, int32_t* out, int32_t* cnt_out,
                             const int32_t* ptab, int32_t* phys_out) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sh_bin, sh_above;
  __shared__ int warp_tot[NT / 32 + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (nb <= K) {
    for (int i = tid; i < K; i += NT) {
      out[i] = i < nb ? i : -1;
      if (phys_out) phys_out[i] = i < nb ? ptab[i] : -1;
    }
    if (tid == 0) *cnt_out = nb;
    return;
  }
  const int wbeg = nb - w_pages;
  for (int p = tid; p < nb; p += NT)
    keys[p] = (p < s_pages || p >= wbeg) ? 0u : f32_order_key(__ldcg(srow + p));
  __syncthreads();

  uint32_t prefix = 0, pmask = 0;
  int k_rem = K - s_pages - w_pages;     // < number of candidates here
  if (k_rem == 0) prefix = 0xFFFFFFFFu;  // forced pages only: no key reaches T
#pragma unroll 1
  for (int shift = 24; shift >= 0 && k_rem > 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int p = tid; p < nb; p += NT) {
      const uint32_t key = keys[p];
      if ((key & pmask) == prefix) {
        const uint32_t bin = (key >> shift) & 255u;
        const unsigned act = __activemask();
        const unsigned peers = __match_any_sync(act, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[lane * 8 + i];
        tot += c[i];
      }
      uint32_t incl = tot;  // keys in bins of lanes >= this lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t u = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += u;
      }
      uint32_t run = incl - tot;  // keys in higher bins than this lane's
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (run < (uint32_t)k_rem && run + c[i] >= (uint32_t)k_rem) {
          sh_bin = lane * 8 + i;
          sh_above = run;
        }
        run += c[i];
      }
    }
    __syncthreads();
    prefix |= sh_bin << shift;
    pmask |= 255u << shift;
    k_rem -= (int)sh_above;
    __syncthreads();
  }
  const uint32_t T = prefix;

  const int seg = (nb + NT - 1) / NT;
  const int beg = min(nb, tid * seg), end = min(nb, beg + seg);
  int n_eq = 0;
  for (int p = beg; p < end; ++p) n_eq += keys[p] == T;
  int tot;
  const int eq_rank = block_excl_scan<NT>(n_eq, warp_tot, &tot);
  int n_sel = 0;
  for (int p = beg, er = eq_rank; p < end; ++p) {
    const uint32_t key = keys[p];
    const bool is_eq = key == T;
    n_sel += (p < s_pages || p >= wbeg) || key > T || (is_eq && er < k_rem);
    er += is_eq;
  }
  int pos = block_excl_scan<NT>(n_sel, warp_tot, &tot);
  for (int p = beg, er = eq_rank; p < end; ++p) {
    const uint32_t key = keys[p];
    const bool is_eq = key == T;
    if ((p < s_pages || p >= wbeg) || key > T || (is_eq && er < k_rem)) {
      out[pos] = p;
      if (phys_out) phys_out[pos] = ptab[p];
      ++pos;
    }
    er += is_eq;
  }
  for (int i = tot + tid; i < K; i += NT) {
    out[i] = -1;
    if (phys_out) phys_out[i] = -1;
  }
  if (tid == 0) *cnt_out = tot;
}

// Recompute the summary of one (physical page, KV head) from K (one warp).
template <int D>
__device__ __forceinline__ void warp_refresh_summary(const uint4* __restrict__ k_cache,
                                                     uint4* __restrict__ summ, int phys, int h,
                                                     int Hkv, int P, int valid, int lane) {
  constexpr int CPR = D / 8;     // 8 or 16 chunks per row
  constexpr int RPI = 32 / CPR;  // rows per warp iteration
  const int c = lane % CPR;
  const uint4* blk = k_cache + ((size_t)phys * Hkv + h) * P * CPR;
  uint4 mn = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
  uint4 mx = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
  for (int t = lane / CPR; t < valid; t += RPI) {
    const uint4 v = __ldcg(blk + (size_t)t * CPR + c);
    const uint32_t k0 = bf2_key(v.x), k1 = bf2_key(v.y), k2 = bf2_key(v.z), k3 = bf2_key(v.w);
    mn.x = __vmins2(mn.x, k0); mn.y = __vmins2(mn.y, k1);
    mn.z = __vmins2(mn.z, k2); mn.w = __vmins2(mn.w, k3);
    mx.x = __vmaxs2(mx.x, k0); mx.y = __vmaxs2(mx.y, k1);
    mx.z = __vmaxs2(mx.z, k2); mx.w = __vmaxs2(mx.w, k3);
  }
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
    mn.x = __vmins2(mn.x, __shfl_xor_sync(0xffffffffu, mn.x, off));
    mn.y = __vmins2(mn.y, __shfl_xor_sync(0xffffffffu, mn.y, off));
    mn.z = __vmins2(mn.z, __shfl_xor_sync(0xffffffffu, mn.z, off));
    mn.w = __vmins2(mn.w, __shfl_xor_sync(0xffffffffu, mn.w, off));
    mx.x = __vmaxs2(mx.x, __shfl_xor_sync(0xffffffffu, mx.x, off));
    mx.y = __vmaxs2(mx.y, __shfl_xor_sync(0xffffffffu, mx.y, off));
    mx.z = __vmaxs2(mx.z, __shfl_xor_sync(0xffffffffu, mx.z, off));
    mx.w = __vmaxs2(mx.w, __shfl_xor_sync(0xffffffffu, mx.w, off));
  }
  uint4* out = summ + ((size_t)phys * Hkv + h) * 2 * CPR;
  if (lane < CPR) {
    __stcg(out + c, make_uint4(bf2_key(mn.x), bf2_key(mn.y), bf2_key(mn.z), bf2_key(mn.w)));
    __stcg(out + CPR + c, make_uint4(bf2_key(mx.x), bf2_key(mx.y), bf2_key(mx.z), bf2_key(mx.w)));
  }
}

struct ScoreArgs {
  const uint16_t* q;
  uint4* summ;
  const uint4* k_cache;  // non-null: refresh the last n_tail pages' summaries first
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;       // [B][Hkv][max_pages]
  uint32_t* arrivals;  // [B][Hkv] CTA arrival counters (zero between calls)
  int32_t* sel;        // [B][Hkv][K]
  int32_t* sel_count;  // [B][Hkv]
  int32_t* sel_phys;   // [B][Hkv][K] physical pages of the selection (nullable)
  int32_t* status;
  int Hq, Hkv, P, max_pages, n_pool, K, s_pages, w_pages, n_tail;
};

template <int D>
__global__ void __launch_bounds__(kScoreThreads) score_select_kernel(const ScoreArgs a) {
  constexpr int NCH = 2 * D / 8;      // 16-byte chunks per summary row [kmin | kmax]
  constexpr int J = NCH / 4;          // chunks per lane per row
  extern __shared__ uint32_t keys[];  // [max_pages], used by the selecting CTA only
  __shared__ int is_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, t = lane & 3;
  const int h = blockIdx.x % a.Hkv, tile = blockIdx.x / a.Hkv, b = blockIdx.y;
  const int G = a.Hq / a.Hkv;
  const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
  const int nb = (L + a.P - 1) / a.P;
  const int ntiles = max(1, (nb + kPagesPerCta - 1) / kPagesPerCta);
  float* srow = a.scores + ((size_t)b * a.Hkv + h) * a.max_pages;

  // the previous kernel of the stream may still be using this workspace
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // let the attention kernel get launched; it waits for this grid before reading
  asm volatile("griddepcontrol.launch_dependents;");

  const int p0 = tile * kPagesPerCta + warp * 16;
  if (tile >= ntiles) {  // past the sequence: scores are -inf there
    if (lane < 16 && p0 + lane < a.max_pages) srow[p0 + lane] = -INFINITY;
    return;
  }

  if (p0 < a.max_pages) {
    // decode-time refresh of the newest pages' summaries that fall in this warp's tile
    bool refreshed = false;
    if (a.k_cache) {
      for (int lp = max(p0, nb - a.n_tail); lp < min(p0 + 16, nb); ++lp) {
        const int ph = a.page_table[(size_t)b * a.max_pages + lp];
        if (ph < 0 || ph >= a.n_pool) continue;
        warp_refresh_summary<D>(a.k_cache, a.summ, ph, h, a.Hkv, a.P, min(a.P, L - lp * a.P),
                                lane);
        refreshed = true;
      }
      if (refreshed) {
        __threadfence_block();
        __syncwarp();
      }
    }

    // A: summary rows of pages p0 + r and p0 + r + 8 (chunk 4j + t of each row)
    const int pa = p0 + r, pb = p0 + r + 8;
    uint4 ra[J], rb[J];
    {
      const int pha = pa < nb ? a.page_table[(size_t)b * a.max_pages + pa] : 0;
      const int phb = pb < nb ? a.page_table[(size_t)b * a.max_pages + pb] : 0;
      if ((pha < 0 || pha >= a.n_pool || phb < 0 || phb >= a.n_pool) && t == 0)
        report(a.status, SA_ERR_DEVICE_CHECK);
      const uint4* rowa = (pa < nb && pha >= 0 && pha < a.n_pool)
                              ? a.summ + ((size_t)pha * a.Hkv + h) * NCH
                              : nullptr;
      const uint4* rowb = (pb < nb && phb >= 0 && phb < a.n_pool)
                              ? a.summ + ((size_t)phb * a.Hkv + h) * NCH
                              : nullptr;
      if (refreshed) {  // rows just written by this warp: read them through L2
#pragma unroll
        for (int j = 0; j < J; ++j) {
          ra[j] = rowa ? __ldcg(rowa + 4 * j + t) : make_uint4(0, 0, 0, 0);
          rb[j] = rowb ? __ldcg(rowb + 4 * j + t) : make_uint4(0, 0, 0, 0);
        }
      } else {
#pragma unroll
        for (int j = 0; j < J; ++j) {
          ra[j] = rowa ? ldg_nc_v4(rowa + 4 * j + t) : make_uint4(0, 0, 0, 0);
          rb[j] = rowb ? ldg_nc_v4(rowb + 4 * j + t) : make_uint4(0, 0, 0, 0);
        }
      }
    }

    // B: [min(q,0) | max(q,0)] of query head n = r of the group, same chunk order
    uint4 bq[J];
    if (r < G) {
      const uint4* qrow =
          reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + h * G + r) * D);
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int c = 4 * j + t;  // chunk of the 2D-long contraction
        const uint4 v = qrow[c % (D / 8)];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t neg = ((w[e] >> 15) & 0x00010001u) * 0xFFFFu;  // negative halves
          w[e] = (c < D / 8) ? (w[e] & neg) : (w[e] & ~neg);
        }
        bq[j] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < J; ++j) bq[j] = make_uint4(0, 0, 0, 0);
    }

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < J; ++j) {
      mma_bf16_16816(acc, ra[j].x, rb[j].x, ra[j].y, rb[j].y, bq[j].x, bq[j].y);
      mma_bf16_16816(acc, ra[j].z, rb[j].z, ra[j].w, rb[j].w, bq[j].z, bq[j].w);
    }
    // acc: [page r][heads 2t, 2t+1], [page r+8][heads 2t, 2t+1]
    const bool v0 = 2 * t < G, v1 = 2 * t + 1 < G;
    float m0 = fmaxf(v0 ? acc[0] : -INFINITY, v1 ? acc[1] : -INFINITY);
    float m1 = fmaxf(v0 ? acc[2] : -INFINITY, v1 ? acc[3] : -INFINITY);
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
    if (t == 0) {
      if (pa < a.max_pages) srow[pa] = pa < nb ? m0 : -INFINITY;
      if (pb < a.max_pages) srow[pb] = pb < nb ? m1 : -INFINITY;
    }
  }

  // ---- arrival: the last CTA of this (sequence, KV head) selects ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t* cnt = a.arrivals + (size_t)b * a.Hkv + h;
    const uint32_t old = atomicAdd(cnt, 1u);
    is_last = old == (uint32_t)(ntiles - 1);
    if (is_last) *cnt = 0;  // ready for the next call
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  block_select<kScoreThreads>(srow, nb, a.K, a.s_pages, a.w_pages, keys,
                              a.sel + ((size_t)b * a.Hkv + h) * a.K,
                              a.sel_count + (size_t)b * a.Hkv + h,
                              a.page_table + (size_t)b * a.max_pages,
                              a.sel_phys ? a.sel_phys + ((size_t)b * a.Hkv + h) * a.K : nullptr);
}

cudaError_t launch_score_select(const sa_geom& g, const void* q, void* summ, const void* k_cache,
                                int n_tail, const int32_t* page_table, const int32_t* seq_lens,
                                float* scores, uint32_t* arrivals, int K, int sink_pages,
                                int window_pages, int32_t* sel, int32_t* sel_count,
                                int32_t* sel_phys, int32_t* status, cudaStream_t stream) {
  ScoreArgs a;
  a.sel_phys = sel_phys;
  a.q = static_cast<const uint16_t*>(q);
  a.summ = static_cast<uint4*>(summ);
  a.k_cache = static_cast<const uint4*>(k_cache);
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.scores = scores;
  a.arrivals = arrivals;
  a.sel = sel;
  a.sel_count = sel_count;
  a.status = status;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.P = g.P;
  a.max_pages = g.max_pages;
  a.n_pool = g.n_pool;
  a.K = K;
  a.s_pages = sink_pages;
  a.w_pages = window_pages;
  a.n_tail = n_tail;
  const int ntiles = (g.max_pages + kPagesPerCta - 1) / kPagesPerCta;
  const size_t smem = (size_t)g.max_pages * sizeof(uint32_t);
  void (*kern)(const ScoreArgs);
  if (g.Dk == 64)
    kern = score_select_kernel<64>;
  else if (g.Dk == 128)
    kern = score_select_kernel<128>;
  else
    return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ntiles * g.Hkv, g.B);
  cfg.blockDim = dim3(kScoreThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace sa
