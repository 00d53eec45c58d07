// sa_select.cuh -- device pieces of the top-k page selection: the decode-time refresh of
// a page's summary, the block scan, and the exact radix threshold over order-preserving
// 32-bit keys.
//
// Method (SparseEngine blog, hook-point paragraph: Quest picks the pages to read from the
// current query; SCBench notes, Tri-shape section: sink tokens and the local window are
// always kept): per (sequence, KV head) the forced pages plus the best remaining pages by
// the page bound, equal scores going to the lower page index.
#pragma once

#include "sa_common.cuh"

namespace sa {

constexpr int kMaxTail = 16;
constexpr int kHistBits = 11;  // digit of the one-pass histogram
constexpr int kHistBins = 1 << kHistBits;
constexpr int kBinCap = 256;            // boundary-bin size ranked exactly
constexpr uint32_t kWin = 0xFFFFFFFFu;  // marks a candidate taken from the boundary bin

// Barrier over the NT threads taking part in a selection: the whole CTA (ID < 0) or a
// named hardware barrier shared by the first NT threads of the CTA.
template <int ID, int NT>
struct SelBar {
  __device__ __forceinline__ static void sync() {
    if constexpr (ID < 0)
      __syncthreads();
    else
      asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(NT) : "memory");
  }
};

// Shared-memory scratch of one selection.
struct SelScratch {
  uint32_t* hist;      // [kHistBins]
  uint32_t* bin_key;   // [kBinCap]
  int* bin_page;       // [kBinCap]
  int* warp_tot;       // [NT / 32 + 1]
  uint32_t* red;       // [2 * NT / 32]
  uint32_t* misc;      // [4]: boundary bin, count above it, bin fill counter
};

template <int NT, class Bar>
__device__ __forceinline__ int sel_block_excl_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  Bar::sync();
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
  Bar::sync();
  const int res = warp_tot[warp] + incl - v;
  *total = warp_tot[NT / 32];
  Bar::sync();
  return res;
}

// Pieces of the decode-time refresh of one (physical page, KV head), one warp: lane l
// works on 16-byte chunk l % (D / 8) of the rows.

// The G <= 8 query rows at qh (chunk of this lane; zero past G).  Loaded before K so
// that their loads are in flight together.
template <int D>
__device__ __forceinline__ void warp_load_q(const uint16_t* qh, int G, int lane, uint4 (&qv)[8]) {
  constexpr int CPR = D / 8;
#pragma unroll
  for (int g = 0; g < 8; ++g)
    qv[g] = (g < G && lane < CPR)
                ? *reinterpret_cast<const uint4*>(qh + (size_t)g * D + (lane % CPR) * 8)
                : make_uint4(0, 0, 0, 0);
}

// Channel-wise min and max (bf16 patterns) of the page's `valid` rows of K; every lane
// ends with those of its chunk.
template <int D>
__device__ __forceinline__ void warp_page_minmax(const uint4* __restrict__ k_cache, int phys,
                                                 int h, int Hkv, int P, int valid, int lane,
                                                 uint4& kmin, uint4& kmax) {
  constexpr int CPR = D / 8;     // 8 or 16 chunks per row
  constexpr int RPI = 32 / CPR;  // rows per warp iteration
  const int c = lane % CPR;
  const uint4* blk = k_cache + ((size_t)phys * Hkv + h) * P * CPR;
  uint4 mn = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
  uint4 mx = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
  // up to 16 rows per lane in flight at once (a whole page of 32 rows at Dk = 128): the
  // refresh sits on its warp's critical path, so one memory round trip, not several
  constexpr int kBatch = 16;
  for (int t0 = lane / CPR; t0 < valid; t0 += kBatch * RPI) {
    uint4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int t = t0 + i * RPI;
      if (t < valid) v[i] = __ldcg(blk + (size_t)t * CPR + c);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (t0 + i * RPI < valid) {
        const uint32_t k0 = bf2_key(v[i].x), k1 = bf2_key(v[i].y);
        const uint32_t k2 = bf2_key(v[i].z), k3 = bf2_key(v[i].w);
        mn.x = __vmins2(mn.x, k0); mn.y = __vmins2(mn.y, k1);
        mn.z = __vmins2(mn.z, k2); mn.w = __vmins2(mn.w, k3);
        mx.x = __vmaxs2(mx.x, k0); mx.y = __vmaxs2(mx.y, k1);
        mx.z = __vmaxs2(mx.z, k2); mx.w = __vmaxs2(mx.w, k3);
      }
    }
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
  kmin = make_uint4(bf2_key(mn.x), bf2_key(mn.y), bf2_key(mn.z), bf2_key(mn.w));
  kmax = make_uint4(bf2_key(mx.x), bf2_key(mx.y), bf2_key(mx.z), bf2_key(mx.w));
}

// max over the G query heads of sum_c max(q_gc * hi_c, q_gc * lo_c), lo/hi the bf16
// pairs of this lane's 8 channels (lanes past the row add nothing); in every lane.
template <int D>
__device__ __forceinline__ float warp_bound_score(const uint4 (&qv)[8], int G, int lane,
                                                  const uint32_t (&lo)[4],
                                                  const uint32_t (&hi)[4]) {
  constexpr int CPR = D / 8;
  float best = -INFINITY;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    if (g >= G) break;
    const uint32_t qw[4] = {qv[g].x, qv[g].y, qv[g].z, qv[g].w};
    float part = 0.f;
    if (lane < CPR) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float qf = __uint_as_float(hf ? (qw[e] & 0xFFFF0000u) : (qw[e] << 16));
          const float a0 = __uint_as_float(hf ? (lo[e] & 0xFFFF0000u) : (lo[e] << 16));
          const float a1 = __uint_as_float(hf ? (hi[e] & 0xFFFF0000u) : (hi[e] << 16));
          part += fmaxf(qf * a1, qf * a0);
        }
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    best = fmaxf(best, part);
  }
  return best;
}

// Recompute the bf16 summary of one (physical page, KV head) from K (one warp), store
// it, and return in every lane its score for the G query heads at qh (max over heads).
template <int D>
__device__ float warp_refresh_and_score(const uint4* __restrict__ k_cache,
                                        uint4* __restrict__ summ, const uint16_t* qh, int G,
                                        int phys, int h, int Hkv, int P, int valid, int lane) {
  constexpr int CPR = D / 8;
  uint4 qv[8];
  warp_load_q<D>(qh, G, lane, qv);
  uint4 kmin, kmax;
  warp_page_minmax<D>(k_cache, phys, h, Hkv, P, valid, lane, kmin, kmax);
  uint4* out = summ + ((size_t)phys * Hkv + h) * 2 * CPR;
  const int c = lane % CPR;
  if (lane < CPR) {
    __stcg(out + c, kmin);
    __stcg(out + CPR + c, kmax);
  }
  const uint32_t lo[4] = {kmin.x, kmin.y, kmin.z, kmin.w};
  const uint32_t hi[4] = {kmax.x, kmax.y, kmax.z, kmax.w};
  return warp_bound_score<D>(qv, G, lane, lo, hi);
}

// Threshold of the top-k_rem0 candidates among keys[0, nb) (forced pages, p < s_pages or
// p >= wbeg, are not candidates; k_rem0 < the number of candidates).  [kmn, kmx] is the
// candidates' key range.  A candidate p is taken when keys[p] == kWin (marked here) or
// keys[p] >= the returned threshold (a 33-bit value).  MSB-first radix select with 11-bit
// digits from the highest bit in which the candidates differ; it stops as soon as the
// boundary bin is wholly taken or holds at most kBinCap candidates, which are then ranked
// exactly by (key desc, page asc).  All-equal boundary keys take the lowest pages.
// Every one of the NT threads calls it; Bar synchronises them.
template <int NT, class Bar>
__device__ uint64_t radix_select_threshold(uint32_t* keys, int nb, int s_pages, int wbeg,
                                           int k_rem0, uint32_t kmn, uint32_t kmx,
                                           const SelScratch& sh) {
  const int tid = threadIdx.x;
  uint64_t thr = 1ull << 32;  // above every key: forced pages only
  if (k_rem0 <= 0) return thr;
  const uint32_t diff = kmn ^ kmx;
  int hi = diff ? 31 - __clz(diff) : -1;  // highest undecided bit
  uint32_t pmask;                         // bits decided so far (above hi)
  if (hi < 0)
    pmask = 0xFFFFFFFFu;  // all candidates are equal
  else if (hi == 31)
    pmask = 0u;
  else
    pmask = ~((2u << hi) - 1u);
  uint32_t pval = kmn & pmask;
  int k_need = k_rem0;
  int state = 0;  // 0: go on, 1: thr set, 2: tie on the full key
  while (state == 0) {
    if (hi < 0) {
      state = 2;
      break;
    }
    const int lo = max(0, hi - (kHistBits - 1));
    const uint32_t dmask = (2u << (hi - lo)) - 1u;
    for (int i = tid; i < kHistBins; i += NT) sh.hist[i] = 0;
    Bar::sync();
    for (int p = tid; p < nb; p += NT) {
      const uint32_t key = keys[p];
      if (!(p < s_pages || p >= wbeg) && (key & pmask) == pval)
        atomicAdd(&sh.hist[(key >> lo) & dmask], 1u);
    }
    Bar::sync();
    if (tid == 0) SA_TRACE_POINT(1, 5);  // histogram built
    // bins owned BPT per thread; candidates in bins above each thread's range
    constexpr int BPT = kHistBins / NT;
    int mine = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) mine += sh.hist[tid * BPT + i];
    int total;
    const int below = sel_block_excl_scan<NT, Bar>(mine, sh.warp_tot, &total);
    int run = total - below - mine;
    for (int i = BPT - 1; i >= 0; --i) {
      const int cnt = sh.hist[tid * BPT + i];
      if (run < k_need && run + cnt >= k_need) {
        sh.misc[0] = tid * BPT + i;
        sh.misc[1] = run;
      }
      run += cnt;
    }
    Bar::sync();
    if (tid == 0) SA_TRACE_POINT(1, 6);  // boundary bin found
    const uint32_t bstar = sh.misc[0];
    k_need -= (int)sh.misc[1];
    const int nbin = sh.hist[bstar];
    pval |= bstar << lo;
    pmask |= dmask << lo;
    if (nbin == k_need) {  // the whole boundary bin is taken
      thr = pval;
      state = 1;
    } else if (nbin <= kBinCap) {
      // exact ranking inside the boundary bin: larger key first, then lower page
      if (tid == 0) sh.misc[2] = 0;
      Bar::sync();
      for (int p = tid; p < nb; p += NT) {
        const uint32_t key = keys[p];
        if (!(p < s_pages || p >= wbeg) && (key & pmask) == pval) {
          const int i = atomicAdd(&sh.misc[2], 1u);
          sh.bin_key[i] = key;
          sh.bin_page[i] = p;
        }
      }
      Bar::sync();
      // each warp ranks members w, w + NT / 32, ...; its lanes split the comparisons
      const int lane = tid & 31;
      for (int i = tid >> 5; i < nbin; i += NT / 32) {
        const uint32_t key = sh.bin_key[i];
        const int pg = sh.bin_page[i];
        int rank = 0;
        for (int j = lane; j < nbin; j += 32) {
          const uint32_t kj = sh.bin_key[j];
          rank += kj > key || (kj == key && sh.bin_page[j] < pg);
        }
        rank = __reduce_add_sync(0xffffffffu, rank);
        if (lane == 0 && rank < k_need) keys[pg] = kWin;
      }
      thr = (uint64_t)pval + (1ull << lo);
      state = 1;
    }
    hi = lo - 1;
    Bar::sync();
  }
  if (state == 2) {
    // the boundary keys are all equal to T = pval: take the lowest-index ones
    const uint32_t T = pval;
    const int seg = (nb + NT - 1) / NT;
    const int beg = min(nb, tid * seg), end = min(nb, beg + seg);
    int n_eq = 0;
    for (int p = beg; p < end; ++p) n_eq += !(p < s_pages || p >= wbeg) && keys[p] == T;
    int tot;
    int er = sel_block_excl_scan<NT, Bar>(n_eq, sh.warp_tot, &tot);
    for (int p = beg; p < end; ++p) {
      if (!(p < s_pages || p >= wbeg) && keys[p] == T) {
        if (er < k_need) keys[p] = kWin;
        ++er;
      }
    }
    thr = (uint64_t)T + 1;
    Bar::sync();
  }
  return thr;
}

// Candidates' key range [kmn, kmx] reduced over the NT threads (per-thread partials in).
template <int NT, class Bar>
__device__ __forceinline__ void block_key_range(uint32_t& kmn, uint32_t& kmx, uint32_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  kmn = __reduce_min_sync(0xffffffffu, kmn);
  kmx = __reduce_max_sync(0xffffffffu, kmx);
  if (lane == 0) {
    red[warp] = kmn;
    red[NT / 32 + warp] = kmx;
  }
  Bar::sync();
  kmn = 0xFFFFFFFFu;
  kmx = 0u;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    kmn = min(kmn, red[w]);
    kmx = max(kmx, red[NT / 32 + w]);
  }
}

}  // namespace sa
