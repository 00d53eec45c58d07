// sa_topk.cu -- top-k page selection with forced sink / local-window pages.
//
// Method: per (sequence, KV head) keep budget/P pages: the attention-sink pages and
// the local-window pages always (the A-shape pattern of SCBench's Tri-shape section),
// plus the best-scoring remaining pages (Quest's query-aware choice, "SparseEngine"
// blog hook-point paragraph; the "top pages" of the Vortex summary, section 1).
// Equal scores go to the lower page index; the result is the ascending page list.
//
// One CTA per (sequence, KV head).  Scores become order-preserving 32-bit keys in
// shared memory (forced pages get key 0, below every real score).  An MSB-first
// 8-bit radix select (4 passes; warp-aggregated shared-memory histograms; one warp
// scans the 256 bins) finds the exact key T of the k-th best candidate and how many
// keys equal to T are still needed.  A final pass marks forced pages, keys > T and
// the lowest-index keys == T, and two block-wide scans compact the marks into the
// ascending output list.  Deterministic: no result depends on thread timing.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int wv = lane < NT / 32 ? warp_tot[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += u;
    }
    if (lane < NT / 32) warp_tot[lane] = wi - wv;  // exclusive warp offsets
    if (lane == 31) warp_tot[NT / 32] = wi;        // block total
  }
  __syncthreads();
  int res = warp_tot[warp] + incl - v;
  *total = warp_tot[NT / 32];
  __syncthreads();
  return res;
}

template <int NT>
__global__ void __launch_bounds__(NT)
    topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int Hkv,
                int P, int max_pages, int K, int s_pages, int w_pages, int32_t* __restrict__ sel,
                int32_t* __restrict__ sel_count) {
  extern __shared__ uint32_t keys[];  // [max_pages]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sh_bin, sh_above;
  __shared__ int warp_tot[NT / 32 + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x, b = blockIdx.y;
  const int L = min(max(seq_lens[b], 0), max_pages * P);
  const int nb = (L + P - 1) / P;
  int32_t* out = sel + ((size_t)b * Hkv + h) * K;
  if (nb <= K) {
    for (int i = tid; i < K; i += NT) out[i] = i < nb ? i : -1;
    if (tid == 0) sel_count[(size_t)b * Hkv + h] = nb;
    return;
  }
  const float* srow = scores + ((size_t)b * Hkv + h) * max_pages;
  const int wbeg = nb - w_pages;
  for (int p = tid; p < nb; p += NT)
    keys[p] = (p < s_pages || p >= wbeg) ? 0u : f32_order_key(srow[p]);

  uint32_t prefix = 0, pmask = 0;
  int k_rem = K - s_pages - w_pages;  // < number of candidates
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
      for (int i = 0; i < 8; ++i) { c[i] = hist[lane * 8 + i]; tot += c[i]; }
      uint32_t incl = tot;  // sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        uint32_t u = __shfl_down_sync(0xffffffffu, incl, off);
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
  }
  const uint32_t T = prefix;  // key of the k-th best candidate; k_rem keys == T needed

  // final pass over contiguous segments: eq ranks, then output positions
  const int seg = (nb + NT - 1) / NT;
  const int beg = min(nb, tid * seg), end = min(nb, beg + seg);
  int n_eq = 0;
  for (int p = beg; p < end; ++p) n_eq += keys[p] == T;
  int tot;
  int eq_rank = block_excl_scan<NT>(n_eq, warp_tot, &tot);
  int n_sel = 0;
  for (int p = beg, er = eq_rank; p < end; ++p) {
    const uint32_t key = keys[p];
    const bool forced = p < s_pages || p >= wbeg;
    const bool is_eq = key == T;
    n_sel += forced || key > T || (is_eq && er < k_rem);
    er += is_eq;
  }
  int pos = block_excl_scan<NT>(n_sel, warp_tot, &tot);
  for (int p = beg, er = eq_rank; p < end; ++p) {
    const uint32_t key = keys[p];
    const bool forced = p < s_pages || p >= wbeg;
    const bool is_eq = key == T;
    if (forced || key > T || (is_eq && er < k_rem)) out[pos++] = p;
    er += is_eq;
  }
  for (int i = tot + tid; i < K; i += NT) out[i] = -1;
  if (tid == 0) sel_count[(size_t)b * Hkv + h] = tot;
}

cudaError_t launch_topk(const sa_geom& g, const float* scores, const int32_t* seq_lens, int K,
                        int sink_pages, int window_pages, int32_t* sel, int32_t* sel_count,
                        cudaStream_t stream) {
  constexpr int NT = 512;
  const size_t smem = (size_t)g.max_pages * sizeof(uint32_t);
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  dim3 grid(g.Hkv, g.B);
  topk_kernel<NT><<<grid, NT, smem, stream>>>(scores, seq_lens, g.Hkv, g.P, g.max_pages, K,
                                              sink_pages, window_pages, sel, sel_count);
  return cudaGetLastError();
}

}  // namespace sa
