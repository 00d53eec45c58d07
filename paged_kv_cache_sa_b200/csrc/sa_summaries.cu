// sa_summaries.cu -- per-page channel-wise min/max key summaries.
//
// Method: for every valid page of a sequence and every KV head, the min and the max
// of each key channel over the page's valid tokens (the per-page key summary Quest
// scores against the query; "SparseEngine" blog, hook-point paragraph).  Summaries
// live with the PHYSICAL page, so a remapped or shared page keeps its summary.
//
// One warp per (page, KV head).  A (page, head) block is P*Dk contiguous bf16; lanes
// read it in 16-byte vectors, reduce with SIMD 16-bit min/max on an order key
// (-0 < +0, bit-exact), then combine lanes with shuffles.  HBM-bound: bytes per
// (page, head) = valid_tokens * Dk * 2 read + 2 * Dk * 2 written.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

// CPR = 16-byte chunks per key row (Dk / 8).
template <int CPR>
__global__ void __launch_bounds__(256) summaries_kernel(const uint4* __restrict__ k_cache,
                                                        const int32_t* __restrict__ page_table,
                                                        const int32_t* __restrict__ seq_lens,
                                                        uint4* __restrict__ summ, int Hkv, int P,
                                                        int max_pages, int n_pool, int n_tail) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int L = min(max(seq_lens[b], 0), max_pages * P);
  const int nb = (L + P - 1) / P;
  int lp = blockIdx.x;
  if (n_tail > 0) {
    lp = nb - n_tail + (int)blockIdx.x;
    if (lp < 0) return;
  }
  if (lp >= nb) return;
  const int phys = page_table[(size_t)b * max_pages + lp];
  if (phys < 0 || phys >= n_pool) return;  // not a page of the pool: nothing to summarise
  const int valid = min(P, L - lp * P);
  for (int h = threadIdx.x >> 5; h < Hkv; h += blockDim.x >> 5) {
  const uint4* blk = k_cache + ((size_t)phys * Hkv + h) * P * CPR;
  uint4* out = summ + ((size_t)phys * Hkv + h) * 2 * CPR;

  if constexpr (32 % CPR == 0) {
    // lanes split a row; each lane keeps one chunk index for the whole page
    constexpr int RPI = 32 / CPR;  // rows per iteration
    const int c = lane % CPR;
    uint4 mn = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
    uint4 mx = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
#pragma unroll 4
    for (int t = lane / CPR; t < valid; t += RPI) {
      uint4 v = ldg_nc_v4(blk + (size_t)t * CPR + c);
      uint32_t k0 = bf2_key(v.x), k1 = bf2_key(v.y), k2 = bf2_key(v.z), k3 = bf2_key(v.w);
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
    if (lane < CPR) {
      out[c] = make_uint4(bf2_key(mn.x), bf2_key(mn.y), bf2_key(mn.z), bf2_key(mn.w));
      out[CPR + c] = make_uint4(bf2_key(mx.x), bf2_key(mx.y), bf2_key(mx.z), bf2_key(mx.w));
    }
  } else {
    // wide rows (latent keys): each lane owns chunks lane, lane+32, ... of every row
    constexpr int NC = (CPR + 31) / 32;
    uint4 mn[NC], mx[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      mn[j] = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
      mx[j] = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
    }
#pragma unroll 4
    for (int t = 0; t < valid; ++t) {
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const int c = lane + 32 * j;
        if (c < CPR) {
          uint4 v = ldg_nc_v4(blk + (size_t)t * CPR + c);
          uint32_t k0 = bf2_key(v.x), k1 = bf2_key(v.y), k2 = bf2_key(v.z), k3 = bf2_key(v.w);
          mn[j].x = __vmins2(mn[j].x, k0); mn[j].y = __vmins2(mn[j].y, k1);
          mn[j].z = __vmins2(mn[j].z, k2); mn[j].w = __vmins2(mn[j].w, k3);
          mx[j].x = __vmaxs2(mx[j].x, k0); mx[j].y = __vmaxs2(mx[j].y, k1);
          mx[j].z = __vmaxs2(mx[j].z, k2); mx[j].w = __vmaxs2(mx[j].w, k3);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int c = lane + 32 * j;
      if (c < CPR) {
        out[c] = make_uint4(bf2_key(mn[j].x), bf2_key(mn[j].y), bf2_key(mn[j].z),
                            bf2_key(mn[j].w));
        out[CPR + c] = make_uint4(bf2_key(mx[j].x), bf2_key(mx[j].y), bf2_key(mx[j].z),
                                  bf2_key(mx[j].w));
      }
    }
  }
  }  // heads
}

cudaError_t launch_summaries(const sa_geom& g, const void* k_cache, const int32_t* page_table,
                             const int32_t* seq_lens, void* summ, int n_tail,
                             cudaStream_t stream) {
  const int grid_x = n_tail > 0 ? n_tail : g.max_pages;
  dim3 grid(grid_x, g.B);
  dim3 block(32 * (g.Hkv < 8 ? g.Hkv : 8));
  const uint4* k = static_cast<const uint4*>(k_cache);
  uint4* s = static_cast<uint4*>(summ);
  switch (g.Dk) {
    case 64:
      summaries_kernel<8><<<grid, block, 0, stream>>>(k, page_table, seq_lens, s, g.Hkv, g.P,
                                                      g.max_pages, g.n_pool, n_tail);
      break;
    case 128:
      summaries_kernel<16><<<grid, block, 0, stream>>>(k, page_table, seq_lens, s, g.Hkv, g.P,
                                                       g.max_pages, g.n_pool, n_tail);
      break;
    case 576:
      summaries_kernel<72><<<grid, block, 0, stream>>>(k, page_table, seq_lens, s, g.Hkv, g.P,
                                                       g.max_pages, g.n_pool, n_tail);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace sa
