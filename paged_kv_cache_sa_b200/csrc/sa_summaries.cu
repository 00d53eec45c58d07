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
//
// fp8 records (grouped-query head dims).  The same min/max, then stored as OCP FP8
// E4M3 codes rounded outward -- the min row toward -inf, the max row toward +inf --
// after scaling the (page, head) record by 2^-e, e the smallest integer with
// max|value| * 2^-e <= 448, the largest finite code.  Decoded values (code * 2^e) then
// bracket every key of the page, so the page bound over them is still an upper bound
// (the quantised-KV option the SparseEngine blog's hook-point paragraph lists next to
// Quest; the pages give no format).  Record: [Dk codes min][Dk codes max][int8 e][15
// zero bytes].  The encoder works on the bf16 bit fields, so no value is rounded before
// the one outward step.
#include "sa_common.cuh"
#include "sa_fp8.cuh"
#include "sa_internal.h"

namespace sa {

// CPR = 16-byte chunks per key row (Dk / 8).  F8: write fp8 records (CPR 8 or 16).
template <int CPR, bool F8 = false>
__global__ void __launch_bounds__(256) summaries_kernel(const uint4* __restrict__ k_cache,
                                                        const int32_t* __restrict__ page_table,
                                                        const int32_t* __restrict__ seq_lens,
                                                        void* __restrict__ summ_out, int Hkv, int P,
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
  if constexpr (32 % CPR == 0) {
    for (int h = threadIdx.x >> 5; h < Hkv; h += blockDim.x >> 5) {
      const uint4* blk = k_cache + ((size_t)phys * Hkv + h) * P * CPR;
      uint4* out = static_cast<uint4*>(summ_out) + ((size_t)phys * Hkv + h) * 2 * CPR;
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
      const uint4 lo = make_uint4(bf2_key(mn.x), bf2_key(mn.y), bf2_key(mn.z), bf2_key(mn.w));
      const uint4 hi = make_uint4(bf2_key(mx.x), bf2_key(mx.y), bf2_key(mx.z), bf2_key(mx.w));
      if constexpr (F8) {
        // every lane holds chunk lane % CPR: the warp max covers the whole record
        uint32_t am = max_mag2(max_mag2(max_mag2(max_mag2(0u, lo.x), lo.y), lo.z), lo.w);
        am = max_mag2(max_mag2(max_mag2(max_mag2(am, hi.x), hi.y), hi.z), hi.w);
        am = __reduce_max_sync(0xffffffffu, am);
        const int e = fp8_record_exp(am);
        constexpr int D = CPR * 8;
        uint8_t* rec = static_cast<uint8_t*>(summ_out) + ((size_t)phys * Hkv + h) * (2 * D + 16);
        if (lane < CPR) {
          *reinterpret_cast<uint2*>(rec + c * 8) =
              make_uint2(e4m3_pack(lo.x, lo.y, e, false), e4m3_pack(lo.z, lo.w, e, false));
          *reinterpret_cast<uint2*>(rec + D + c * 8) =
              make_uint2(e4m3_pack(hi.x, hi.y, e, true), e4m3_pack(hi.z, hi.w, e, true));
        }
        if (lane == 0)
          *reinterpret_cast<uint4*>(rec + 2 * D) = make_uint4((uint32_t)e & 0xFFu, 0u, 0u, 0u);
      } else if (lane < CPR) {
        out[c] = lo;
        out[CPR + c] = hi;
      }
    }  // heads
  } else {
    // wide rows (latent keys): the block's warps split the page's tokens (warp w takes
    // rows w, w + nw, ...), each lane owning chunks lane, lane + 32, ... of a row; the
    // warps' partial minima and maxima meet in shared memory
    constexpr int NC = (CPR + 31) / 32;
    __shared__ uint4 part[2][8][CPR];
    const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;  // nw <= 8
    for (int h = 0; h < Hkv; ++h) {
      const uint4* blk = k_cache + ((size_t)phys * Hkv + h) * P * CPR;
      uint4* out = static_cast<uint4*>(summ_out) + ((size_t)phys * Hkv + h) * 2 * CPR;
      uint4 mn[NC], mx[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        mn[j] = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
        mx[j] = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
      }
#pragma unroll 4
      for (int t = w; t < valid; t += nw) {
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
          part[0][w][c] = mn[j];
          part[1][w][c] = mx[j];
        }
      }
      __syncthreads();
      // one thread per (row, chunk): fold the warps' partials, back to bf16 patterns
      for (int e = threadIdx.x; e < 2 * CPR; e += blockDim.x) {
        const int r = e / CPR, c = e % CPR;
        uint4 v = part[r][0][c];
        for (int ww = 1; ww < nw; ++ww) {
          const uint4 u = part[r][ww][c];
          if (r == 0) {
            v.x = __vmins2(v.x, u.x); v.y = __vmins2(v.y, u.y);
            v.z = __vmins2(v.z, u.z); v.w = __vmins2(v.w, u.w);
          } else {
            v.x = __vmaxs2(v.x, u.x); v.y = __vmaxs2(v.y, u.y);
            v.z = __vmaxs2(v.z, u.z); v.w = __vmaxs2(v.w, u.w);
          }
        }
        out[r * CPR + c] = make_uint4(bf2_key(v.x), bf2_key(v.y), bf2_key(v.z), bf2_key(v.w));
      }
      __syncthreads();
    }
  }
}

cudaError_t launch_summaries_fp8(const sa_geom& g, const void* k_cache,
                                 const int32_t* page_table, const int32_t* seq_lens, void* summ8,
                                 int n_tail, cudaStream_t stream) {
  const int grid_x = n_tail > 0 ? n_tail : g.max_pages;
  dim3 grid(grid_x, g.B);
  dim3 block(32 * (g.Hkv < 8 ? g.Hkv : 8));
  const uint4* k = static_cast<const uint4*>(k_cache);
  switch (g.Dk) {
    case 64:
      summaries_kernel<8, true><<<grid, block, 0, stream>>>(k, page_table, seq_lens, summ8, g.Hkv,
                                                            g.P, g.max_pages, g.n_pool, n_tail);
      break;
    case 128:
      summaries_kernel<16, true><<<grid, block, 0, stream>>>(k, page_table, seq_lens, summ8,
                                                             g.Hkv, g.P, g.max_pages, g.n_pool,
                                                             n_tail);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_summaries(const sa_geom& g, const void* k_cache, const int32_t* page_table,
                             const int32_t* seq_lens, void* summ, int n_tail,
                             cudaStream_t stream) {
  const int grid_x = n_tail > 0 ? n_tail : g.max_pages;
  dim3 grid(grid_x, g.B);
  // a warp per KV head (up to 8); latent rows: eight warps share each page's tokens
  dim3 block(g.Dk == 576 ? 256 : 32 * (g.Hkv < 8 ? g.Hkv : 8));
  const uint4* k = static_cast<const uint4*>(k_cache);
  void* s = summ;
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
