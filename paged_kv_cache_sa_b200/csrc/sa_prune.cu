// sa_prune.cu -- prefix-cache pruning: keep-mask stream compaction into fresh pages.
//
// Method ("SparseEngine" blog, physical-vs-logical and Prefix-Cache Pruning paragraphs):
// the product marks what to keep; the engine keeps only that part, physically frees the
// rest, and leaves the conversation-position marker untouched.  Here: kept tokens are
// compacted, in order, into caller-provided fresh pages (session after session), the
// page table is rewritten, the logical length is returned unchanged, and the new pages
// get their key summaries in the same pass that copies them.
//
// Four launches, no host round trip:
//   count  (chunk, session)   kept tokens per 4096-token chunk (16 keep bytes a thread)
//   plan   (one CTA)          chunk prefix sums, kept length, fresh-page offset per
//                             session, capacity check (SA_ERR_NO_SPACE -> nothing written)
//   pos    (chunk, session)   block scan of the keep flags -> pos_map; -1 tails; new
//                             page-table slice
//   copy   (new page, session) thread (head, 16-byte chunk): gathers the P kept rows of
//                             its chunk through pos_map and the old page table, writes them
//                             to the fresh page, min/max on the fly -> summary; zero pads.
// Bit-exact (copies and integer work only).  HBM-bound: bytes = kept tokens *
// Hkv * (Dk + Dv) * 2 read + the same written + the keep mask.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kPruneChunk = 4096;
constexpr int kPruneThreads = 256;  // 16 keep bytes per thread -> one chunk per CTA

struct PruneWs {
  int32_t* chunk_cnt;   // [B][nchunks]
  int32_t* chunk_base;  // [B][nchunks]
  int32_t* sess_off;    // [B]   first fresh page of each session
  int32_t* sess_kept;   // [B]
};

static int prune_nchunks(const sa_geom& g) {
  const int64_t width = (int64_t)g.max_pages * g.P;
  return (int)((width + kPruneChunk - 1) / kPruneChunk);
}

size_t prune_workspace_bytes(const sa_geom& g) {
  const size_t nc = (size_t)prune_nchunks(g);
  const size_t a = ((size_t)g.B * nc * 4 + 255) & ~size_t(255);
  const size_t s = ((size_t)g.B * 4 + 255) & ~size_t(255);
  return 256 + 2 * a + 2 * s;
}

static PruneWs carve(const sa_geom& g, void* ws) {
  const size_t nc = (size_t)prune_nchunks(g);
  const size_t a = ((size_t)g.B * nc * 4 + 255) & ~size_t(255);
  const size_t s = ((size_t)g.B * 4 + 255) & ~size_t(255);
  uint8_t* base = static_cast<uint8_t*>(ws) + 256;
  PruneWs w;
  w.chunk_cnt = reinterpret_cast<int32_t*>(base);
  w.chunk_base = reinterpret_cast<int32_t*>(base + a);
  w.sess_off = reinterpret_cast<int32_t*>(base + 2 * a);
  w.sess_kept = reinterpret_cast<int32_t*>(base + 2 * a + s);
  return w;
}

__device__ __forceinline__ int count_keep16(const uint8_t* row, int t0, int L) {
  // number of nonzero keep bytes among tokens [t0, t0 + 16) that are < L
  if (t0 >= L) return 0;
  if (t0 + 16 <= L) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + t0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    int n = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // per byte: nonzero -> 1
      uint32_t x = w[e];
      x = (x | (x >> 4)) & 0x0F0F0F0Fu;
      x = (x | (x >> 2)) & 0x03030303u;
      x = (x | (x >> 1)) & 0x01010101u;
      n += __popc(x);
    }
    return n;
  }
  int n = 0;
  for (int t = t0; t < L; ++t) n += row[t] != 0;
  return n;
}

__device__ __forceinline__ int block_scan_excl(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NWARP = kPruneThreads / 32;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < NWARP ? wsum[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += u;
    }
    if (lane < NWARP) wsum[lane] = wi - wv;
    if (lane == 31) wsum[NWARP] = wi;
  }
  __syncthreads();
  const int res = wsum[warp] + incl - v;
  *total = wsum[NWARP];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kPruneThreads)
    prune_count_kernel(const uint8_t* __restrict__ keep, const int32_t* __restrict__ seq_lens,
                       int64_t width, int nchunks, int32_t* __restrict__ chunk_cnt) {
  __shared__ int wsum[kPruneThreads / 32 + 1];
  const int c = blockIdx.x, b = blockIdx.y;
  const long long Lr = seq_lens[b] < 0 ? 0 : seq_lens[b];
  const int L = (int)(Lr < width ? Lr : width);
  const uint8_t* row = keep + (size_t)b * width;
  const int t0 = c * kPruneChunk + threadIdx.x * 16;
  const int n = count_keep16(row, t0, L);
  int tot;
  (void)block_scan_excl(n, wsum, &tot);
  if (threadIdx.x == 0) chunk_cnt[(size_t)b * nchunks + c] = tot;
}

__global__ void __launch_bounds__(1024)
    prune_plan_kernel(const int32_t* __restrict__ seq_lens, int B, int P, int nchunks,
                      int64_t n_free, const int32_t* __restrict__ chunk_cnt,
                      int32_t* __restrict__ chunk_base, int32_t* __restrict__ sess_off,
                      int32_t* __restrict__ sess_kept, int32_t* __restrict__ new_seq_lens,
                      int32_t* __restrict__ logical_len, WsHeader* hdr) {
  __shared__ long long carry;
  __shared__ long long wtot[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    long long np = 0;
    if (b < B) {
      int run = 0;
      for (int c = 0; c < nchunks; ++c) {
        chunk_base[(size_t)b * nchunks + c] = run;
        run += chunk_cnt[(size_t)b * nchunks + c];
      }
      sess_kept[b] = run;
      np = (run + P - 1) / P;
    }
    // block exclusive scan of np (64-bit)
    long long incl = np;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += u;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x / 32;
      const long long wv = lane < nw ? wtot[lane] : 0;
      long long wi = wv;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long u = __shfl_up_sync(0xffffffffu, wi, off);
        if (lane >= off) wi += u;
      }
      if (lane < nw) wtot[lane] = wi - wv;
      if (lane == 31) wtot[32] = wi;
    }
    __syncthreads();
    if (b < B) sess_off[b] = (int32_t)(carry + wtot[warp] + incl - np);
    __syncthreads();
    if (threadIdx.x == 0) carry += wtot[32];
    __syncthreads();
  }
  if (carry > n_free) {
    if (threadIdx.x == 0) {
      report(&hdr->status_bits, SA_ERR_NO_SPACE);
      hdr->abort = 1;
    }
    return;
  }
  if (threadIdx.x == 0) hdr->abort = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    new_seq_lens[b] = sess_kept[b];
    logical_len[b] = seq_lens[b];  // the position marker is carried over unchanged
  }
}

__global__ void __launch_bounds__(kPruneThreads)
    prune_pos_kernel(const uint8_t* __restrict__ keep, const int32_t* __restrict__ seq_lens,
                     const int32_t* __restrict__ free_pages, int64_t width, int max_pages, int P,
                     int nchunks, const int32_t* __restrict__ chunk_base,
                     const int32_t* __restrict__ sess_off, const int32_t* __restrict__ sess_kept,
                     int32_t* __restrict__ pos_map, int32_t* __restrict__ new_page_table,
                     const WsHeader* hdr) {
  __shared__ int wsum[kPruneThreads / 32 + 1];
  if (*(volatile const int32_t*)&hdr->abort) return;
  const int c = blockIdx.x, b = blockIdx.y;
  const long long Lr = seq_lens[b] < 0 ? 0 : seq_lens[b];
  const int L = (int)(Lr < width ? Lr : width);
  const int kept = sess_kept[b];
  const uint8_t* row = keep + (size_t)b * width;
  int32_t* prow = pos_map + (size_t)b * width;
  const int t0 = c * kPruneChunk + threadIdx.x * 16;
  // kept ranks of this chunk
  uint32_t mask = 0;
  if (t0 < L) {
    for (int e = 0; e < 16; ++e)
      if (t0 + e < L && row[t0 + e]) mask |= 1u << e;
  }
  int tot;
  int rank = chunk_base[(size_t)b * nchunks + c] + block_scan_excl(__popc(mask), wsum, &tot);
  while (mask) {
    const int e = __ffs(mask) - 1;
    mask &= mask - 1;
    prow[rank++] = t0 + e;
  }
  // ranks >= kept in this chunk's index slice get -1
  const int64_t s0 = (int64_t)c * kPruneChunk;
  const int64_t s1 = width < s0 + kPruneChunk ? width : s0 + kPruneChunk;
  for (int64_t i = (s0 > kept ? s0 : (int64_t)kept) + threadIdx.x; i < s1; i += blockDim.x)
    prow[i] = -1;
  // new page table entries of this chunk's page slice
  const int np = (kept + P - 1) / P;
  const int j0 = (int)(s0 / P);
  const int j1 = (int)((s1 + P - 1) / P < max_pages ? (s1 + P - 1) / P : max_pages);
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x)
    new_page_table[(size_t)b * max_pages + j] = j < np ? free_pages[sess_off[b] + j] : -1;
}

// thread = (KV head, 16-byte chunk); CPR = Dk/8 chunks per K row, CPRV = Dv/8 (0: V aliases K)
template <int CPR, int CPRV>
__global__ void prune_copy_kernel(const uint4* __restrict__ k_cache, const uint4* __restrict__ v_cache,
                                  const int32_t* __restrict__ page_table,
                                  const int32_t* __restrict__ free_pages, int Hkv, int P,
                                  int max_pages, int n_pool, int64_t width, const int32_t* __restrict__ pos_map,
                                  const int32_t* __restrict__ sess_off,
                                  const int32_t* __restrict__ sess_kept, uint4* __restrict__ k_dst,
                                  uint4* __restrict__ v_dst, uint4* __restrict__ summ,
                                  const WsHeader* hdr) {
  if (*(volatile const int32_t*)&hdr->abort) return;
  const int j = blockIdx.x, b = blockIdx.y;
  const int kept = sess_kept[b];
  if (j * P >= kept) return;
  const int n = min(P, kept - j * P);
  const int dst = free_pages[sess_off[b] + j];
  if (dst < 0 || dst >= n_pool) {
    if (threadIdx.x == 0) report(const_cast<int32_t*>(&hdr->status_bits), SA_ERR_DEVICE_CHECK);
    return;
  }
  const int32_t* prow = pos_map + (size_t)b * width + (size_t)j * P;
  const int32_t* ptab = page_table + (size_t)b * max_pages;
  for (int item = threadIdx.x; item < Hkv * CPR; item += blockDim.x) {
    const int h = item / CPR, c = item % CPR;
    uint4 mn = make_uint4(0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu, 0x7FFF7FFFu);
    uint4 mx = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
    uint4* kd = k_dst + ((size_t)dst * Hkv + h) * P * CPR + c;
#pragma unroll 4
    for (int t = 0; t < P; ++t) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < n) {
        const int pos = prow[t];
        const int src = ptab[pos / P];
        if (src < 0 || src >= n_pool) {
          report(const_cast<int32_t*>(&hdr->status_bits), SA_ERR_DEVICE_CHECK);
          continue;
        }
        v = ldg_nc_v4(k_cache + (((size_t)src * Hkv + h) * P + pos % P) * CPR + c);
        const uint32_t k0 = bf2_key(v.x), k1 = bf2_key(v.y), k2 = bf2_key(v.z), k3 = bf2_key(v.w);
        mn.x = __vmins2(mn.x, k0); mn.y = __vmins2(mn.y, k1);
        mn.z = __vmins2(mn.z, k2); mn.w = __vmins2(mn.w, k3);
        mx.x = __vmaxs2(mx.x, k0); mx.y = __vmaxs2(mx.y, k1);
        mx.z = __vmaxs2(mx.z, k2); mx.w = __vmaxs2(mx.w, k3);
      }
      kd[(size_t)t * CPR] = v;
    }
    uint4* so = summ + ((size_t)dst * Hkv + h) * 2 * CPR;
    so[c] = make_uint4(bf2_key(mn.x), bf2_key(mn.y), bf2_key(mn.z), bf2_key(mn.w));
    so[CPR + c] = make_uint4(bf2_key(mx.x), bf2_key(mx.y), bf2_key(mx.z), bf2_key(mx.w));
  }
  if constexpr (CPRV > 0) {
    for (int item = threadIdx.x; item < Hkv * CPRV; item += blockDim.x) {
      const int h = item / CPRV, c = item % CPRV;
      uint4* vd = v_dst + ((size_t)dst * Hkv + h) * P * CPRV + c;
#pragma unroll 4
      for (int t = 0; t < P; ++t) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < n) {
          const int pos = prow[t];
          const int src = ptab[pos / P];
          if (src >= 0 && src < n_pool)
            v = ldg_nc_v4(v_cache + (((size_t)src * Hkv + h) * P + pos % P) * CPRV + c);
        }
        vd[(size_t)t * CPRV] = v;
      }
    }
  }
}

cudaError_t launch_prune(const sa_geom& g, const void* k_cache, const void* v_cache,
                         const int32_t* page_table, const int32_t* seq_lens, const uint8_t* keep,
                         const int32_t* free_pages, int64_t n_free, void* k_dst, void* v_dst,
                         void* summ, int32_t* new_page_table, int32_t* new_seq_lens,
                         int32_t* pos_map, int32_t* logical_len, void* ws, cudaStream_t stream) {
  const int nchunks = prune_nchunks(g);
  const int64_t width = (int64_t)g.max_pages * g.P;
  PruneWs w = carve(g, ws);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  prune_count_kernel<<<dim3(nchunks, g.B), kPruneThreads, 0, stream>>>(keep, seq_lens, width,
                                                                       nchunks, w.chunk_cnt);
  prune_plan_kernel<<<1, 1024, 0, stream>>>(seq_lens, g.B, g.P, nchunks, n_free, w.chunk_cnt,
                                            w.chunk_base, w.sess_off, w.sess_kept, new_seq_lens,
                                            logical_len, hdr);
  prune_pos_kernel<<<dim3(nchunks, g.B), kPruneThreads, 0, stream>>>(
      keep, seq_lens, free_pages, width, g.max_pages, g.P, nchunks, w.chunk_base, w.sess_off,
      w.sess_kept, pos_map, new_page_table, hdr);
  const dim3 cgrid(g.max_pages, g.B);
  const uint4* kc = static_cast<const uint4*>(k_cache);
  const uint4* vc = static_cast<const uint4*>(v_cache);
  uint4* kd = static_cast<uint4*>(k_dst);
  uint4* vd = static_cast<uint4*>(v_dst);
  uint4* sm = static_cast<uint4*>(summ);
  if (g.v_aliases_k) {
    if (g.Dk != 576) return cudaErrorInvalidValue;
    prune_copy_kernel<72, 0><<<cgrid, 96, 0, stream>>>(kc, nullptr, page_table, free_pages, g.Hkv,
                                                       g.P, g.max_pages, g.n_pool, width, pos_map, w.sess_off,
                                                       w.sess_kept, kd, nullptr, sm, hdr);
  } else if (g.Dk == 128) {
    const int th = g.Hkv * 16 < 512 ? g.Hkv * 16 : 512;
    prune_copy_kernel<16, 16><<<cgrid, th, 0, stream>>>(kc, vc, page_table, free_pages, g.Hkv, g.P,
                                                        g.max_pages, g.n_pool, width, pos_map, w.sess_off,
                                                        w.sess_kept, kd, vd, sm, hdr);
  } else if (g.Dk == 64) {
    const int th = g.Hkv * 8 < 512 ? g.Hkv * 8 : 512;
    prune_copy_kernel<8, 8><<<cgrid, th, 0, stream>>>(kc, vc, page_table, free_pages, g.Hkv, g.P,
                                                      g.max_pages, g.n_pool, width, pos_map, w.sess_off,
                                                      w.sess_kept, kd, vd, sm, hdr);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace sa
