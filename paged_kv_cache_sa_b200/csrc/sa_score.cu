// sa_score.cu -- page scoring (the query-aware page bound) for grouped-query heads.
//
// Method ("SparseEngine" blog, hook-point paragraph: Quest chooses decode pages from
// the current query): S(b,h,p) = max over the query heads g of KV head h of
//   u_g(p) = sum_c max(q_gc * kmax_c, q_gc * kmin_c).
// Because kmax >= kmin, max(q*kmax, q*kmin) = max(q,0)*kmax + min(q,0)*kmin exactly,
// so u = [kmin | kmax] . [min(q,0) | max(q,0)]: a contraction of length 2*Dk.  Every
// bf16 x bf16 product is exact in fp32; accumulation is fp32.
//
// The G <= 8 query heads of a group are the N=8 side of one m16n8k16 tensor-core tile
// and 16 pages are its M side.  The A fragments are loaded straight from HBM: each
// lane reads 16-byte vectors of two summary rows, and the channel order inside the
// contraction is permuted so that every 16-byte vector lands in the fragment slots
// of the lane that loaded it (the same permutation is applied to the query side, so
// the sum is unchanged).  A warp-level load instruction covers 64 contiguous bytes of
// each of 8 rows: every 32-byte sector fetched is used.  The GQA max-reduction is a
// register max plus two warp shuffles.  HBM-bound: bytes per (page, KV head) =
// 2 * Dk * 2 (summary) + 4 (page-table entry) + 4 (score written).
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

template <int D, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    score_gqa_kernel(const uint16_t* __restrict__ q, const uint4* __restrict__ summ,
                     const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens,
                     float* __restrict__ scores, int Hq, int Hkv, int P, int max_pages,
                     int n_pool, int32_t* __restrict__ status) {
  constexpr int NCH = 2 * D / 8;  // 16-byte chunks per summary row [kmin | kmax]
  constexpr int J = NCH / 4;      // chunks per lane per row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, t = lane & 3;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv;
  const int L = min(max(seq_lens[b], 0), max_pages * P);
  const int nb = (L + P - 1) / P;
  const int p0 = (blockIdx.x * WARPS + warp) * 16;
  if (p0 >= max_pages) return;
  float* srow = scores + ((size_t)b * Hkv + h) * max_pages;
  if (p0 >= nb) {  // whole tile past the sequence: scores are -inf there
    if (lane < 16 && p0 + lane < max_pages) srow[p0 + lane] = -INFINITY;
    return;
  }

  // A: summary rows of pages p0 + r and p0 + r + 8 (chunk 4j + t of each row)
  const int pa = p0 + r, pb = p0 + r + 8;
  uint4 ra[J], rb[J];
  {
    const uint4* rowa = nullptr;
    const uint4* rowb = nullptr;
    const int qa_ = pa < nb ? page_table[(size_t)b * max_pages + pa] : 0;
    const int qb_ = pb < nb ? page_table[(size_t)b * max_pages + pb] : 0;
    if ((qa_ < 0 || qa_ >= n_pool || qb_ < 0 || qb_ >= n_pool) && t == 0)
      report(status, SA_ERR_DEVICE_CHECK);
    if (pa < nb && qa_ >= 0 && qa_ < n_pool) rowa = summ + ((size_t)qa_ * Hkv + h) * NCH;
    if (pb < nb && qb_ >= 0 && qb_ < n_pool) rowb = summ + ((size_t)qb_ * Hkv + h) * NCH;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      ra[j] = rowa ? ldg_nc_v4(rowa + 4 * j + t) : make_uint4(0, 0, 0, 0);
      rb[j] = rowb ? ldg_nc_v4(rowb + 4 * j + t) : make_uint4(0, 0, 0, 0);
    }
  }

  // B: [min(q,0) | max(q,0)] of query head n = r of the group, same chunk order
  uint4 bq[J];
  if (r < G) {
    const uint4* qrow = reinterpret_cast<const uint4*>(q + ((size_t)b * Hq + h * G + r) * D);
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int c = 4 * j + t;  // chunk of the 2D-long contraction
      uint4 v = qrow[c % (D / 8)];
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t neg = ((w[e] >> 15) & 0x00010001u) * 0xFFFFu;  // halves with sign bit set
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
    if (pa < max_pages) srow[pa] = pa < nb ? m0 : -INFINITY;
    if (pb < max_pages) srow[pb] = pb < nb ? m1 : -INFINITY;
  }
}

cudaError_t launch_score(const sa_geom& g, const void* q, const void* summ,
                         const int32_t* page_table, const int32_t* seq_lens, float* scores,
                         int32_t* status, cudaStream_t stream) {
  constexpr int WARPS = 4;
  dim3 grid((g.max_pages + 16 * WARPS - 1) / (16 * WARPS), g.Hkv, g.B);
  const uint16_t* qq = static_cast<const uint16_t*>(q);
  const uint4* s = static_cast<const uint4*>(summ);
  switch (g.Dk) {
    case 64:
      score_gqa_kernel<64, WARPS><<<grid, WARPS * 32, 0, stream>>>(
          qq, s, page_table, seq_lens, scores, g.Hq, g.Hkv, g.P, g.max_pages, g.n_pool, status);
      break;
    case 128:
      score_gqa_kernel<128, WARPS><<<grid, WARPS * 32, 0, stream>>>(
          qq, s, page_table, seq_lens, scores, g.Hq, g.Hkv, g.P, g.max_pages, g.n_pool, status);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace sa
