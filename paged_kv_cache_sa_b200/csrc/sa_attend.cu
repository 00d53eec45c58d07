// sa_attend.cu -- gathered split-KV attention over the selected pages, and the merge.
//
// Method: exact softmax attention over the tokens of the selected pages (SubQ/SSA
// article, SSA section: exact attention on the chosen positions), reached through the
// page table without the caller knowing where pages live (Vortex summary, section 1),
// computed with an online softmax that never materialises the score row
// (FlashAttention paragraph of the same article), split across the selected pages
// and merged by log-sum-exp.
//
// Grouped-query kernel, one CTA per (split, KV head, sequence):
//  * a producer warp gathers each selected page's K and V blocks ([P x Dk] bf16,
//    contiguous per (page, head)) with 2-D TMA tile loads into a ring of shared-memory
//    stages (128-byte swizzle, mbarrier transaction counts, no multicast);
//  * four consumer warps take pages round-robin.  Per 16-token slice: S = Q K^T on
//    m16n8k16 tensor-core tiles (the G <= 8 query heads are the M side; K fragments
//    come from the swizzled stage with conflict-free 16-byte shared loads in a
//    permuted channel order that Q's fragments share), online softmax in registers
//    (base-2, scale folded in; row max over 4 lanes with 2 shuffles), then
//    O^T += V^T P^T with the channels as the M side so the S accumulators are
//    directly the P^T operand;
//  * warps merge their (m, l, O) in shared memory; one split writes out/lse directly,
//    several write partials that the merge kernel combines.
// HBM-bound: bytes per selected token and KV head = (Dk + Dv) * 2.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kAttnConsumerWarps = 4;

template <int D, int P>
struct AttnShape {
  // A stage holds one "unit": CT consecutive tokens of one (page, KV head), K and V.
  static constexpr int CT = P < 32 ? P : 32;            // tokens per unit
  static constexpr int UPP = P / CT;                    // units per page
  static constexpr int HALVES = D / 64;                 // 128-byte column halves per row
  static constexpr int HALF_BYTES = CT * 128;           // one TMA box: CT rows x 128 B
  static constexpr int KV_BYTES = HALVES * HALF_BYTES;  // K of one unit
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;      // K + V
  // stage count: a multiple of the consumer-warp count, so that the unit a warp waits
  // for and the previous unit of the same stage belong to the same warp (an mbarrier
  // parity wait must never run more than one phase ahead of the barrier)
  static constexpr int NST = (64 * 1024 / STAGE_BYTES) / kAttnConsumerWarps * kAttnConsumerWarps;
  static constexpr int MT = D / 16;                     // PV m-tiles (channels)
  static constexpr int JQ = D / 32;                     // 16-byte Q/K chunks per lane
  static constexpr int VC = D / 64;                     // 16-byte V chunks per lane per token
  static constexpr int COMB_BYTES = kAttnConsumerWarps * 8 * (D + 2) * 4;
  static constexpr int SMEM_BYTES = NST * STAGE_BYTES + 1024;
  static_assert(NST >= kAttnConsumerWarps && NST % kAttnConsumerWarps == 0, "stage ring");
  static_assert(COMB_BYTES <= NST * STAGE_BYTES, "combine area fits in the stages");
};

// logical 16-byte chunk (within a Dk row) that lane-group t loads for its j-th Q/K chunk
__device__ __forceinline__ int qk_chunk(int j, int t) { return (j >> 1) * 8 + 2 * t + (j & 1); }

__device__ __forceinline__ uint32_t half_of(const uint4& v, int e) {
  // 16-bit element e (0..7) of a 16-byte vector, in the low half of the result
  const uint32_t w = (e >> 1) == 0 ? v.x : (e >> 1) == 1 ? v.y : (e >> 1) == 2 ? v.z : v.w;
  return (e & 1) ? (w >> 16) : (w & 0xFFFFu);
}

template <int D, int P>
__global__ void __launch_bounds__((kAttnConsumerWarps + 1) * 32, 2)
    attend_gqa_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const uint16_t* __restrict__ q,
                      const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens,
                      const int32_t* __restrict__ sel, const int32_t* __restrict__ sel_count,
                      int sel_stride, int Hq, int Hkv, int max_pages, int n_pool, int pps,
                      int nsplit,
                      float scale_log2, float* __restrict__ part, float* __restrict__ out,
                      float* __restrict__ lse, int32_t* __restrict__ status) {
  using S = AttnShape<D, P>;
  constexpr int NW = kAttnConsumerWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[S::NST];
  __shared__ __align__(8) uint64_t empty_bar[S::NST];
  __shared__ int lp_list[256];
  __shared__ int ph_list[256];
  __shared__ int abort_flag;
  __shared__ int issued;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv;
  const int L = min(max(seq_lens[b], 0), max_pages * P);
  const int nb = (L + P - 1) / P;
  const int cnt = min(max(sel_count[(size_t)b * Hkv + h], 0), sel_stride);
  const int pbeg = split * pps;
  const int np = max(0, min(cnt, pbeg + pps) - pbeg);

  if (tid == 0) {
    for (int s = 0; s < S::NST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    abort_flag = 0;
    issued = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < np; i += blockDim.x) {
    int lp = sel[((size_t)b * Hkv + h) * sel_stride + pbeg + i];
    int ph = (lp >= 0 && lp < nb) ? page_table[(size_t)b * max_pages + lp] : -1;
    if (ph < 0 || ph >= n_pool) {  // out-of-range index: report, read page 0, mask it out
      report(status, SA_ERR_DEVICE_CHECK);
      lp = nb;
      ph = 0;
    }
    lp_list[i] = lp;
    ph_list[i] = ph;
  }
  __syncthreads();

  // per-warp softmax state (consumers)
  float m_run = -INFINITY, l_run = 0.f;
  float o[S::MT][4];
#pragma unroll
  for (int i = 0; i < S::MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int r = lane >> 2, t = lane & 3;

  if (warp == NW) {
    // ---------------- producer: TMA gather of K and V page blocks ----------------
    if (lane == 0 && np > 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
      const int nu = np * S::UPP;
      for (int i = 0; i < nu; ++i) {
        const int st = i % S::NST;
        if (i >= S::NST) {
          if (!mbar_wait(&empty_bar[st], ((i / S::NST) - 1) & 1)) {
            report(status, SA_ERR_TIMEOUT);
            atomicExch(&abort_flag, 1);
            break;
          }
        }
        if (*(volatile int*)&abort_flag) break;
        uint8_t* kdst = stages + st * S::STAGE_BYTES;
        uint8_t* vdst = kdst + S::KV_BYTES;
        const int row = (ph_list[i / S::UPP] * Hkv + h) * P + (i % S::UPP) * S::CT;
        mbar_arrive_expect_tx(&full_bar[st], S::STAGE_BYTES);
#pragma unroll
        for (int hf = 0; hf < S::HALVES; ++hf) {
          tma_load_2d(kdst + hf * S::HALF_BYTES, &kmap, hf * 64, row, &full_bar[st]);
          tma_load_2d(vdst + hf * S::HALF_BYTES, &vmap, hf * 64, row, &full_bar[st]);
        }
        issued = i + 1;
      }
    }
  } else {
    // ---------------- consumers ----------------
    // Q fragments (A operand, rows = query heads of the group; rows 8..15 are zero)
    uint4 qa[S::JQ];
    if (r < G) {
      const uint4* qrow = reinterpret_cast<const uint4*>(q + ((size_t)b * Hq + h * G + r) * D);
#pragma unroll
      for (int j = 0; j < S::JQ; ++j) qa[j] = qrow[qk_chunk(j, t)];
    } else {
#pragma unroll
      for (int j = 0; j < S::JQ; ++j) qa[j] = make_uint4(0, 0, 0, 0);
    }
    const uint32_t stage0 = smem_u32(stages);
    const int nu = np * S::UPP;
    for (int i = warp; i < nu; i += NW) {
      const int st = i % S::NST;
      if (*(volatile int*)&abort_flag) break;
      if (!mbar_wait(&full_bar[st], (i / S::NST) & 1)) {
        report(status, SA_ERR_TIMEOUT);
        atomicExch(&abort_flag, 1);
        break;
      }
      const int nv = min(S::CT, L - lp_list[i / S::UPP] * P - (i % S::UPP) * S::CT);
      const uint32_t kbase = stage0 + st * S::STAGE_BYTES;
      const uint32_t vbase = kbase + S::KV_BYTES;
#pragma unroll 1
      for (int sub = 0; sub < S::CT / 16; ++sub) {
        if (sub * 16 >= nv) break;
        // ---- S = Q K^T for 16 tokens (two n-tiles of 8) ----
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
          const int row = sub * 16 + nt * 8 + r;
#pragma unroll
          for (int j = 0; j < S::JQ; ++j) {
            const int lc = qk_chunk(j, t);
            const uint32_t addr =
                kbase + (lc >> 3) * S::HALF_BYTES + row * 128 + (((lc & 7) ^ (row & 7)) << 4);
            const uint4 kv = lds_v4(addr);
            mma_bf16_16816(sc[nt], qa[j].x, 0u, qa[j].y, 0u, kv.x, kv.y);
            mma_bf16_16816(sc[nt], qa[j].z, 0u, qa[j].w, 0u, kv.z, kv.w);
          }
        }
        // ---- online softmax (rows = query head r; lanes t hold tokens 2t,2t+1,8+2t,9+2t)
        float x[4];
        x[0] = sc[0][0] * scale_log2;
        x[1] = sc[0][1] * scale_log2;
        x[2] = sc[1][0] * scale_log2;
        x[3] = sc[1][1] * scale_log2;
        const int tok0 = sub * 16 + 2 * t;
        if (tok0 >= nv) x[0] = -INFINITY;
        if (tok0 + 1 >= nv) x[1] = -INFINITY;
        if (tok0 + 8 >= nv) x[2] = -INFINITY;
        if (tok0 + 9 >= nv) x[3] = -INFINITY;
        float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const float m_new = fmaxf(m_run, mt);  // finite: token 0 of a slice is valid
        const float alpha = fast_exp2(m_run - m_new);
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = fast_exp2(x[e] - m_new);
        l_run = l_run * alpha + (p[0] + p[1]) + (p[2] + p[3]);
        m_run = m_new;
        const float al0 = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
        const float al1 = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
#pragma unroll
        for (int i2 = 0; i2 < S::MT; ++i2) {
          o[i2][0] *= al0; o[i2][1] *= al1; o[i2][2] *= al0; o[i2][3] *= al1;
        }
        const uint32_t pb0 = pack_bf16(p[0], p[1]);
        const uint32_t pb1 = pack_bf16(p[2], p[3]);
        // ---- O^T += V^T P^T: lane loads channels [D/8*r, D/8*r + D/8) of 4 tokens ----
        uint4 xv[4][S::VC];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int tk = sub * 16 + 2 * t + (k & 1) + (k >> 1) * 8;
#pragma unroll
          for (int c = 0; c < S::VC; ++c) {
            const int lc = (D / 64) * r + c;  // logical chunk: channels 8*lc .. 8*lc+7
            const uint32_t addr =
                vbase + (lc >> 3) * S::HALF_BYTES + tk * 128 + (((lc & 7) ^ (tk & 7)) << 4);
            xv[k][c] = lds_v4(addr);
          }
        }
        // tokens past nv carry p = 0 but their V slots may hold anything: zero them
        if (tok0 >= nv) {
#pragma unroll
          for (int c = 0; c < S::VC; ++c) xv[0][c] = make_uint4(0, 0, 0, 0);
        }
        if (tok0 + 1 >= nv) {
#pragma unroll
          for (int c = 0; c < S::VC; ++c) xv[1][c] = make_uint4(0, 0, 0, 0);
        }
        if (tok0 + 8 >= nv) {
#pragma unroll
          for (int c = 0; c < S::VC; ++c) xv[2][c] = make_uint4(0, 0, 0, 0);
        }
        if (tok0 + 9 >= nv) {
#pragma unroll
          for (int c = 0; c < S::VC; ++c) xv[3][c] = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i2 = 0; i2 < S::MT; ++i2) {
          // channel rows: phi(i2, r) = (D/8) r + i2, phi(i2, r+8) = (D/8) r + MT + i2
          const int e0 = i2, e1 = S::MT + i2;
          const uint32_t lo0 = half_of(xv[0][e0 >> 3], e0 & 7), hi0 = half_of(xv[1][e0 >> 3], e0 & 7);
          const uint32_t lo1 = half_of(xv[0][e1 >> 3], e1 & 7), hi1 = half_of(xv[1][e1 >> 3], e1 & 7);
          const uint32_t lo2 = half_of(xv[2][e0 >> 3], e0 & 7), hi2 = half_of(xv[3][e0 >> 3], e0 & 7);
          const uint32_t lo3 = half_of(xv[2][e1 >> 3], e1 & 7), hi3 = half_of(xv[3][e1 >> 3], e1 & 7);
          mma_bf16_16816(o[i2], lo0 | (hi0 << 16), lo1 | (hi1 << 16), lo2 | (hi2 << 16),
                         lo3 | (hi3 << 16), pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }
    // reduce l over the 4 lanes of a head row
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  }
  __syncthreads();

  if (abort_flag) {
    // a wait expired: let any copy still in flight land (bounded), then leave
    if (warp == NW && lane == 0) {
      for (int i = max(0, issued - S::NST); i < issued; ++i)  // units
        (void)mbar_wait(&full_bar[i % S::NST], (i / S::NST) & 1);
    }
    return;
  }

  // ---------------- merge the consumer warps (stages are free now) ----------------
  float* cm = reinterpret_cast<float*>(stages);  // [NW][8]
  float* cl = cm + NW * 8;                        // [NW][8]
  float* co = cl + NW * 8;                        // [NW][8][D]
  if (warp < NW) {
    if (t == 0) {
      cm[warp * 8 + r] = m_run;
      cl[warp * 8 + r] = l_run;
    }
#pragma unroll
    for (int i2 = 0; i2 < S::MT; ++i2) {
      const int c0 = (D / 8) * r + i2, c1 = (D / 8) * r + S::MT + i2;
      co[(warp * 8 + 2 * t) * D + c0] = o[i2][0];
      co[(warp * 8 + 2 * t + 1) * D + c0] = o[i2][1];
      co[(warp * 8 + 2 * t) * D + c1] = o[i2][2];
      co[(warp * 8 + 2 * t + 1) * D + c1] = o[i2][3];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int gi = idx / D, c = idx % D;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mstar = fmaxf(mstar, cm[w * 8 + gi]);
    float lsum = 0.f, osum = 0.f;
    if (mstar != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = cm[w * 8 + gi];
        if (mw == -INFINITY) continue;
        const float f = fast_exp2(mw - mstar);
        lsum += cl[w * 8 + gi] * f;
        osum += co[(w * 8 + gi) * D + c] * f;
      }
    }
    const int hq = h * G + gi;
    if (nsplit == 1) {
      out[((size_t)b * Hq + hq) * D + c] = lsum > 0.f ? osum / lsum : 0.f;
      if (c == 0)
        lse[(size_t)b * Hq + hq] =
            lsum > 0.f ? (mstar + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
    } else {
      float* pr = part + ((((size_t)b * Hkv + h) * nsplit + split) * G + gi) * (D + 2);
      pr[c] = osum;
      if (c == 0) {
        pr[D] = mstar;
        pr[D + 1] = lsum;
      }
    }
  }
}

// Combine the split partials of one (sequence, KV head): m* = max m_s,
// l = sum l_s 2^(m_s - m*), o = sum o_s 2^(m_s - m*) / l, lse = (m* + log2 l) ln 2.
template <int D>
__global__ void merge_kernel(const float* __restrict__ part, int Hq, int Hkv, int nsplit,
                             float* __restrict__ out, float* __restrict__ lse) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = Hq / Hkv;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int gi = idx / D, c = idx % D;
    const float* base = part + (((size_t)b * Hkv + h) * nsplit * G + gi) * (D + 2);
    const size_t stride = (size_t)G * (D + 2);
    float mstar = -INFINITY;
    for (int s = 0; s < nsplit; ++s) mstar = fmaxf(mstar, base[s * stride + D]);
    float lsum = 0.f, osum = 0.f;
    if (mstar != -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const float ms = base[s * stride + D];
        if (ms == -INFINITY) continue;
        const float f = fast_exp2(ms - mstar);
        lsum += base[s * stride + D + 1] * f;
        osum += base[s * stride + c] * f;
      }
    }
    const int hq = h * G + gi;
    out[((size_t)b * Hq + hq) * D + c] = lsum > 0.f ? osum / lsum : 0.f;
    if (c == 0)
      lse[(size_t)b * Hq + hq] =
          lsum > 0.f ? (mstar + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
  }
}

template <int D, int P>
static cudaError_t launch_attend_t(const sa_geom& g, const DecodePlan& plan, const void* q,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* page_table, const int32_t* seq_lens,
                                   const int32_t* sel, const int32_t* sel_count, int sel_stride,
                                   float scale, float* part, float* out, float* lse,
                                   int32_t* status, cudaStream_t stream) {
  using S = AttnShape<D, P>;
  CUtensorMap kmap, vmap;
  const uint64_t rows = (uint64_t)g.n_pool * g.Hkv * P;
  if (!encode_rows_tmap(&kmap, k_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  if (!encode_rows_tmap(&vmap, v_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attend_gqa_kernel<D, P>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(plan.nsplit, g.Hkv, g.B);
  const float scale_log2 = scale * 1.4426950408889634f;
  attend_gqa_kernel<D, P><<<grid, (kAttnConsumerWarps + 1) * 32, S::SMEM_BYTES, stream>>>(
      kmap, vmap, static_cast<const uint16_t*>(q), page_table, seq_lens, sel, sel_count,
      sel_stride, g.Hq, g.Hkv, g.max_pages, g.n_pool, plan.pps, plan.nsplit, scale_log2, part,
      out, lse, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || plan.nsplit == 1) return e;
  dim3 mgrid(g.Hkv, g.B);
  const int threads = plan.G * D < 1024 ? plan.G * D : 1024;
  merge_kernel<D><<<mgrid, threads, 0, stream>>>(part, g.Hq, g.Hkv, plan.nsplit, out, lse);
  return cudaGetLastError();
}

cudaError_t launch_attend(const sa_geom& g, const DecodePlan& plan, const void* q,
                          const void* k_cache, const void* v_cache, const int32_t* page_table,
                          const int32_t* seq_lens, const int32_t* sel, const int32_t* sel_count,
                          int sel_stride, float scale, float* part, float* out, float* lse,
                          int32_t* status, cudaStream_t stream) {
#define SA_ATTEND_CASE(DD, PP)                                                                 \
  if (g.Dk == DD && g.P == PP)                                                                 \
    return launch_attend_t<DD, PP>(g, plan, q, k_cache, v_cache, page_table, seq_lens, sel,    \
                                   sel_count, sel_stride, scale, part, out, lse, status, stream);
  SA_ATTEND_CASE(64, 16)
  SA_ATTEND_CASE(64, 32)
  SA_ATTEND_CASE(64, 64)
  SA_ATTEND_CASE(128, 16)
  SA_ATTEND_CASE(128, 32)
  SA_ATTEND_CASE(128, 64)
#undef SA_ATTEND_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
