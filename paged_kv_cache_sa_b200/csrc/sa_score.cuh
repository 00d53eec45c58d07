// sa_score.cuh -- device code of the page scoring and the top-k selection: the scoring
// grid's CTA program and the per-(sequence, KV head) selection, as functions that the
// separate kernels (sa_score.cu) and the single-launch decode (sa_fused.cu) run.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sa_common.cuh"
#include "sa_fp8.cuh"
#include "sa_internal.h"
#include "sa_select.cuh"

namespace sa {

constexpr int kTilePages = 16;  // pages per tile: the M side of one MMA
constexpr int kScoreConsumers = 8;
constexpr int kScoreThreads = (kScoreConsumers + 1) * 32;
constexpr int kMaxTilesPerCta = 64;
constexpr int kSlotPad = 64;  // odd multiple of 64 B between page slots: no bank conflicts
constexpr int kSelectThreads = 512;
constexpr int kScoreSmemLimit = 227 * 1024;

struct ScoreArgs {
  const uint16_t* q;
  const uint8_t* summ;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;  // [B][Hkv][max_pages]
  int32_t* status;
  const uint4* k_cache;  // non-null: refresh the newest n_tail pages' summaries from K first
  uint4* summ_w;         // the summaries (bf16 rows or fp8 records), written by that refresh
  int n_tail;
  int B, Hq, Hkv, G, P, max_pages, n_pool;
  int HG, n_hg, WPS, NST;              // heads per tile, head groups, warp groups, stages
  int slot_bytes, q_off, stage_bytes;  // stage: [16][slot_bytes] page slots | q rows
  int rec_bytes;                       // summary bytes per (page, KV head)
};

// Four E4M3 codes (bytes of w, lowest first) as two bf16x2 words, exactly: the
// hardware e4m3x2 -> f16x2 conversion, then f16 -> f32 -> bf16 (no rounding anywhere:
// every E4M3 value has at most 4 significant bits within the exponent range of both).
__device__ __forceinline__ void e4m3x4_to_bf16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const __half2 a = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  const __half2 b = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const float2 fa = __half22float2(a), fb = __half22float2(b);
  const __nv_bfloat162 ba = __floats2bfloat162_rn(fa.x, fa.y);
  const __nv_bfloat162 bb = __floats2bfloat162_rn(fb.x, fb.y);
  lo = *reinterpret_cast<const uint32_t*>(&ba);
  hi = *reinterpret_cast<const uint32_t*>(&bb);
}

// the sequence owning flattened tile u: largest b with pre[b] <= u
__device__ __forceinline__ int find_seq(const int* pre, int n, int u) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// fp8 form of the decode-time refresh (one warp): the page's min/max rows from K, encoded
// into the record exactly as the summaries kernel encodes them and stored, and in every
// lane the page's score over the decoded record (max over the G heads, then the
// record's 2^e, as the stream applies it).
template <int D>
__device__ float warp_refresh_and_score_fp8(const uint4* __restrict__ k_cache,
                                            uint8_t* __restrict__ summ8, const uint16_t* qh,
                                            int G, int phys, int h, int Hkv, int P, int valid,
                                            int lane) {
  constexpr int CPR = D / 8;
  uint4 qv[8];
  warp_load_q<D>(qh, G, lane, qv);
  uint4 kmin, kmax;
  warp_page_minmax<D>(k_cache, phys, h, Hkv, P, valid, lane, kmin, kmax);
  uint32_t am = max_mag2(max_mag2(max_mag2(max_mag2(0u, kmin.x), kmin.y), kmin.z), kmin.w);
  am = max_mag2(max_mag2(max_mag2(max_mag2(am, kmax.x), kmax.y), kmax.z), kmax.w);
  am = __reduce_max_sync(0xffffffffu, am);
  const int e = fp8_record_exp(am);
  const uint2 cmin = make_uint2(e4m3_pack(kmin.x, kmin.y, e, false),
                                e4m3_pack(kmin.z, kmin.w, e, false));
  const uint2 cmax = make_uint2(e4m3_pack(kmax.x, kmax.y, e, true),
                                e4m3_pack(kmax.z, kmax.w, e, true));
  uint8_t* rec = summ8 + ((size_t)phys * Hkv + h) * (2 * D + 16);
  const int c = lane % CPR;
  if (lane < CPR) {
    *reinterpret_cast<uint2*>(rec + c * 8) = cmin;
    *reinterpret_cast<uint2*>(rec + D + c * 8) = cmax;
  }
  if (lane == 0)
    *reinterpret_cast<uint4*>(rec + 2 * D) = make_uint4((uint32_t)e & 0xFFu, 0u, 0u, 0u);
  uint32_t lo[4], hi[4];
  e4m3x4_to_bf16(cmin.x, lo[0], lo[1]);
  e4m3x4_to_bf16(cmin.y, lo[2], lo[3]);
  e4m3x4_to_bf16(cmax.x, hi[0], hi[1]);
  e4m3x4_to_bf16(cmax.y, hi[2], hi[3]);
  return ldexpf(warp_bound_score<D>(qv, G, lane, lo, hi), e);
}

// Tiles per sequence (n_hg * ceil(pages / 16)) prefix-summed over the batch by one warp;
// returns the total.  With pre/nbs non-null the prefix and page counts are stored.
__device__ __forceinline__ int tile_prefix(const ScoreArgs& a, int lane, int* pre, int* nbs) {
  int carry = 0;
  for (int b0 = 0; b0 < a.B; b0 += 32) {
    const int b = b0 + lane;
    int n = 0;
    if (b < a.B) {
      const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
      const int nb = (L + a.P - 1) / a.P;
      n = a.n_hg * ((nb + kTilePages - 1) / kTilePages);
      if (nbs) nbs[b] = nb;
    }
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (pre && b < a.B) pre[b] = carry + incl - n;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (pre && lane == 0) pre[a.B] = carry;
  return carry;
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}

// The scoring grid's CTA program (kScoreThreads threads), on `smem_raw` (dynamic shared
// memory of score_smem bytes).
template <int D, bool F8>
__device__ __forceinline__ void score_stream_body(const ScoreArgs& a, uint8_t* smem_raw) {
  constexpr int J = D / 16;  // 16-byte chunks per lane of the 2*D-long contraction row
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  int* pre = reinterpret_cast<int*>(stages + (size_t)a.NST * a.stage_bytes);  // [B + 1]
  int* nbs = pre + a.B + 1;                        // [B] pages per sequence
  int* ptab = nbs + a.B;                           // [kMaxTilesPerCta * 16]
  int* t_b = ptab + kMaxTilesPerCta * kTilePages;  // per tile of the slice
  int* t_hg = t_b + kMaxTilesPerCta;
  int* t_p0 = t_hg + kMaxTilesPerCta;
  int* t_np = t_p0 + kMaxTilesPerCta;  // pages in the tile
  int* t_vm = t_np + kMaxTilesPerCta;  // mask of pages with a valid slot
  __shared__ __align__(8) uint64_t full_bar[8];
  __shared__ __align__(8) uint64_t empty_bar[8];
  __shared__ int abort_flag;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, n_cta = gridDim.x;
  if (tid == 0) SA_TRACE_POINT(0, 0);  // entry

  if (tid == 0) {
    for (int s = 0; s < a.NST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], a.HG);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  // everything read below may come from the previous kernel of the stream: one thread
  // waits for it (which makes its memory visible to this grid), the rest block on the
  // CTA barrier.  No early launch of the next grid: the selection grid would start while
  // most SMs still stream, and its CTAs would pile onto the first SMs to free up (several
  // per SM, contending); launched as this grid exits, they spread over idle SMs.
  if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  if (tid == 0) SA_TRACE_POINT(0, 1);  // dependency wait passed

  // The slice of the flattened tile list this CTA streams: every warp derives it from
  // the sequence lengths itself, so no CTA-wide barrier stands before the first copy.
  // Per-tile tables are written by the producer before it arrives on the tile's stage
  // barrier (release), and read by the consumers after waiting on it (acquire).
  const bool is_prod = warp == kScoreConsumers;
  const int total = tile_prefix(a, lane, is_prod ? pre : nullptr, is_prod ? nbs : nullptr);
  const int W = max(1, (total + n_cta - 1) / n_cta);
  const int T0 = min(total, c * W);
  const int nt = min(total, T0 + W) - T0;  // <= kMaxTilesPerCta (the host sizes the grid)

  if (is_prod) {
    // ===================== producer warp =====================
    __syncwarp();
    // 1. per tile of the slice (one lane each): sequence, head group, first page, page
    //    count; its page-table entries gathered by asynchronous 4-byte copies, all in
    //    flight together
    for (int i = lane; i < nt; i += 32) {
      const int u = T0 + i;
      const int b = find_seq(pre, a.B, u);
      const int ntb = (pre[b + 1] - pre[b]) / a.n_hg;  // tiles per head group
      const int rem = u - pre[b];
      const int p0 = (rem % ntb) * kTilePages;
      const int np = min(kTilePages, nbs[b] - p0);
      t_b[i] = b;
      t_hg[i] = rem / ntb;
      t_p0[i] = p0;
      t_np[i] = np;
      const int32_t* src = a.page_table + (size_t)b * a.max_pages + p0;
      for (int pg = 0; pg < np; ++pg) cp_async4(ptab + i * kTilePages + pg, src + pg);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
    __syncwarp();
    if (lane == 0) SA_TRACE_POINT(0, 2);  // slice tables ready

    // 2. bulk-copy issue: lanes 0-15 check and copy one page each, lane 16 the queries
    const uint32_t slot_data = (uint32_t)a.HG * a.rec_bytes;  // one page's records of the group
    const uint32_t q_bytes = (uint32_t)a.HG * a.G * D * 2;
    uint64_t t_idle = 0;
    const uint64_t ef = l2_evict_first();
    for (int k = 0; k < nt;) {
      const int s = k % a.NST;
      bool ready = k < a.NST;
      if (!ready && lane == 0) ready = mbar_test(&empty_bar[s], ((k / a.NST) - 1) & 1);
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) {
        const uint64_t now = global_ns();
        if (t_idle == 0) t_idle = now;
        const int to = (now - t_idle > kWaitLimitNs) || *(volatile int*)&abort_flag;
        if (__shfl_sync(0xffffffffu, to, 0)) {
          if (lane == 0) {
            report(a.status, SA_ERR_TIMEOUT);
            atomicExch(&abort_flag, 1);
          }
          break;
        }
        continue;
      }
      t_idle = 0;
      const int b = t_b[k], hg = t_hg[k], np = t_np[k];
      const int ph = lane < np ? ptab[k * kTilePages + lane] : -1;
      const bool ok = ph >= 0 && ph < a.n_pool;
      if (lane < np && !ok) report(a.status, SA_ERR_DEVICE_CHECK);
      const int vm = (int)(__ballot_sync(0xffffffffu, ok) & 0xFFFFu);
      uint8_t* st = stages + (size_t)s * a.stage_bytes;
      if (lane == 0) {
        t_vm[k] = vm;
        mbar_arrive_expect_tx(&full_bar[s], __popc(vm) * slot_data + q_bytes);
      }
      __syncwarp();
      if (ok) {
        bulk_load_hint(st + lane * a.slot_bytes,
                       a.summ + ((size_t)ph * a.Hkv + hg * a.HG) * (size_t)a.rec_bytes,
                       slot_data, &full_bar[s], ef);
      } else if (lane == kTilePages) {
        bulk_load(st + a.q_off, a.q + ((size_t)b * a.Hq + (size_t)hg * a.HG * a.G) * D, q_bytes,
                  &full_bar[s]);
      }
      ++k;
    }
  } else {
    // ===================== consumer warps =====================
    // 0. decode-time refresh of the newest pages' summaries from K (the pages that
    //    received appended tokens), spread over the grid's consumer warps while the first
    //    copies are in flight.  Their scores replace the streamed ones (the stream skips
    //    those pages), so the stream may read either version of the summaries.
    {
      const int n_items = a.B * a.Hkv * a.n_tail;
      for (int i = c + n_cta * warp; i < n_items; i += n_cta * kScoreConsumers) {
        const int pr = i / a.n_tail;
        const int b = pr / a.Hkv, h = pr % a.Hkv;
        const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
        const int lp = (L + a.P - 1) / a.P - a.n_tail + i % a.n_tail;
        if (lp < 0) continue;
        const int ph = a.page_table[(size_t)b * a.max_pages + lp];
        float sc = 0.f;
        if (ph >= 0 && ph < a.n_pool) {
          const uint16_t* qh = a.q + ((size_t)b * a.Hq + h * a.G) * D;
          const int valid = min(a.P, L - lp * a.P);
          if constexpr (F8)
            sc = warp_refresh_and_score_fp8<D>(a.k_cache, reinterpret_cast<uint8_t*>(a.summ_w),
                                               qh, a.G, ph, h, a.Hkv, a.P, valid, lane);
          else
            sc = warp_refresh_and_score<D>(a.k_cache, a.summ_w, qh, a.G, ph, h, a.Hkv, a.P,
                                           valid, lane);
        }
        if (lane == 0) a.scores[(size_t)pr * a.max_pages + lp] = sc;
      }
    }
    const int r = lane >> 2, t = lane & 3;
    const int grp = warp / a.HG, hh = warp % a.HG;  // stage group, head within the group
    const bool v0 = 2 * t < a.G, v1 = 2 * t + 1 < a.G;
    for (int k = grp; k < nt; k += a.WPS) {
      const int s = k % a.NST;
      bool ok = !*(volatile int*)&abort_flag;
      if (ok && !mbar_wait(&full_bar[s], (k / a.NST) & 1)) {
        report(a.status, SA_ERR_TIMEOUT);
        atomicExch(&abort_flag, 1);
        ok = false;
      }
      if (ok && k == grp && lane == 0 && warp == 0) SA_TRACE_POINT(0, 3);  // first stage
      if (ok) {
        const int b = t_b[k], h = t_hg[k] * a.HG + hh, p0 = t_p0[k], np = t_np[k];
        const int vm = t_vm[k];
        const uint32_t st = smem_u32(stages + (size_t)s * a.stage_bytes);
        // B: [min(q,0) | max(q,0)] of query head n = r of KV head h, chunk 4j + t
        uint32_t bq[J][4];
        const uint32_t qrow = st + a.q_off + (uint32_t)(hh * a.G + (r < a.G ? r : 0)) * D * 2;
#pragma unroll
        for (int j = 0; j < J; ++j) {
          const int cc = 4 * j + t;  // chunk of the 2D-long contraction
          const uint4 v = lds_v4(qrow + (cc % (D / 8)) * 16);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t neg = ((w[e] >> 15) & 0x00010001u) * 0xFFFFu;  // negative halves
            bq[j][e] = r < a.G ? ((cc < D / 8) ? (w[e] & neg) : (w[e] & ~neg)) : 0u;
          }
        }
        // A: rows r and r + 8 of the tile (pages p0 + r, p0 + r + 8)
        const bool va = (vm >> r) & 1, vb = (vm >> (r + 8)) & 1;
        const uint32_t rowa = st + r * a.slot_bytes + hh * a.rec_bytes;
        const uint32_t rowb = rowa + 8 * a.slot_bytes;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < J; ++j) {
          uint4 ra, rb;
          if constexpr (F8) {
            // chunk 4j + t of the contraction = 8 codes (channels of the same q chunk)
            const uint2 ca = va ? lds_v2(rowa + (4 * j + t) * 8) : make_uint2(0, 0);
            const uint2 cb = vb ? lds_v2(rowb + (4 * j + t) * 8) : make_uint2(0, 0);
            e4m3x4_to_bf16(ca.x, ra.x, ra.y);
            e4m3x4_to_bf16(ca.y, ra.z, ra.w);
            e4m3x4_to_bf16(cb.x, rb.x, rb.y);
            e4m3x4_to_bf16(cb.y, rb.z, rb.w);
          } else {
            ra = va ? lds_v4(rowa + (4 * j + t) * 16) : make_uint4(0, 0, 0, 0);
            rb = vb ? lds_v4(rowb + (4 * j + t) * 16) : make_uint4(0, 0, 0, 0);
          }
          mma_bf16_16816(acc, ra.x, rb.x, ra.y, rb.y, bq[j][0], bq[j][1]);
          mma_bf16_16816(acc, ra.z, rb.z, ra.w, rb.w, bq[j][2], bq[j][3]);
        }
        // acc: [page r][heads 2t, 2t+1], [page r+8][heads 2t, 2t+1]
        float m0 = fmaxf(v0 ? acc[0] : -INFINITY, v1 ? acc[1] : -INFINITY);
        float m1 = fmaxf(v0 ? acc[2] : -INFINITY, v1 ? acc[3] : -INFINITY);
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
        if constexpr (F8) {
          // the records' exponents (an invalid page scored 0 stays 0)
          const uint8_t* sp = stages + (size_t)s * a.stage_bytes + hh * a.rec_bytes + 2 * D;
          m0 = ldexpf(m0, (int)(int8_t)sp[r * a.slot_bytes]);
          m1 = ldexpf(m1, (int)(int8_t)sp[(r + 8) * a.slot_bytes]);
        }
        if (t == 0) {
          // pages refreshed above keep the score computed from their fresh summary
          const int lim = a.n_tail > 0 ? min(np, nbs[b] - a.n_tail - p0) : np;
          float* srow = a.scores + ((size_t)b * a.Hkv + h) * a.max_pages + p0;
          if (r < lim) srow[r] = m0;
          if (r + 8 < lim) srow[r + 8] = m1;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
  }
  if (lane == 0 && warp == 0) SA_TRACE_POINT(0, 4);  // consumer 0 done
  if (warp == kScoreConsumers) {
    // scores past each sequence's last page are -inf (pairs spread over the CTAs)
    for (int pr = c; pr < a.B * a.Hkv; pr += n_cta) {
      const int b = pr / a.Hkv;
      const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
      float* srow = a.scores + (size_t)pr * a.max_pages;
      for (int p = (L + a.P - 1) / a.P + lane; p < a.max_pages; p += 32) srow[p] = -INFINITY;
    }
  }
  __syncthreads();
  if (abort_flag && warp == kScoreConsumers && lane == 0) {
    // a wait expired: give copies still in flight a bounded time (10 ms) to land
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 10000000ull) {
    }
  }
}

struct SelectArgs {
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;       // [B][Hkv][max_pages]
  int32_t* sel;        // [B][Hkv][K]
  int32_t* sel_count;  // [B][Hkv]
  int32_t* sel_phys;   // [B][Hkv][K] physical pages of the selection (nullable)
  int32_t* status;
  int Hkv, P, max_pages, K, s_pages, w_pages;
  int ptab_in_smem;  // the sequence's page-table row is staged next to the keys
};

// The selection of (sequence b, KV head h) by the first NT threads of the CTA (Bar
// synchronises them): keys (and the page table when a.ptab_in_smem) in `keys`, scratch
// in `sh`.
template <int NT, class Bar>
__device__ __forceinline__ void select_body(const SelectArgs& a, int b, int h, uint32_t* keys,
                                            const SelScratch& sh) {
  uint32_t* red = sh.red;
  int* warp_tot = sh.warp_tot;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // The scoring grid passed its own wait before letting this grid start, so the
  // inputs of the call (everything but the scores) are complete here.
  const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
  const int nb = (L + a.P - 1) / a.P;
  const int32_t* ptab_g = a.page_table + (size_t)b * a.max_pages;
  float* srow = a.scores + ((size_t)b * a.Hkv + h) * a.max_pages;
  // 1. wait for the scores (one thread; the rest block on the CTA barrier)
  if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  Bar::sync();
  asm volatile("griddepcontrol.launch_dependents;");
  if (tid == 0) SA_TRACE_POINT(1, 0);  // scores visible
  int32_t* out = a.sel + ((size_t)b * a.Hkv + h) * a.K;
  int32_t* cnt_out = a.sel_count + (size_t)b * a.Hkv + h;
  int32_t* phys_out = a.sel_phys ? a.sel_phys + ((size_t)b * a.Hkv + h) * a.K : nullptr;
  const int K = a.K;
  if (nb <= K) {  // everything fits the budget
    for (int i = tid; i < K; i += NT) {
      out[i] = i < nb ? i : -1;
      if (phys_out) phys_out[i] = i < nb ? ptab_g[i] : -1;
    }
    if (tid == 0) *cnt_out = nb;
    return;
  }
  int32_t* ptab_s = a.ptab_in_smem ? reinterpret_cast<int32_t*>(keys + a.max_pages) : nullptr;
  // 2. keys (8 loads in flight per thread) and the candidates' key range.  The
  //    page-table row goes to shared memory by asynchronous copies (no registers held),
  //    waited for before the list is written.
  const int wbeg = nb - a.w_pages;
  uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
  for (int p0 = 0; p0 < nb; p0 += NT * 8) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int p = p0 + k * NT + tid;
      v[k] = p < nb ? __ldcg(srow + p) : 0.f;
    }
    if (ptab_s) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int p = p0 + k * NT + tid;
        if (p < nb) cp_async4(ptab_s + p, ptab_g + p);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int p = p0 + k * NT + tid;
      if (p < nb) {
        const bool forced = p < a.s_pages || p >= wbeg;
        const uint32_t key = forced ? 0u : f32_order_key(v[k]);
        keys[p] = key;
        if (!forced) {
          kmn = min(kmn, key);
          kmx = max(kmx, key);
        }
      }
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (tid == 0) SA_TRACE_POINT(1, 4);  // this thread's keys stored
  block_key_range<NT, Bar>(kmn, kmx, red);
  if (tid == 0) SA_TRACE_POINT(1, 1);  // keys and their range

  // 3. threshold: a candidate is taken when its key >= thr or it was marked kWin
  const uint64_t thr = radix_select_threshold<NT, Bar>(keys, nb, a.s_pages, wbeg,
                                                       K - a.s_pages - a.w_pages, kmn, kmx, sh);
  if (tid == 0) SA_TRACE_POINT(1, 2);  // threshold

  // 4. ascending list: forced pages and taken candidates.  Each warp owns a contiguous
  // run of pages (a multiple of 32) and compacts it with ballots; one block barrier
  // gives every warp its offset.
  auto taken = [&](int p) {
    if (p < a.s_pages || p >= wbeg) return true;
    const uint32_t key = keys[p];
    return key == kWin || (uint64_t)key >= thr;
  };
  const int per_warp = ((nb + NT - 1) / NT) * 32;
  const int w0 = min(nb, warp * per_warp), w1 = min(nb, w0 + per_warp);
  int n_sel = 0;
  for (int p0 = w0; p0 < w1; p0 += 32) {
    const int p = p0 + lane;
    n_sel += __popc(__ballot_sync(0xffffffffu, p < w1 && taken(p)));
  }
  if (lane == 0) warp_tot[warp] = n_sel;
  asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's page-table copies
  Bar::sync();
  if (tid == 0) SA_TRACE_POINT(1, 7);  // list counts
  int pos = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int v = warp_tot[w];
    pos += w < warp ? v : 0;
    tot += v;
  }
  for (int p0 = w0; p0 < w1; p0 += 32) {
    const int p = p0 + lane;
    const bool tk = p < w1 && taken(p);
    const unsigned m = __ballot_sync(0xffffffffu, tk);
    if (tk) {
      const int at = pos + __popc(m & ((1u << lane) - 1u));
      out[at] = p;
      if (phys_out) phys_out[at] = ptab_s ? ptab_s[p] : ptab_g[p];
    }
    pos += __popc(m);
  }
  for (int i = tot + tid; i < K; i += NT) {
    out[i] = -1;
    if (phys_out) phys_out[i] = -1;
  }
  if (tid == 0) *cnt_out = tot;
  if (tid == 0) SA_TRACE_POINT(1, 3);  // list written
}

}  // namespace sa
