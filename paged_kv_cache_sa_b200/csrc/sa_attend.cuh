// sa_attend.cuh -- device code of the gathered split-KV attention and its merge: the
// attention grid's CTA program and one merge task, as functions that the separate
// kernels (sa_attend.cu) and the single-launch decode (sa_fused.cu) run.
#pragma once

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kMaxUnitsPerCta = 256;  // CTA table capacity
constexpr int kMaxPairs = 4096;       // pairs (sequence x KV head) per call
constexpr int kSmemLimit = 227 * 1024;
constexpr int kAttnWarps = 8;  // consumer warps per CTA

// NC consumer warps, SPW stages (units in flight) per consumer warp
template <int D, int P, int NC, int SPW>
struct AttnShape {
  static constexpr int THREADS = (NC + 1) * 32;  // consumers, producer
  static constexpr int CT = 16;                         // tokens per unit
  static constexpr int UPP = P / CT;                    // units per page
  static constexpr int HALVES = D / 64;                 // 128-B halves per row
  static constexpr int HALF_BYTES = CT * 128;           // one TMA box
  static constexpr int KV_BYTES = HALVES * HALF_BYTES;  // K of one unit
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;      // K + V
  static constexpr int NST = SPW * NC;
  static constexpr int MT = D / 16;  // PV m-tiles (channels)
  static constexpr int JQ = D / 32;  // 16-byte Q/K chunks per lane
  static constexpr int HS = D + 4;   // floats per query head in a state: O[D], m, l, pad
  // dynamic shared memory: stages | pair prefix | unit tables
  static size_t smem_bytes(int n_pairs) {
    return 1024 + (size_t)NST * STAGE_BYTES + (size_t)(n_pairs + 1) * 4 +
           (size_t)3 * kMaxUnitsPerCta * 4 + 16;
  }
};

struct AttnArgs {
  const uint16_t* q;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* sel;
  const int32_t* sel_count;
  const int32_t* sel_phys;  // physical page of each selected entry (nullable)
  float* part;              // [#warps][2][G][D+4] states of cut pairs
  int32_t* pre_out;         // [n_pairs + 1] pair prefix of units (written by CTA 0)
  float* out;
  float* lse;
  int32_t* status;
  int sel_stride, Hq, Hkv, B, max_pages, n_pool;
  int counts_from_lens;  // sel_count[p] == min(ceil(seq_len / P), sel_stride) for every pair
  float scale_log2;
};

// logical 16-byte chunk (within a Dk row) that lane-group t loads for its j-th Q/K chunk
__device__ __forceinline__ int qk_chunk(int j, int t) { return (j >> 1) * 8 + 2 * t + (j & 1); }

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// the pair owning flattened unit u: largest p with pre[p] <= u
__device__ __forceinline__ int find_pair(const int* pre, int n_pairs, int u) {
  int lo = 0, hi = n_pairs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Units per warp for `total` units over `n_warps` warps (at least 1).
__device__ __forceinline__ int units_per_warp(int total, int n_warps) {
  return max(1, (total + n_warps - 1) / n_warps);
}

// The attention grid's CTA program ((NC + 1) * 32 threads), on `smem_raw` (dynamic shared
// memory of AttnShape::smem_bytes); kmap / vmap point at the kernel's tensor-map
// parameters.
template <int D, int P, int NC, int SPW>
__device__ __forceinline__ void attend_gqa_body(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                                const AttnArgs& a, uint8_t* smem_raw) {
  using S = AttnShape<D, P, NC, SPW>;
  constexpr int kThreads = S::THREADS;
  constexpr int HS = S::HS;
  const int G = a.Hq / a.Hkv;
  const int n_pairs = a.B * a.Hkv;
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* pre = reinterpret_cast<int*>(stages + S::NST * S::STAGE_BYTES);  // [n_pairs + 1]
  int* u_row = pre + n_pairs + 1;        // first K/V row of the unit in the pool
  int* u_nv = u_row + kMaxUnitsPerCta;   // valid tokens of the unit (0: skip)
  int* u_pair = u_nv + kMaxUnitsPerCta;  // pair of the unit
  __shared__ __align__(8) uint64_t full_bar[S::NST];
  __shared__ __align__(8) uint64_t empty_bar[S::NST];
  __shared__ int sh_nu, sh_U0, sh_W, abort_flag;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, n_cta = gridDim.x;
  if (tid == 0) SA_TRACE_POINT(2, 0);  // entry

  if (tid == 0) {
    for (int s = 0; s < S::NST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NC) {
    // ===================== producer warp: tables =====================
    // 1. pair prefix sums of units.  A selection made by this library holds exactly
    //    min(ceil(seq_len / P), K) pages per pair, known from the sequence lengths alone,
    //    so that case needs nothing from the previous kernel yet.
    int carry = 0;
    if (!a.counts_from_lens) asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int p0 = 0; p0 < n_pairs; p0 += 32) {
      const int p = p0 + lane;
      int u = 0;
      if (p < n_pairs) {
        int cnt;
        if (a.counts_from_lens) {
          const int Lb = min(max(a.seq_lens[p / a.Hkv], 0), a.max_pages * P);
          cnt = min((Lb + P - 1) / P, a.sel_stride);
        } else {
          cnt = min(max(__ldcg(a.sel_count + p), 0), a.sel_stride);
        }
        u = cnt * S::UPP;
      }
      int incl = u;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (p < n_pairs) pre[p] = carry + incl - u;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) pre[n_pairs] = carry;
    const int total = carry;
    const int W = units_per_warp(total, n_cta * NC);
    const int U0 = min(total, c * NC * W);
    const int nu = min(total, U0 + NC * W) - U0;
    __syncwarp();
    // 2. per unit of the CTA's range: its pair and place in the pair's selection
    constexpr int R = kMaxUnitsPerCta / 32;
    int up[R], ui[R], upart[R], lp[R], ph[R], L[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int j = lane + 32 * k;
      up[k] = ui[k] = upart[k] = ph[k] = L[k] = 0;
      lp[k] = -1;
      if (j < nu) {
        const int u = U0 + j;
        const int p = find_pair(pre, n_pairs, u);
        const int lu = u - pre[p];
        up[k] = p;
        ui[k] = lu / S::UPP;
        upart[k] = lu % S::UPP;
        u_pair[j] = p;
      }
    }
    // 3. the selection itself comes from the previous kernel of the stream
    if (lane == 0) SA_TRACE_POINT(2, 1);  // lengths-only tables built
    if (a.counts_from_lens) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (lane == 0) SA_TRACE_POINT(2, 2);  // selection visible
    asm volatile("griddepcontrol.launch_dependents;");
    if (c == 0)
      for (int p = lane; p <= n_pairs; p += 32) a.pre_out[p] = pre[p];
    // 4. first K/V row and valid tokens of every unit (all loads in flight together)
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int j = lane + 32 * k;
      if (j < nu) {
        // selection entries through L2: in the single-launch decode other CTAs wrote them
        lp[k] = __ldcg(a.sel + (size_t)up[k] * a.sel_stride + ui[k]);
        L[k] = a.seq_lens[up[k] / a.Hkv];
        if (a.sel_phys) ph[k] = __ldcg(a.sel_phys + (size_t)up[k] * a.sel_stride + ui[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int j = lane + 32 * k;
      if (j < nu) {
        const int b = up[k] / a.Hkv, h = up[k] % a.Hkv;
        const int Lb = min(max(L[k], 0), a.max_pages * P);
        const int nb = (Lb + P - 1) / P;
        int phys = -1;
        if (lp[k] >= 0 && lp[k] < nb)
          phys = a.sel_phys ? ph[k] : a.page_table[(size_t)b * a.max_pages + lp[k]];
        int nv = 0;
        if (phys < 0 || phys >= a.n_pool) {
          report(a.status, SA_ERR_DEVICE_CHECK);
          phys = -1;
        } else {
          nv = max(0, min(S::CT, Lb - lp[k] * P - upart[k] * S::CT));
        }
        u_row[j] = phys >= 0 ? (phys * a.Hkv + h) * P + upart[k] * S::CT : 0;
        u_nv[j] = nv;
      }
    }
    if (lane == 0) SA_TRACE_POINT(2, 13);  // unit loads landed
    if (lane == 0) {
      sh_nu = nu;
      sh_U0 = U0;
      sh_W = W;
    }
    __syncwarp();
    named_bar(1, kThreads);  // tables ready
    if (lane == 0) SA_TRACE_POINT(2, 3);  // unit tables ready

    // ===================== producer warp: TMA issue =====================
    if (lane == 0) {
      prefetch_tmap(kmap);
      prefetch_tmap(vmap);
    }
    // lane w < NC feeds consumer warp w: units [w*W, min(nu, (w+1)*W)) in order
    int j = lane * W;
    const int j_end = lane < NC ? min(nu, j + W) : 0;
    int k = 0;  // units issued to consumer warp `lane`
    uint64_t t_idle = 0;
    const uint64_t ef = l2_evict_first();
    for (;;) {
      const bool busy = j < j_end;
      bool issued = false;
      if (busy) {
        const int st = lane + NC * (k % SPW);
        if (k < SPW || mbar_test(&empty_bar[st], ((k / SPW) - 1) & 1)) {
          if (u_nv[j] > 0) {
            uint8_t* kdst = stages + st * S::STAGE_BYTES;
            uint8_t* vdst = kdst + S::KV_BYTES;
            const int row = u_row[j];
            mbar_arrive_expect_tx(&full_bar[st], S::STAGE_BYTES);
#pragma unroll
            for (int hf = 0; hf < S::HALVES; ++hf) {
              tma_load_2d_hint(kdst + hf * S::HALF_BYTES, kmap, hf * 64, row, &full_bar[st],
                               ef);
              tma_load_2d_hint(vdst + hf * S::HALF_BYTES, vmap, hf * 64, row, &full_bar[st],
                               ef);
            }
          } else {
            mbar_arrive(&full_bar[st]);
          }
          ++k;
          ++j;
          issued = true;
        }
      }
      if (!__any_sync(0xffffffffu, busy)) break;
      if (__any_sync(0xffffffffu, issued)) {
        t_idle = 0;
      } else {
        const uint64_t now = global_ns();
        if (t_idle == 0) t_idle = now;
        const int to = (now - t_idle > kWaitLimitNs) || *(volatile int*)&abort_flag;
        if (__any_sync(0xffffffffu, to)) {
          if (lane == 0) {
            report(a.status, SA_ERR_TIMEOUT);
            atomicExch(&abort_flag, 1);
          }
          break;
        }
      }
    }
  } else {
    // ===================== consumer warps =====================
    // The producer alone waits for the previous grid (the wait makes its memory visible
    // to this whole grid); consumers block on the hardware barrier until the tables,
    // built after that wait, are ready.  (Every thread takes part in the early launch of
    // the merge grid.)
    asm volatile("griddepcontrol.launch_dependents;");
    named_bar(1, kThreads);  // tables ready
    const int r = lane >> 2, t = lane & 3;
    const uint32_t stage0 = smem_u32(stages);
    const int W = sh_W, U0 = sh_U0, nu = sh_nu;
    const int j0 = min(nu, warp * W), j1 = min(nu, j0 + W);
    const int gw = c * NC + warp;          // global warp: owner of states part[gw][0..1]
    const int wa = U0 + j0, wb = U0 + j1;  // the warp's range in the flattened list
    // ldmatrix.x4.trans row of this lane: tokens 0-7 (lanes 0-15) or 8-15 (16-31),
    // channel chunk 2*i2 (lanes 0-7, 16-23) or 2*i2 + 1 (8-15, 24-31)
    const int vtok = (lane & 7) + ((lane >> 4) << 3);
    const int vsub = (lane >> 3) & 1;
    uint4 qa[S::JQ];
    float m_run = -INFINITY, l_run = 0.f;
    float o[S::MT][4];
    int cur = -1;  // pair of the running state

    // Write the running state of pair `p`: normalised output when the pair lies wholly
    // inside the warp's range, else the raw (m, l, O) state for the merge kernel.
    auto finish = [&](int p) {
      float lt = l_run;
      lt += __shfl_xor_sync(0xffffffffu, lt, 1);
      lt += __shfl_xor_sync(0xffffffffu, lt, 2);
      const int ua = pre[p], ub = pre[p + 1];
      const int b = p / a.Hkv, h = p % a.Hkv;
      if (ua >= wa && ub <= wb) {
        // heads 2t and 2t+1 of this lane's O^T fragments: their l lives in the lanes
        // with r == head
        const float l0 = __shfl_sync(0xffffffffu, lt, (2 * t) * 4);
        const float l1 = __shfl_sync(0xffffffffu, lt, (2 * t + 1) * 4);
        const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
        const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
        float* ob = a.out + ((size_t)b * a.Hq + h * G) * D;
#pragma unroll
        for (int i2 = 0; i2 < S::MT; ++i2) {
          const int c0 = 16 * i2 + r, c1 = 16 * i2 + 8 + r;
          if (2 * t < G) {
            ob[(2 * t) * D + c0] = o[i2][0] * i0;
            ob[(2 * t) * D + c1] = o[i2][2] * i0;
          }
          if (2 * t + 1 < G) {
            ob[(2 * t + 1) * D + c0] = o[i2][1] * i1;
            ob[(2 * t + 1) * D + c1] = o[i2][3] * i1;
          }
        }
        if (t == 0 && r < G)
          a.lse[(size_t)b * a.Hq + h * G + r] =
              lt > 0.f ? (m_run + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
      } else {
        const int slot = ua < wa ? 0 : 1;
        float* my = a.part + ((size_t)gw * 2 + slot) * G * HS;
#pragma unroll
        for (int i2 = 0; i2 < S::MT; ++i2) {
          const int c0 = 16 * i2 + r, c1 = 16 * i2 + 8 + r;
          if (2 * t < G) {
            my[(2 * t) * HS + c0] = o[i2][0];
            my[(2 * t) * HS + c1] = o[i2][2];
          }
          if (2 * t + 1 < G) {
            my[(2 * t + 1) * HS + c0] = o[i2][1];
            my[(2 * t + 1) * HS + c1] = o[i2][3];
          }
        }
        if (t == 0 && r < G) {
          my[r * HS + D] = m_run;
          my[r * HS + D + 1] = lt;
        }
      }
    };

    for (int j = j0, kc = 0; j < j1; ++j, ++kc) {
      const int p = u_pair[j];
      if (p != cur) {
        if (cur >= 0) finish(cur);
        cur = p;
        const int b = p / a.Hkv, h = p % a.Hkv;
        if (r < G) {
          const uint4* qrow =
              reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + h * G + r) * D);
#pragma unroll
          for (int jj = 0; jj < S::JQ; ++jj) qa[jj] = qrow[qk_chunk(jj, t)];
        } else {
#pragma unroll
          for (int jj = 0; jj < S::JQ; ++jj) qa[jj] = make_uint4(0, 0, 0, 0);
        }
        m_run = -INFINITY;
        l_run = 0.f;
#pragma unroll
        for (int i = 0; i < S::MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      }
      const int st = warp + NC * (kc % SPW);
      bool ok = !*(volatile int*)&abort_flag;
      if (ok && !mbar_wait(&full_bar[st], (kc / SPW) & 1)) {
        report(a.status, SA_ERR_TIMEOUT);
        atomicExch(&abort_flag, 1);
        ok = false;
      }
      if (kc == 0 && lane == 0 && warp == 0) SA_TRACE_POINT(2, 4);  // first unit
      const int nv = ok ? u_nv[j] : 0;
      const uint32_t kbase = stage0 + st * S::STAGE_BYTES;
      const uint32_t vbase = kbase + S::KV_BYTES;
      if (nv > 0 && nv < S::CT) {
        // rows past the valid tokens may hold anything: zero them in V (p = 0 there)
        uint8_t* vrow = stages + st * S::STAGE_BYTES + S::KV_BYTES;
        for (int e = lane; e < (S::CT - nv) * S::HALVES * 8; e += 32) {
          const int row = nv + e / (S::HALVES * 8), cc = e % (S::HALVES * 8);
          *reinterpret_cast<uint4*>(vrow + (cc >> 3) * S::HALF_BYTES + row * 128 +
                                    ((cc & 7) << 4)) = make_uint4(0, 0, 0, 0);
        }
        // the next TMA copy into this stage must not overtake these plain stores
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      if (nv > 0) {
        // ---- S = Q K^T for 16 tokens (two n-tiles of 8) ----
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
          const int row = nt * 8 + r;
#pragma unroll
          for (int jj = 0; jj < S::JQ; ++jj) {
            const int lc = qk_chunk(jj, t);
            const uint32_t addr =
                kbase + (lc >> 3) * S::HALF_BYTES + row * 128 + (((lc & 7) ^ (row & 7)) << 4);
            const uint4 kv = lds_v4(addr);
            mma_bf16_16816(sc[nt], qa[jj].x, 0u, qa[jj].y, 0u, kv.x, kv.y);
            mma_bf16_16816(sc[nt], qa[jj].z, 0u, qa[jj].w, 0u, kv.z, kv.w);
          }
        }
        // ---- online softmax: row = query head r; lane t: tokens 2t,2t+1,8+2t,9+2t ----
        float x[4];
        x[0] = 2 * t < nv ? sc[0][0] * a.scale_log2 : -INFINITY;
        x[1] = 2 * t + 1 < nv ? sc[0][1] * a.scale_log2 : -INFINITY;
        x[2] = 2 * t + 8 < nv ? sc[1][0] * a.scale_log2 : -INFINITY;
        x[3] = 2 * t + 9 < nv ? sc[1][1] * a.scale_log2 : -INFINITY;
        float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const float m_new = fmaxf(m_run, mt);  // finite: token 0 of a unit is valid
        const float alpha = fast_exp2(m_run - m_new);
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = fast_exp2(x[e] - m_new);
        l_run = l_run * alpha + (pr[0] + pr[1]) + (pr[2] + pr[3]);
        m_run = m_new;
        const float al0 = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
        const float al1 = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
        const uint32_t pb0 = pack_bf16(pr[0], pr[1]);
        const uint32_t pb1 = pack_bf16(pr[2], pr[3]);
        // ---- O^T += V^T P^T: m-tile i2 = channels 16 i2 .. 16 i2 + 15 ----
#pragma unroll
        for (int i2 = 0; i2 < S::MT; ++i2) {
          o[i2][0] *= al0;
          o[i2][1] *= al1;
          o[i2][2] *= al0;
          o[i2][3] *= al1;
          const int lc = 2 * i2 + vsub;
          const uint32_t addr =
              vbase + (lc >> 3) * S::HALF_BYTES + vtok * 128 + (((lc & 7) ^ (vtok & 7)) << 4);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_trans(addr, a0, a1, a2, a3);
          mma_bf16_16816(o[i2], a0, a1, a2, a3, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }
    if (cur >= 0) finish(cur);
    if (lane == 0) SA_TRACE_POINT(2, 5 + warp);  // warp's range done
  }
  __syncthreads();
  if (abort_flag && warp == NC && lane == 0) {
    // a wait expired: give copies still in flight a bounded time (10 ms) to land
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 10000000ull) {
    }
  }
}

// Merge of the pairs cut by warp-range boundaries.  One warp per (pair, query head);
// lane i holds channels 4i .. 4i+3.  The states of pair p are those of global warps
// pre[p] / W .. (pre[p+1] - 1) / W, merged in that order with a running maximum.
struct MergeArgs {
  const float* part;
  const int32_t* pre;
  float* out;
  float* lse;
  int n_pairs, G, Hkv, Hq, n_warps;
};

// One merge task, wi = (pair, query head), by one warp.
template <int D>
__device__ __forceinline__ void merge_task(const MergeArgs& a, int wi, int lane) {
  constexpr int HS = D + 4;
  constexpr int CH = 16;  // states in flight per lane
  const int p = wi / a.G, gi = wi % a.G;
  const int b = p / a.Hkv, h = p % a.Hkv;
  float* o = a.out + ((size_t)b * a.Hq + h * a.G + gi) * D;
  float* lse = a.lse + (size_t)b * a.Hq + h * a.G + gi;
  const int ua = __ldcg(a.pre + p), ub = __ldcg(a.pre + p + 1);
  const bool on = lane < D / 4;
  if (ua == ub) {  // nothing selected (empty sequence)
    if (on) reinterpret_cast<float4*>(o)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0) *lse = -INFINITY;
    return;
  }
  const int total = __ldcg(a.pre + a.n_pairs);
  const int W = max(1, (total + a.n_warps - 1) / a.n_warps);
  const int gf = ua / W, gl = (ub - 1) / W;
  if (gf == gl) return;  // wholly inside one warp's range: written by the attention
  float m_run = -INFINITY, l_run = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int g0 = gf; g0 <= gl; g0 += CH) {
    float mk[CH], lk[CH];
    float4 vk[CH];
#pragma unroll
    for (int k = 0; k < CH; ++k) {
      const int gw = g0 + k;
      mk[k] = -INFINITY;
      lk[k] = 0.f;
      vk[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gw <= gl) {
        const int slot = ua < gw * W ? 0 : 1;
        const float* st = a.part + (((size_t)gw * 2 + slot) * a.G + gi) * HS;
        mk[k] = __ldcg(st + D);
        lk[k] = __ldcg(st + D + 1);
        if (on) vk[k] = __ldcg(reinterpret_cast<const float4*>(st) + lane);
      }
    }
    float mc = m_run;
#pragma unroll
    for (int k = 0; k < CH; ++k) mc = fmaxf(mc, mk[k]);
    if (mc == -INFINITY) continue;  // nothing valid yet
    const float f = fast_exp2(m_run - mc);  // 0 when m_run = -inf
    l_run *= f;
    acc.x *= f;
    acc.y *= f;
    acc.z *= f;
    acc.w *= f;
#pragma unroll
    for (int k = 0; k < CH; ++k) {
      const float w = mk[k] == -INFINITY ? 0.f : fast_exp2(mk[k] - mc);
      l_run += lk[k] * w;
      acc.x += vk[k].x * w;
      acc.y += vk[k].y * w;
      acc.z += vk[k].z * w;
      acc.w += vk[k].w * w;
    }
    m_run = mc;
  }
  const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
  if (on)
    reinterpret_cast<float4*>(o)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lane == 0) *lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace sa
