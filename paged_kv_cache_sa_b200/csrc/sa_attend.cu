// sa_attend.cu -- gathered split-KV attention over the selected pages, then the merge.
//
// Method: exact softmax attention over the tokens of the selected pages (SubQ/SSA
// article, SSA section: exact attention on the chosen positions), reached through the
// page table without the caller knowing where pages live (Vortex summary, section 1),
// with an online softmax that never materialises the score row (FlashAttention
// paragraph of the same article); the pages are split across warps and the partial
// results merged by log-sum-exp (flash-decoding style split-KV).
//
// Work layout.  The selected pages of all (sequence, KV head) pairs, cut into units of
// 16 tokens, form one flattened list (pair-major, ascending page order).  Warp w of CTA c
// (global warp gw = c * NC + w) takes the contiguous range [gw*W, (gw+1)*W) of it,
// W = ceil(total / #warps), so every SM streams the same number of bytes whatever the
// sequence lengths.
//  * Producer warp: builds the CTA's tables in shared memory (pair prefix sums, then per
//    unit: pair, first K/V row, valid tokens -- all lanes' loads in flight together).
//    Then lane w feeds consumer warp w's private ring of stages with its units in order:
//    2-D TMA tile loads of the unit's K and V (128-byte swizzle, mbarrier transaction
//    counts, no multicast).
//  * NC consumer warps, per unit: S = Q K^T on m16n8k16 tensor-core tiles (the G <= 8
//    query heads are the M side; K fragments come from the swizzled stage with
//    conflict-free 16-byte shared loads in a permuted channel order that Q's fragments
//    share), online softmax in registers (base 2, scale folded in), then O^T += V^T P^T
//    with the channels as the M side (V^T fragments by ldmatrix.trans, the S
//    accumulators are directly the P^T operand).  When the pair changes, or the range
//    ends, a pair lying wholly inside the warp's range is normalised and written out;
//    a pair cut by the range boundary leaves its (m, l, O) state in the workspace
//    (slot 0: the pair began before the range, slot 1: it goes on after it).
//  * attend_merge_kernel (launched programmatically dependent, so its CTAs are resident
//    before the attention grid ends) merges the states of every cut pair in range order
//    (deterministic), and writes the empty pairs (out = 0, lse = -inf).
// No global memory traffic but the K/V stream happens while a warp streams: a load or
// fence issued behind the SM's deep queue of TMA reads waits for that whole queue.
// HBM-bound: bytes per selected token and KV head = (Dk + Dv) * 2.
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

template <int D, int P, int NC, int SPW>
__global__ void __launch_bounds__((NC + 1) * 32, 1)
    attend_gqa_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  using S = AttnShape<D, P, NC, SPW>;
  constexpr int kThreads = S::THREADS;
  constexpr int HS = S::HS;
  const int G = a.Hq / a.Hkv;
  const int n_pairs = a.B * a.Hkv;
  extern __shared__ uint8_t smem_raw[];
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
          cnt = min(max(a.sel_count[p], 0), a.sel_stride);
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
    if (a.counts_from_lens) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    if (c == 0)
      for (int p = lane; p <= n_pairs; p += 32) a.pre_out[p] = pre[p];
    // 4. first K/V row and valid tokens of every unit (all loads in flight together)
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int j = lane + 32 * k;
      if (j < nu) {
        lp[k] = a.sel[(size_t)up[k] * a.sel_stride + ui[k]];
        L[k] = a.seq_lens[up[k] / a.Hkv];
        if (a.sel_phys) ph[k] = a.sel_phys[(size_t)up[k] * a.sel_stride + ui[k]];
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
    if (lane == 0) {
      sh_nu = nu;
      sh_U0 = U0;
      sh_W = W;
    }
    __syncwarp();
    named_bar(1, kThreads);  // tables ready

    // ===================== producer warp: TMA issue =====================
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
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
              tma_load_2d_hint(kdst + hf * S::HALF_BYTES, &kmap, hf * 64, row, &full_bar[st],
                               ef);
              tma_load_2d_hint(vdst + hf * S::HALF_BYTES, &vmap, hf * 64, row, &full_bar[st],
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

template <int D>
__global__ void __launch_bounds__(128) attend_merge_kernel(const MergeArgs a) {
  constexpr int HS = D + 4;
  constexpr int CH = 16;  // states in flight per lane
  // one thread waits for the attention grid; the rest block on the CTA barrier
  if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;");
  const int lane = threadIdx.x & 31;
  const int wi = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (wi >= a.n_pairs * a.G) return;
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

static cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

template <int D, int P, int NC, int SPW>
static cudaError_t launch_attend_t(const sa_geom& g, const void* k_cache, const void* v_cache,
                                   AttnArgs a, int n_cta, cudaStream_t stream) {
  using S = AttnShape<D, P, NC, SPW>;
  CUtensorMap kmap, vmap;
  const uint64_t rows = (uint64_t)g.n_pool * g.Hkv * P;
  if (!encode_rows_tmap(&kmap, k_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  if (!encode_rows_tmap(&vmap, v_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  const size_t smem = S::smem_bytes(g.B * g.Hkv);
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(attend_gqa_kernel<D, P, NC, SPW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // largest carveout for every decode kernel: neighbours can share an SM
    e = cudaFuncSetAttribute(attend_gqa_kernel<D, P, NC, SPW>,
                             cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attend_merge_kernel<D>,
                             cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  void* args[] = {&kmap, &vmap, &a};
  cudaError_t e = launch_pdl(reinterpret_cast<const void*>(attend_gqa_kernel<D, P, NC, SPW>),
                             dim3(n_cta), dim3(S::THREADS), smem, stream, args);
  if (e != cudaSuccess) return e;
  MergeArgs m;
  m.part = a.part;
  m.pre = a.pre_out;
  m.out = a.out;
  m.lse = a.lse;
  m.n_pairs = g.B * g.Hkv;
  m.G = g.Hq / g.Hkv;
  m.Hkv = g.Hkv;
  m.Hq = g.Hq;
  m.n_warps = n_cta * NC;
  void* margs[] = {&m};
  const int n_tasks = m.n_pairs * m.G;
  return launch_pdl(reinterpret_cast<const void*>(attend_merge_kernel<D>),
                    dim3((n_tasks + 3) / 4), dim3(128), 0, stream, margs);
}

// Pipeline shape: kAttnWarps consumer warps with SPW units in flight each; the deepest
// ring that fits next to the tables is used.
template <int D, int P>
static cudaError_t launch_attend_d(const sa_geom& g, const void* k_cache, const void* v_cache,
                                   AttnArgs a, int n_cta, cudaStream_t stream) {
  constexpr int kDeep = D <= 64 ? 4 : 3;
  if (AttnShape<D, P, kAttnWarps, kDeep>::smem_bytes(g.B * g.Hkv) <= (size_t)kSmemLimit)
    return launch_attend_t<D, P, kAttnWarps, kDeep>(g, k_cache, v_cache, a, n_cta, stream);
  return launch_attend_t<D, P, kAttnWarps, 2>(g, k_cache, v_cache, a, n_cta, stream);
}

int attend_ctas(const sa_geom& g, int K, int sms) {
  // enough CTAs that no CTA's range exceeds the table capacity even when every pair
  // selects all K pages
  const long long units = (long long)g.B * g.Hkv * K * (g.P / 16);
  const long long need = (units + kMaxUnitsPerCta - 1) / kMaxUnitsPerCta;
  return (int)(need > sms ? need : sms);
}

size_t attend_partial_floats(const sa_geom& g, int n_cta) {
  return (size_t)n_cta * kAttnWarps * 2 * (g.Hq / g.Hkv) * (g.Dv + 4);
}

bool attend_supported(const sa_geom& g) {
  return g.B * g.Hkv <= kMaxPairs &&
         AttnShape<128, 16, kAttnWarps, 2>::smem_bytes(g.B * g.Hkv) <= (size_t)kSmemLimit;
}

cudaError_t launch_attend(const sa_geom& g, const AttendCall& c, cudaStream_t stream) {
  AttnArgs a;
  a.q = static_cast<const uint16_t*>(c.q);
  a.page_table = c.page_table;
  a.seq_lens = c.seq_lens;
  a.sel = c.sel;
  a.sel_count = c.sel_count;
  a.sel_phys = c.sel_phys;
  a.part = c.part;
  a.pre_out = c.pre;
  a.out = c.out;
  a.lse = c.lse;
  a.status = c.status;
  a.sel_stride = c.sel_stride;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.B = g.B;
  a.max_pages = g.max_pages;
  a.n_pool = g.n_pool;
  a.counts_from_lens = c.counts_from_lens;
  a.scale_log2 = c.scale * 1.4426950408889634f;
#define SA_ATTEND_CASE(DD, PP) \
  if (g.Dk == DD && g.P == PP) \
    return launch_attend_d<DD, PP>(g, c.k_cache, c.v_cache, a, c.n_cta, stream);
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
