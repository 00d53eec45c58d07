// sa_attend.cu -- gathered split-KV attention over the selected pages, merge fused in.
//
// Method: exact softmax attention over the tokens of the selected pages (SubQ/SSA
// article, SSA section: exact attention on the chosen positions), reached through the
// page table without the caller knowing where pages live (Vortex summary, section 1),
// with an online softmax that never materialises the score row (FlashAttention
// paragraph of the same article); the pages are split across CTAs and the partial
// results merged by log-sum-exp.
//
// Work layout.  The selected pages of all (sequence, KV head) pairs, cut into units of
// 16 tokens, form one flattened list (pair-major, ascending page order).  CTA c (one
// per SM) takes the contiguous slice [c*W, (c+1)*W) of it, W = ceil(total / #CTAs), so
// every SM streams the same number of bytes whatever the sequence lengths.
//  * Producer warp: builds the slice's tables in shared memory (pair prefix sums, then
//    per unit: pair, physical page, valid tokens -- all lanes' loads in flight together)
//    and splits the slice into per-pair segments.  Then lane w feeds consumer warp w's
//    private ring of stages with units w, w+8, w+16, ...: 2-D TMA tile loads of the
//    unit's K and V (128-byte swizzle, mbarrier transaction counts, no multicast).
//  * 8 consumer warps, per unit: S = Q K^T on m16n8k16 tensor-core tiles (the G <= 8
//    query heads are the M side; K fragments come from the swizzled stage with
//    conflict-free 16-byte shared loads in a permuted channel order that Q's fragments
//    share), online softmax in registers (base 2, scale folded in), then O^T += V^T P^T
//    with the channels as the M side (V^T fragments by ldmatrix.trans, the S
//    accumulators are directly the P^T operand).
//  * At the end of every segment the 8 warps' (m, l, O) meet in shared memory; one warp
//    merges them.  A pair covered by one CTA is written out directly; otherwise the
//    CTA's partial goes to the workspace and the last CTA of the pair (atomic counter,
//    no waiting) merges the 2-4 partials in CTA order (deterministic).
// HBM-bound: bytes per selected token and KV head = (Dk + Dv) * 2.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kMaxUnitsPerCta = 256;  // slice table capacity
constexpr int kMaxPairs = 4096;       // pairs (sequence x KV head) per call
constexpr int kSmemLimit = 227 * 1024;
constexpr int kGmax = 8;  // query heads per KV head

// NC consumer warps, SPW stages (units in flight) per consumer warp
template <int D, int P, int NC, int SPW>
struct AttnShape {
  static constexpr int THREADS = (NC + 2) * 32;  // consumers, producer, merger
  static constexpr int CT = 16;                         // tokens per unit
  static constexpr int UPP = P / CT;                    // units per page
  static constexpr int HALVES = D / 64;                 // 128-B halves per row
  static constexpr int HALF_BYTES = CT * 128;           // one TMA box
  static constexpr int KV_BYTES = HALVES * HALF_BYTES;  // K of one unit
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;      // K + V
  static constexpr int NST = SPW * NC;
  static constexpr int MT = D / 16;  // PV m-tiles (channels)
  static constexpr int JQ = D / 32;  // 16-byte Q/K chunks per lane
  static constexpr int HS = D + 4;  // floats per query head in a state: O[D], m, l, pad
  // dynamic shared memory: stages | combine states [2][NC][G][HS] | pair prefix | unit and
  // segment tables
  static size_t smem_bytes(int G, int n_pairs) {
    return 1024 + (size_t)NST * STAGE_BYTES + (size_t)2 * NC * G * HS * 4 +
           (size_t)(n_pairs + 1) * 4 + (size_t)7 * kMaxUnitsPerCta * 4 + 16;
  }
};

struct AttnArgs {
  const uint16_t* q;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* sel;
  const int32_t* sel_count;
  const int32_t* sel_phys;  // physical page of each selected entry (nullable)
  float* part;              // [#CTAs][2][G][D+2] CTA partials
  uint32_t* merge_cnt;      // [B*Hkv] arrivals of CTA partials (zero between calls)
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

__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
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

// Merge n (<= 32) states (each [G][HS]: O row, m, l) at buf into one.  dst == nullptr:
// write the normalised result to out ([G][D]) and lse ([G]); otherwise store the merged
// state at dst (global or shared; dst may be buf itself, state 0).  One warp.  All
// heads are reduced into registers first and written after a single __syncwarp: a
// __syncwarp between global stores would wait for them to complete.
template <int D>
__device__ __noinline__ void merge_states(float* buf, int n, int STATE, int G, int lane,
                                          float* dst, float* out, float* lse) {
  constexpr int HS = D + 4;
  float acc[kGmax][D / 32], mst[kGmax], lsm[kGmax];
#pragma unroll
  for (int gi = 0; gi < kGmax; ++gi) {
    mst[gi] = -INFINITY;
    lsm[gi] = 0.f;
#pragma unroll
    for (int q4 = 0; q4 < D / 32; ++q4) acc[gi][q4] = 0.f;
    if (gi < G) {
      // lane w < n holds state w's (m, l); its weight is 2^(m_w - m*)
      const float mw = lane < n ? buf[lane * STATE + gi * HS + D] : -INFINITY;
      const float lw = lane < n ? buf[lane * STATE + gi * HS + D + 1] : 0.f;
      float mstar = mw;
#pragma unroll
      for (int off = 16; off; off >>= 1)
        mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, off));
      const float fw = (mw == -INFINITY) ? 0.f : fast_exp2(mw - mstar);
      float lsum = lw * fw;
#pragma unroll
      for (int off = 16; off; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
      mst[gi] = mstar;
      lsm[gi] = lsum;
#pragma unroll 1
      for (int w = 0; w < n; ++w) {
        const float f = __shfl_sync(0xffffffffu, fw, w);
        const float* row = buf + w * STATE + gi * HS;
#pragma unroll
        for (int q4 = 0; q4 < D / 32; ++q4) acc[gi][q4] += row[lane + 32 * q4] * f;
      }
    }
  }
  __syncwarp();  // every read of buf is done before dst (possibly buf) is written
#pragma unroll
  for (int gi = 0; gi < kGmax; ++gi) {
    if (gi >= G) continue;
    if (dst) {
      float* drow = dst + gi * HS;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) drow[lane + 32 * q4] = acc[gi][q4];
      if (lane == 0) {
        drow[D] = mst[gi];
        drow[D + 1] = lsm[gi];
      }
    } else {
      const float lsum = lsm[gi];
      float* o = out + gi * D;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) o[lane + 32 * q4] = lsum > 0.f ? acc[gi][q4] / lsum : 0.f;
      if (lane == 0)
        lse[gi] = lsum > 0.f ? (mst[gi] + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
    }
  }
}

template <int D, int P, int NC, int SPW>
__global__ void __launch_bounds__((NC + 2) * 32, 1)
    attend_gqa_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  using S = AttnShape<D, P, NC, SPW>;
  constexpr int kConsumers = NC;
  constexpr int kAttnThreads = S::THREADS;
  const int G = a.Hq / a.Hkv;
  const int n_pairs = a.B * a.Hkv;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int HS = S::HS;
  const int STATE = G * HS;  // floats of one warp's state
  float* comb = reinterpret_cast<float*>(stages + S::NST * S::STAGE_BYTES);
  int* pre = reinterpret_cast<int*>(comb + 2 * NC * STATE);  // [n_pairs + 1]
  int* u_phys = pre + n_pairs + 1;                        // physical page, -1 = masked
  int* u_row = u_phys + kMaxUnitsPerCta;                  // first K/V row in the pool
  int* u_nv = u_row + kMaxUnitsPerCta;                    // valid tokens of the unit
  int* u_pair = u_nv + kMaxUnitsPerCta;
  int* seg_start = u_pair + kMaxUnitsPerCta;              // [kMaxUnitsPerCta + 1]
  int* seg_pair = seg_start + kMaxUnitsPerCta + 1;
  int* seg_ord = seg_pair + kMaxUnitsPerCta;             // processing order of segments
  __shared__ __align__(8) uint64_t full_bar[S::NST];
  __shared__ __align__(8) uint64_t empty_bar[S::NST];
  __shared__ int sh_n_seg, sh_U0, sh_W, abort_flag;

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

  if (warp == kConsumers) {
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
    const int W = max(1, (total + n_cta - 1) / n_cta);
    const int U0 = min(total, c * W);
    const int nu = min(total, U0 + W) - U0;
    __syncwarp();
    // 2. per unit of the slice: its pair and place in the pair's selection
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
    __syncwarp();
    // 3. segments: maximal runs of one pair
    int n_seg = 0;
    for (int j0 = 0; j0 < nu; j0 += 32) {
      const int j = j0 + lane;
      const bool start = j < nu && (j == 0 || u_pair[j] != u_pair[j - 1]);
      const unsigned m = __ballot_sync(0xffffffffu, start);
      if (start) {
        const int k = n_seg + __popc(m & ((1u << lane) - 1));
        seg_start[k] = j;
        seg_pair[k] = u_pair[j];
      }
      n_seg += __popc(m);
    }
    // 4. the selection itself comes from the previous kernel of the stream
    if (a.counts_from_lens) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    // pairs with nothing selected (seq_len 0): out = 0, lse = -inf
    for (int p = c * 32 + lane; p < n_pairs; p += n_cta * 32) {
      if (pre[p + 1] != pre[p]) continue;
      const int b = p / a.Hkv, h = p % a.Hkv;
      for (int gi = 0; gi < G; ++gi) {
        float* o = a.out + ((size_t)b * a.Hq + h * G + gi) * D;
        for (int ch = 0; ch < D; ++ch) o[ch] = 0.f;
        a.lse[(size_t)b * a.Hq + h * G + gi] = -INFINITY;
      }
    }
    // 5. physical page and valid tokens of every unit (all loads in flight together)
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
        u_phys[j] = phys;
        u_row[j] = phys >= 0 ? (phys * a.Hkv + h) * P + upart[k] * S::CT : 0;
        u_nv[j] = nv;
      }
    }
    if (lane == 0) {
      seg_start[n_seg] = nu;
      sh_n_seg = n_seg;
      sh_U0 = U0;
      sh_W = W;
    }
    // processing order: the slice's first and last segments (the ones shared with the
    // neighbouring CTAs) come first, so the cross-CTA merges finish while the whole
    // pairs in between are still streaming
    for (int i = lane; i < n_seg; i += 32)
      seg_ord[i] = i == 0 ? 0 : (i == 1 ? n_seg - 1 : i - 1);
    __syncwarp();
    named_bar(1, kAttnThreads);  // tables ready

    // ===================== producer warp: TMA issue =====================
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    int k = 0;  // units issued to consumer warp `lane`
    // next unit of consumer warp `lane` in processing order: units j == lane (mod NC)
    // of segment seg_ord[oi]
    int oi = 0, j = -1;
    auto advance = [&]() {
      while (oi < n_seg) {
        const int sg = seg_ord[oi];
        const int sa_ = seg_start[sg], sb_ = seg_start[sg + 1];
        j = j < 0 ? sa_ + ((lane - sa_) % kConsumers + kConsumers) % kConsumers : j + kConsumers;
        if (j < sb_) return;
        ++oi;
        j = -1;
      }
    };
    if (lane < kConsumers) advance();
    uint64_t t_idle = 0;
    for (;;) {
      const bool busy = lane < kConsumers && oi < n_seg;
      bool issued = false;
      if (busy) {
        const int st = lane + kConsumers * (k % SPW);
        if (k < SPW || mbar_test(&empty_bar[st], ((k / SPW) - 1) & 1)) {
          if (u_phys[j] >= 0 && u_nv[j] > 0) {
            uint8_t* kdst = stages + st * S::STAGE_BYTES;
            uint8_t* vdst = kdst + S::KV_BYTES;
            const int row = u_row[j];
            mbar_arrive_expect_tx(&full_bar[st], S::STAGE_BYTES);
#pragma unroll
            for (int hf = 0; hf < S::HALVES; ++hf) {
              tma_load_2d(kdst + hf * S::HALF_BYTES, &kmap, hf * 64, row, &full_bar[st]);
              tma_load_2d(vdst + hf * S::HALF_BYTES, &vmap, hf * 64, row, &full_bar[st]);
            }
          } else {
            mbar_arrive(&full_bar[st]);
          }
          ++k;
          advance();
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
  } else if (warp < kConsumers) {
    // ===================== consumer warps =====================
    asm volatile("griddepcontrol.wait;" ::: "memory");
    named_bar(1, kAttnThreads);  // tables ready
    const int r = lane >> 2, t = lane & 3;
    const uint32_t stage0 = smem_u32(stages);
    const int n_seg = sh_n_seg;
    // ldmatrix.x4.trans row of this lane: tokens 0-7 (lanes 0-15) or 8-15 (16-31),
    // channel chunk 2*i2 (lanes 0-7, 16-23) or 2*i2 + 1 (8-15, 24-31)
    const int vtok = (lane & 7) + ((lane >> 4) << 3);
    const int vsub = (lane >> 3) & 1;
    int kc = 0;  // units consumed by this warp
    uint4 qa[S::JQ];
    for (int sgi = 0; sgi < n_seg; ++sgi) {
      const int sg = seg_ord[sgi];  // segment processed in this round
      const int p = seg_pair[sg];
      const int sa_ = seg_start[sg], sb_ = seg_start[sg + 1];
      const int b = p / a.Hkv, h = p % a.Hkv;
      if (r < G) {
        const uint4* qrow =
            reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + h * G + r) * D);
#pragma unroll
        for (int j = 0; j < S::JQ; ++j) qa[j] = qrow[qk_chunk(j, t)];
      } else {
#pragma unroll
        for (int j = 0; j < S::JQ; ++j) qa[j] = make_uint4(0, 0, 0, 0);
      }
      float m_run = -INFINITY, l_run = 0.f;
      float o[S::MT][4];
#pragma unroll
      for (int i = 0; i < S::MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      // my units of this segment: j = warp + 8i within [sa_, sb_)
      const int first = sa_ + ((warp - sa_) % kConsumers + kConsumers) % kConsumers;
      for (int j = first; j < sb_; j += kConsumers, ++kc) {
        const int st = warp + kConsumers * (kc % SPW);
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
            const uint32_t addr = vbase + (lc >> 3) * S::HALF_BYTES + vtok * 128 +
                                  (((lc & 7) ^ (vtok & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(addr, a0, a1, a2, a3);
            mma_bf16_16816(o[i2], a0, a1, a2, a3, pb0, pb1);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
      }
      // ---- segment end: hand this warp's state to the merger (buffer sgi & 1) ----
      float lt = l_run;
      lt += __shfl_xor_sync(0xffffffffu, lt, 1);
      lt += __shfl_xor_sync(0xffffffffu, lt, 2);
      // buffer sgi & 1 was last used for segment sgi - 2: wait until it is merged
      if (sgi >= 2) named_bar(4 + (sgi & 1), (kConsumers + 1) * 32);
      float* my = comb + ((size_t)(sgi & 1) * kConsumers + warp) * STATE;
      // per warp: [G][HS] = O row, m, l
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
      __threadfence_block();
      named_arrive(2 + (sgi & 1), (kConsumers + 1) * 32);
    }
  } else {
    // ===================== merger warp =====================
    named_bar(1, kAttnThreads);  // tables ready
    const int n_seg = sh_n_seg, U0 = sh_U0, W = sh_W;
    for (int sgi = 0; sgi < n_seg; ++sgi) {
      const int sg = seg_ord[sgi];
      const int p = seg_pair[sg];
      const int sa_ = seg_start[sg], sb_ = seg_start[sg + 1];
      const int b = p / a.Hkv, h = p % a.Hkv;
      named_bar(2 + (sgi & 1), (kConsumers + 1) * 32);  // the NC states are written
      float* comb_s = comb + (size_t)(sgi & 1) * kConsumers * STATE;
      do {
      // ---- merge the NC states of this segment (compact code: it runs once per
      //      segment, so it is kept small rather than unrolled) ----
      const int ua = U0 + sa_, ub = U0 + sb_;
      const bool whole = ua == pre[p] && ub == pre[p + 1];
      const int slot = sg == 0 ? 0 : 1;  // only a slice's first / last segment is partial
      float* dst = whole ? nullptr : a.part + ((size_t)c * 2 + slot) * STATE;
      merge_states<D>(comb_s, kConsumers, STATE, G, lane, dst,
                      a.out + ((size_t)b * a.Hq + h * G) * D, a.lse + (size_t)b * a.Hq + h * G);
      if (whole) break;
      // ---- a pair shared with other CTAs: the last CTA to arrive merges ----
      __threadfence();
      __syncwarp();
      const int c_first = pre[p] / W, c_last = (pre[p + 1] - 1) / W;
      uint32_t old = 0;
      if (lane == 0) old = atomicAdd(a.merge_cnt + p, 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old != (uint32_t)(c_last - c_first)) break;
      __threadfence();
      // Fold the pair's CTA partials, up to NC at a time, into the combine area (now idle)
      // and merge them there in CTA order (deterministic).  The running result of the
      // previous chunks is carried as one more state.
      {
        const int np = c_last - c_first + 1;
        const int vec = STATE / 4;  // 16-byte vectors per state
        int carried = 0;            // states already in the buffer (the running result)
        for (int i0 = 0; i0 < np;) {
          const int n = min(kConsumers - carried, np - i0);
          __syncwarp();
          // eight loads in flight per lane before any of them is stored
#pragma unroll 1
          for (int e0 = lane; e0 < n * vec; e0 += 8 * 32) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int e = e0 + 32 * u;
              if (e < n * vec) {
                const int cc = c_first + i0 + e / vec;
                const int sl = cc * W < pre[p] ? 1 : 0;
                v[u] = __ldcg(reinterpret_cast<const float4*>(
                                  a.part + ((size_t)cc * 2 + sl) * STATE) + e % vec);
              }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int e = e0 + 32 * u;
              if (e < n * vec)
                reinterpret_cast<float4*>(comb_s + (size_t)(carried + e / vec) * STATE)[e % vec] =
                    v[u];
            }
          }
          __syncwarp();
          i0 += n;
          const bool last = i0 >= np;
          // merge states [0, carried + n) into state 0 (or into the outputs when last)
          merge_states<D>(comb_s, carried + n, STATE, G, lane, last ? nullptr : comb_s,
                          a.out + ((size_t)b * a.Hq + h * G) * D,
                          a.lse + (size_t)b * a.Hq + h * G);
          carried = 1;
        }
      }
      if (lane == 0) a.merge_cnt[p] = 0;  // ready for the next call
      } while (0);
      // buffer sgi & 1 is free again for segment sgi + 2
      if (sgi + 2 < n_seg) named_arrive(4 + (sgi & 1), (kConsumers + 1) * 32);
    }
  }
  __syncthreads();
  if (abort_flag && warp == NC && lane == 0) {
    // a wait expired: give copies still in flight a bounded time (10 ms) to land
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 10000000ull) {
    }
  }
}

template <int D, int P, int NC, int SPW>
static cudaError_t launch_attend_t(const sa_geom& g, const void* k_cache, const void* v_cache,
                                   AttnArgs a, int n_cta, cudaStream_t stream) {
  using S = AttnShape<D, P, NC, SPW>;
  CUtensorMap kmap, vmap;
  const uint64_t rows = (uint64_t)g.n_pool * g.Hkv * P;
  if (!encode_rows_tmap(&kmap, k_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  if (!encode_rows_tmap(&vmap, v_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  const size_t smem = S::smem_bytes(g.Hq / g.Hkv, g.B * g.Hkv);
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(attend_gqa_kernel<D, P, NC, SPW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_cta);
  cfg.blockDim = dim3(S::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attend_gqa_kernel<D, P, NC, SPW>, kmap, vmap, a);
}

// Pipeline shape: NC consumer warps with SPW units in flight each.  The deepest ring
// that fits next to the combine area and tables is used.
template <int D, int P>
static cudaError_t launch_attend_d(const sa_geom& g, const void* k_cache, const void* v_cache,
                                   AttnArgs a, int n_cta, cudaStream_t stream) {
  const int G = g.Hq / g.Hkv, n_pairs = g.B * g.Hkv;
  if (AttnShape<D, P, 8, 3>::smem_bytes(G, n_pairs) <= (size_t)kSmemLimit)
    return launch_attend_t<D, P, 8, 3>(g, k_cache, v_cache, a, n_cta, stream);
  return launch_attend_t<D, P, 8, 2>(g, k_cache, v_cache, a, n_cta, stream);
}

int attend_ctas(const sa_geom& g, int K, int sms) {
  // enough CTAs that no slice exceeds the table capacity even when every pair selects
  // all K pages
  const long long units = (long long)g.B * g.Hkv * K * (g.P / 16);
  const long long need = (units + kMaxUnitsPerCta - 1) / kMaxUnitsPerCta;
  return (int)(need > sms ? need : sms);
}

size_t attend_partial_floats(const sa_geom& g, int n_cta) {
  return (size_t)n_cta * 2 * (g.Hq / g.Hkv) * (g.Dv + 4);
}

bool attend_supported(const sa_geom& g) {
  return g.B * g.Hkv <= kMaxPairs &&
         AttnShape<128, 16, 8, 2>::smem_bytes(g.Hq / g.Hkv, g.B * g.Hkv) <= (size_t)kSmemLimit;
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
  a.merge_cnt = c.merge_cnt;
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
