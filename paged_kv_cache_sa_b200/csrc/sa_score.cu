// sa_score.cu -- page scoring (the query-aware page bound) and top-k page selection.
//
// Method ("SparseEngine" blog, hook-point paragraph: Quest chooses the pages to read at
// each decode step from the current query; Vortex summary, section 1: hand back the
// top pages; SCBench notes, Tri-shape section: sink tokens + local window always kept):
//   S(b,h,p) = max over the query heads g of KV head h of
//   u_g(p)   = sum_c max(q_gc * kmax_c, q_gc * kmin_c),
// then per (sequence, KV head) the sink and window pages plus the best remaining pages
// up to budget/P (equal scores -> lower page index), as an ascending list.
//
// Scoring (score_stream_kernel).  Because kmax >= kmin,
// max(q*kmax, q*kmin) = max(q,0)*kmax + min(q,0)*kmin exactly, so
// u = [kmin | kmax] . [min(q,0) | max(q,0)], a contraction of length 2*Dk.  Every
// bf16 x bf16 product is exact in fp32; accumulation is fp32.  The G <= 8 query heads
// are the N=8 side of an m16n8k16 tensor-core tile and 16 pages its M side.
// The work is a flattened list of tiles (sequence, head group, 16 consecutive pages);
// each persistent CTA takes a contiguous slice, which every warp derives from the
// sequence lengths itself (no CTA barrier before the first copy).  A producer warp
// gathers the slice's page-table entries with asynchronous 4-byte copies, then each
// tile with one bulk copy per page (the page's summaries of the head group are
// contiguous, 4 KB for 8 heads at Dk = 128; L2 evict-first) plus one for the group's
// query rows, into a ring of shared-memory stages; per-tile tables travel with the
// stage barrier (release/acquire).  Consumer warps (one per KV head of the group) read
// A and B fragments with 16-byte shared loads in a permuted channel order (the query side uses
// the same order, so the sum is unchanged) -- page slots are padded by 64 bytes so
// those loads are free of bank conflicts -- and write the GQA-max score row.
// HBM-bound: bytes per (page, KV head) = 2 * Dk * 2 (summary) + 4 / Hkv (page table).
// fp8 records (score_stream_kernel<D, true>): the same tiles over [Dk codes of min |
// Dk codes of max | int8 e | pad] records of 2 * Dk + 16 bytes, codes widened to bf16
// exactly (every E4M3 value is a bf16 value) before the MMA, the record's 2^e applied
// to the GQA-max score (a positive power of two commutes with the max).  Bytes per
// (page, KV head): 2 * Dk + 16.
//
// Decode-time refresh: when asked, the consumer warps first recompute the summaries of
// each sequence's newest pages from K (the pages that received appended tokens; bf16
// rows, or fp8 records encoded exactly as the summaries kernel encodes them) and score
// them, while the first copies are in flight; the stream skips those pages, so it may
// read either version of their summaries.
//
// Selection (select_kernel, one CTA per (sequence, KV head), launched programmatically
// dependent on the scoring grid, which exits before it starts).  It turns the scores
// into order-preserving 32-bit keys in shared memory (forced pages get key 0, below
// every real score) and runs an MSB-first radix select with 11-bit digits, starting at
// the highest bit in which the candidates' keys differ (shared-memory histogram, block
// scan over the bins).  It stops when the boundary bin is taken whole (threshold key),
// or holds at most 256 candidates, which are then ranked exactly by (key desc, page
// asc) and the winners marked; all-equal boundary keys take the lowest pages.  The
// ascending list of forced and taken pages (and their physical ids) is written with
// per-warp ballots and one block barrier.  Deterministic.
#include "sa_attend.cuh"
#include "sa_score.cuh"

namespace sa {

template <int D, bool F8 = false>
__global__ void __launch_bounds__(kScoreThreads, 1) score_stream_kernel(const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  score_stream_body<D, F8>(a, smem_raw);
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(const SelectArgs a) {
  constexpr int NT = kSelectThreads;
  extern __shared__ uint32_t keys[];  // [max_pages] keys, then [max_pages] page table
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t misc[4], red[2 * (NT / 32)];
  __shared__ uint32_t bin_key[kBinCap];
  __shared__ int bin_page[kBinCap];
  __shared__ int warp_tot[NT / 32 + 1];
  const SelScratch sh{hist, bin_key, bin_page, warp_tot, red, misc};
  select_body<NT, SelBar<-1, NT>>(a, blockIdx.y, blockIdx.x, keys, sh);
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

// shared memory of the scoring grid besides its stages: alignment slack and tables
static size_t score_table_bytes(const sa_geom& g) {
  return 128 + (size_t)(2 * g.B + 1) * 4 + (size_t)kMaxTilesPerCta * kTilePages * 4 +
         (size_t)5 * kMaxTilesPerCta * 4;
}

// Tile shape of the scoring grid for geometry g (see ScoreArgs); f8: fp8 records.
// bf16: up to 8 KV heads per page slot (one 4 KB bulk copy per page at Dk = 128), as many
// stages as fit (a page slot is padded by 64 B when that still leaves the same number of
// stages: conflict-free fragment loads).
static void score_shape(const sa_geom& g, ScoreArgs* a, bool f8 = false) {
  const int D = g.Dk;
  const int G = g.Hq / g.Hkv;
  int hg = 1;  // up to 8 KV heads per page slot: one bulk copy of their records per page
  while (hg < kScoreConsumers && g.Hkv % (hg * 2) == 0) hg *= 2;
  a->HG = hg;
  a->n_hg = g.Hkv / hg;
  a->WPS = kScoreConsumers / hg;
  const size_t limit = (size_t)kScoreSmemLimit - score_table_bytes(g);
  if (!f8) {
    a->rec_bytes = 4 * D;
    const int q_bytes = hg * G * D * 2;
    int best = 0;
    for (int pad = kSlotPad; pad >= 0; pad -= kSlotPad) {
      const int slot = hg * 4 * D + pad;
      const int stage = (kTilePages * slot + q_bytes + 127) & ~127;
      int nst = (int)(limit / stage);
      if (nst > 8) nst = 8;
      nst -= nst % a->WPS;  // a multiple of WPS: one warp group per stage slot
      if (nst > best) {
        best = nst;
        a->slot_bytes = slot;
      }
    }
    a->NST = best;
  } else {
    // 8-byte code loads of four page rows per half-warp are conflict-free when slots sit
    // 32 B apart mod 128; as many stages as fit (a multiple of WPS, at most 8)
    a->rec_bytes = 2 * D + 16;
    a->slot_bytes = ((hg * a->rec_bytes + 127) & ~127) + 32;
    const int stage = (kTilePages * a->slot_bytes + hg * G * D * 2 + 127) & ~127;
    int nst = (int)(limit / stage);
    if (nst > 8) nst = 8;
    nst -= nst % a->WPS;
    a->NST = nst;
  }
  a->q_off = kTilePages * a->slot_bytes;
  a->stage_bytes = (a->q_off + hg * G * D * 2 + 127) & ~127;
}

static size_t score_smem(const sa_geom& g, const ScoreArgs& a) {
  return (size_t)a.NST * a.stage_bytes + score_table_bytes(g);
}

int score_ctas(const sa_geom& g, int sms) {
  ScoreArgs a;
  score_shape(g, &a);
  const long long tiles = (long long)g.B * a.n_hg * ((g.max_pages + kTilePages - 1) / kTilePages);
  const long long need = (tiles + kMaxTilesPerCta - 1) / kMaxTilesPerCta;
  long long n = tiles < sms ? tiles : sms;
  if (need > n) n = need;
  return (int)(n > 0 ? n : 1);
}

bool score_supported(const sa_geom& g) {
  if (!(g.Dk == 64 || g.Dk == 128)) return false;
  ScoreArgs a;
  score_shape(g, &a);
  return a.NST >= 2 && score_smem(g, a) <= (size_t)kScoreSmemLimit;
}

bool score_supported_fp8(const sa_geom& g) {
  if (!(g.Dk == 64 || g.Dk == 128)) return false;
  ScoreArgs a;
  score_shape(g, &a, true);
  return a.NST >= 2 && score_smem(g, a) <= (size_t)kScoreSmemLimit;
}

static ScoreArgs make_score_args(const sa_geom& g, const void* q, const void* summ,
                                 const int32_t* page_table, const int32_t* seq_lens,
                                 float* scores, int32_t* status, bool f8) {
  ScoreArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.summ = static_cast<const uint8_t*>(summ);
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.scores = scores;
  a.status = status;
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.G = g.Hq / g.Hkv;
  a.P = g.P;
  a.max_pages = g.max_pages;
  a.n_pool = g.n_pool;
  a.k_cache = nullptr;
  a.summ_w = nullptr;
  a.n_tail = 0;
  score_shape(g, &a, f8);
  return a;
}

cudaError_t launch_score(const sa_geom& g, const void* q, const void* summ,
                         const int32_t* page_table, const int32_t* seq_lens, float* scores,
                         int n_cta, int32_t* status, cudaStream_t stream, bool fp8,
                         const void* k_cache, int n_tail) {
  ScoreArgs a = make_score_args(g, q, summ, page_table, seq_lens, scores, status, fp8);
  if (k_cache && n_tail > 0) {
    a.k_cache = static_cast<const uint4*>(k_cache);
    a.summ_w = static_cast<uint4*>(const_cast<void*>(summ));
    a.n_tail = n_tail < kMaxTail ? n_tail : kMaxTail;
  }
  const size_t smem = score_smem(g, a);
  const void* kern;
  if (g.Dk == 64)
    kern = fp8 ? reinterpret_cast<const void*>(score_stream_kernel<64, true>)
               : reinterpret_cast<const void*>(score_stream_kernel<64>);
  else if (g.Dk == 128)
    kern = fp8 ? reinterpret_cast<const void*>(score_stream_kernel<128, true>)
               : reinterpret_cast<const void*>(score_stream_kernel<128>);
  else
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // every decode kernel prefers the largest shared-memory carveout, so that the next
  // kernel's CTAs can become resident next to this one's (programmatic launch)
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  return launch_pdl(kern, dim3(n_cta), dim3(kScoreThreads), smem, stream, args);
}

cudaError_t launch_select(const sa_geom& g, const int32_t* page_table, const int32_t* seq_lens,
                          float* scores, int K, int sink_pages, int window_pages, int32_t* sel,
                          int32_t* sel_count, int32_t* sel_phys, int32_t* status,
                          cudaStream_t stream) {
  const void* skern = reinterpret_cast<const void*>(select_kernel);
  SelectArgs s;
  s.page_table = page_table;
  s.seq_lens = seq_lens;
  s.scores = scores;
  s.sel = sel;
  s.sel_count = sel_count;
  s.sel_phys = sel_phys;
  s.status = status;
  s.Hkv = g.Hkv;
  s.P = g.P;
  s.max_pages = g.max_pages;
  s.K = K;
  s.s_pages = sink_pages;
  s.w_pages = window_pages;
  const size_t keys_bytes = (size_t)g.max_pages * 4;
  s.ptab_in_smem = 2 * keys_bytes <= (size_t)200 * 1024;
  const size_t ssmem = s.ptab_in_smem ? 2 * keys_bytes : keys_bytes;
  cudaError_t e =
      cudaFuncSetAttribute(skern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(skern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  void* sargs[] = {&s};
  return launch_pdl(skern, dim3(g.Hkv, g.B), dim3(kSelectThreads), ssmem, stream, sargs);
}

cudaError_t launch_score_select(const sa_geom& g, const void* q, void* summ, const void* k_cache,
                                int n_tail, const int32_t* page_table, const int32_t* seq_lens,
                                float* scores, int n_cta, int K, int sink_pages,
                                int window_pages, int32_t* sel, int32_t* sel_count,
                                int32_t* sel_phys, int32_t* status, cudaStream_t stream) {
  // the newest pages' refresh runs inside the scoring grid
  cudaError_t e = launch_score(g, q, summ, page_table, seq_lens, scores, n_cta, status, stream,
                               false, k_cache, n_tail);
  if (e != cudaSuccess) return e;
  return launch_select(g, page_table, seq_lens, scores, K, sink_pages, window_pages, sel,
                       sel_count, sel_phys, status, stream);
}

// ---------------------------------------------------------------------------------------
// Single-launch decode: the whole grouped-query step (scores with the newest pages'
// refresh, the per-(sequence, KV head) selection, the gathered attention, the merge of
// the cut pairs) in one persistent launch of one 288-thread CTA per SM, the CTAs all
// resident (cooperative launch).  The phases run the same CTA programs as the separate
// kernels; between them a grid barrier on a counter in the workspace header (zeroed
// before the launch) hands the results over.  The barrier is bounded: a CTA that waits
// longer than kWaitLimitNs reports SA_ERR_TIMEOUT and goes on.  The selection is spread
// over the CTAs (CTA c takes pairs c, c + grid, ...) by its first 256 threads.
// ---------------------------------------------------------------------------------------
constexpr int kFusedThreads = kScoreThreads;  // 8 compute warps + 1 producer warp
constexpr int kFusedSelectThreads = 256;
static_assert(kFusedThreads == (kAttnWarps + 1) * 32, "phases share one CTA shape");

// shared-memory scratch of the selection phase, carved after the keys (and page table)
struct FusedSelLayout {
  size_t keys, hist, bin_key, bin_page, warp_tot, red, misc, total;
};
__host__ __device__ inline FusedSelLayout fused_sel_layout(int max_pages, bool ptab) {
  FusedSelLayout l;
  size_t off = 0;
  l.keys = off;
  off += (size_t)(ptab ? 2 : 1) * max_pages * 4;
  off = (off + 15) & ~size_t(15);
  l.hist = off;
  off += kHistBins * 4;
  l.bin_key = off;
  off += kBinCap * 4;
  l.bin_page = off;
  off += kBinCap * 4;
  l.warp_tot = off;
  off += (kFusedSelectThreads / 32 + 1) * 4;
  l.red = off;
  off += 2 * (kFusedSelectThreads / 32) * 4;
  l.misc = off;
  off += 4 * 4;
  l.total = off;
  return l;
}

// Grid barrier number `phase` (1, 2, ...) over the launch's CTAs; false after a timeout.
__device__ __forceinline__ bool fused_grid_sync(int32_t* counter, int phase, int32_t* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's results are visible before it arrives
    atomicAdd(counter, 1);
    const int target = phase * (int)gridDim.x;
    const uint64_t t0 = global_ns();
    int ok = 1;
    while (*(volatile int32_t*)counter < target) {
      if (global_ns() - t0 > kWaitLimitNs) {
        report(status, SA_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(200);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

template <int D, int P, int SPW>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const ScoreArgs sa,
                        const SelectArgs se, const AttnArgs at, const MergeArgs mg,
                        int32_t* counter) {
  extern __shared__ uint8_t smem_raw[];
  // 1. page scores (and the newest pages' refresh)
  score_stream_body<D, false>(sa, smem_raw);
  if (threadIdx.x == 0) SA_TRACE_POINT(4, 0);  // phase 1 done
  // the next phase's bulk copies land where this one read and wrote generically
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (!fused_grid_sync(counter, 1, sa.status)) return;
  // 2. selections
  {
    const FusedSelLayout l = fused_sel_layout(se.max_pages, se.ptab_in_smem != 0);
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const SelScratch sh{reinterpret_cast<uint32_t*>(base + l.hist),
                        reinterpret_cast<uint32_t*>(base + l.bin_key),
                        reinterpret_cast<int*>(base + l.bin_page),
                        reinterpret_cast<int*>(base + l.warp_tot),
                        reinterpret_cast<uint32_t*>(base + l.red),
                        reinterpret_cast<uint32_t*>(base + l.misc)};
    using Bar = SelBar<3, kFusedSelectThreads>;
    if (threadIdx.x < kFusedSelectThreads) {
      for (int pr = blockIdx.x; pr < mg.n_pairs; pr += gridDim.x) {
        select_body<kFusedSelectThreads, Bar>(se, pr / se.Hkv, pr % se.Hkv,
                                              reinterpret_cast<uint32_t*>(base + l.keys), sh);
        Bar::sync();  // the scratch is reused by the next pair
      }
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) SA_TRACE_POINT(4, 1);  // phase 2 done
  if (!fused_grid_sync(counter, 2, sa.status)) return;
  if (threadIdx.x == 0) SA_TRACE_POINT(4, 2);  // barrier 2 passed
  // 3. attention over the selected pages
  attend_gqa_body<D, P, kAttnWarps, SPW>(&kmap, &vmap, at, smem_raw);
  if (threadIdx.x == 0) SA_TRACE_POINT(4, 3);  // phase 3 done
  if (!fused_grid_sync(counter, 3, sa.status)) return;
  if (threadIdx.x == 0) SA_TRACE_POINT(4, 4);  // barrier 3 passed
  // 4. merge of the pairs cut by warp ranges: one warp per (pair, query head)
  const int warp = threadIdx.x >> 5, n_warps = gridDim.x * (kFusedThreads / 32);
  for (int wi = blockIdx.x * (kFusedThreads / 32) + warp; wi < mg.n_pairs * mg.G; wi += n_warps)
    merge_task<D>(mg, wi, threadIdx.x & 31);
}

template <int D, int P>
static cudaError_t launch_fused_t(const sa_geom& g, const FusedCall& f, cudaStream_t stream) {
  constexpr int SPW = D <= 64 ? 4 : 3;
  using S = AttnShape<D, P, kAttnWarps, SPW>;
  const int n_cta = f.n_cta;
  const int n_pairs = g.B * g.Hkv;
  ScoreArgs sa = make_score_args(g, f.q, f.summ, f.page_table, f.seq_lens, f.scores, f.status,
                                 false);
  if (f.n_tail > 0) {
    sa.k_cache = static_cast<const uint4*>(f.k_cache);
    sa.summ_w = static_cast<uint4*>(f.summ);
    sa.n_tail = f.n_tail < kMaxTail ? f.n_tail : kMaxTail;
  }
  SelectArgs se;
  se.page_table = f.page_table;
  se.seq_lens = f.seq_lens;
  se.scores = f.scores;
  se.sel = f.sel;
  se.sel_count = f.sel_count;
  se.sel_phys = f.sel_phys;
  se.status = f.status;
  se.Hkv = g.Hkv;
  se.P = g.P;
  se.max_pages = g.max_pages;
  se.K = f.K;
  se.s_pages = f.s_pages;
  se.w_pages = f.w_pages;
  const size_t score_b = score_smem(g, sa);
  const size_t attn_b = S::smem_bytes(n_pairs);
  se.ptab_in_smem = fused_sel_layout(g.max_pages, true).total + 128 <= score_b;
  const size_t sel_b = fused_sel_layout(g.max_pages, se.ptab_in_smem != 0).total + 128;
  size_t smem = score_b > attn_b ? score_b : attn_b;
  if (sel_b > smem) smem = sel_b;
  AttnArgs at;
  at.q = static_cast<const uint16_t*>(f.q);
  at.page_table = f.page_table;
  at.seq_lens = f.seq_lens;
  at.sel = f.sel;
  at.sel_count = f.sel_count;
  at.sel_phys = f.sel_phys;
  at.part = f.part;
  at.pre_out = f.pre;
  at.out = f.out;
  at.lse = f.lse;
  at.status = f.status;
  at.sel_stride = f.K;
  at.Hq = g.Hq;
  at.Hkv = g.Hkv;
  at.B = g.B;
  at.max_pages = g.max_pages;
  at.n_pool = g.n_pool;
  at.counts_from_lens = 1;
  at.scale_log2 = f.scale * 1.4426950408889634f;
  MergeArgs mg;
  mg.part = f.part;
  mg.pre = f.pre;
  mg.out = f.out;
  mg.lse = f.lse;
  mg.n_pairs = n_pairs;
  mg.G = g.Hq / g.Hkv;
  mg.Hkv = g.Hkv;
  mg.Hq = g.Hq;
  mg.n_warps = n_cta * kAttnWarps;
  CUtensorMap kmap, vmap;
  const uint64_t rows = (uint64_t)g.n_pool * g.Hkv * P;
  if (!encode_rows_tmap(&kmap, f.k_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  if (!encode_rows_tmap(&vmap, f.v_cache, D, rows, 64, S::CT)) return cudaErrorInvalidValue;
  const void* kern = reinterpret_cast<const void*>(fused_decode_kernel<D, P, SPW>);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  int dev = 0, optin = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
      cudaSuccess)
    return e;
  if (smem + fa.sharedSizeBytes > (size_t)optin) return cudaErrorInvalidConfiguration;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  // every CTA must be resident at once for the grid barriers
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedThreads, smem)) !=
      cudaSuccess)
    return e;
  if (per_sm < 1 || n_cta > per_sm * f.n_sm) return cudaErrorCooperativeLaunchTooLarge;
  if ((e = cudaMemsetAsync(f.counter, 0, sizeof(int32_t), stream)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_cta);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int32_t* counter = f.counter;
  void* args[] = {&kmap, &vmap, &sa, &se, &at, &mg, &counter};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

bool fused_supported(const sa_geom& g, int K, int n_sm) {
  if (!(g.Dk == 64 || g.Dk == 128) || g.Dv != g.Dk || g.v_aliases_k) return false;
  if (!(g.P == 16 || g.P == 32 || g.P == 64)) return false;
  if (!score_supported(g)) return false;
  // one CTA per SM covers the scoring slices and the attention ranges
  return score_ctas(g, n_sm) <= n_sm && attend_ctas(g, K, n_sm) <= n_sm;
}

cudaError_t launch_fused(const sa_geom& g, const FusedCall& f, cudaStream_t stream) {
#define SA_FUSED_CASE(DD, PP) \
  if (g.Dk == DD && g.P == PP) return launch_fused_t<DD, PP>(g, f, stream);
  SA_FUSED_CASE(64, 16)
  SA_FUSED_CASE(64, 32)
  SA_FUSED_CASE(64, 64)
  SA_FUSED_CASE(128, 16)
  SA_FUSED_CASE(128, 32)
  SA_FUSED_CASE(128, 64)
#undef SA_FUSED_CASE
  return cudaErrorInvalidValue;
}

#ifdef SA_TRACE
void trace_set_score(void* buf) { cudaMemcpyToSymbol(sa_trace_buf, &buf, sizeof(buf)); }
#endif

}  // namespace sa
