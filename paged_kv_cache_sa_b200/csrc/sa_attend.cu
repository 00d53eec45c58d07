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
#include "sa_attend.cuh"

namespace sa {

template <int D, int P, int NC, int SPW>
__global__ void __launch_bounds__((NC + 1) * 32, 1)
    attend_gqa_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  attend_gqa_body<D, P, NC, SPW>(&kmap, &vmap, a, smem_raw);
}

template <int D>
__global__ void __launch_bounds__(128) attend_merge_kernel(const MergeArgs a) {
  // one thread waits for the attention grid; the rest block on the CTA barrier
  if (threadIdx.x == 0) SA_TRACE_POINT(3, 0);  // entry
  if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) SA_TRACE_POINT(3, 1);  // attention visible
  asm volatile("griddepcontrol.launch_dependents;");
  const int wi = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (wi < a.n_pairs * a.G) merge_task<D>(a, wi, threadIdx.x & 31);
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

#ifdef SA_TRACE
void trace_set_attend(void* buf) { cudaMemcpyToSymbol(sa_trace_buf, &buf, sizeof(buf)); }
#endif

}  // namespace sa
