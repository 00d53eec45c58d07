// sa_mla.cu -- the latent (MLA) geometry on the 5th-generation tensor cores: 128 query
// heads share one 576-wide latent key per token (V = its first 512 channels).  This
// file holds the page scoring (below) and the attention over the selected pages with
// its chunk merge (second section); selection is the shared select_kernel.
//
// Method (the page bound of the SparseEngine blog's hook-point paragraph, Quest):
//   S(b,p) = max over the 128 heads g of sum_c max(q_gc * kmax_c, q_gc * kmin_c)
//          = max_g ( [kmin | kmax](p) . [min(q_g,0) | max(q_g,0)] ),
// a dense contraction of length 2*576 = 1152 per (page, head), exactly (kmax >= kmin).
//
// Kernel shape.  One CTA per (sequence, tile of 128 logical pages).  D[page][head] =
// A . B^T with A = the tile's summary rows (M = 128, gathered through the page table)
// and B = the sequence's sign-split query rows (N = 128 heads), K = 1152 in 18 chunks of
// 64.  Four producer warps stage each chunk with 16-byte cp.async copies into the
// 128-byte-swizzled K-major layout the tensor core reads (8-row groups 1024 bytes
// apart); one thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32, 128x128x16)
// into a 128-column TMEM accumulator and tcgen05.commit frees each stage; four
// epilogue warps read their 32 TMEM lanes (one page row each) with tcgen05.ld and take
// the max over the 128 head columns.  HBM-bound: 2 * 576 * 2 bytes per page.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

namespace mla {

constexpr int kD = 576;            // latent key width
constexpr int kG = 128;            // query heads
constexpr int kK = 2 * kD;         // contraction length
constexpr int kTile = 128;         // pages per CTA (UMMA M)
constexpr int kChunk = 64;         // K elements per stage (128 bytes per row)
constexpr int kChunks = kK / kChunk;  // 18
constexpr int kStages = 4;
constexpr int kRowBytes = kChunk * 2;               // 128
constexpr int kOpBytes = kTile * kRowBytes;         // 16 KB per operand per stage
constexpr int kStageBytes = 2 * kOpBytes;           // A | B
constexpr int kThreads = 256;                       // 4 producer + 4 MMA/epilogue warps
constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes;
static_assert(kD % kChunk == 0, "a chunk never straddles the kmin/kmax halves");

// ---- tcgen05 / cp.async wrappers ------------------------------------------------------

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand, 128-byte swizzle: rows 128 bytes apart, 8-row groups 1024 bytes
// apart (stride-byte offset), descriptor version 1, layout type 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)1 << 16;                         // leading-byte offset (unused here)
  d |= (uint64_t)(1024 >> 4) << 32;               // stride-byte offset
  d |= (uint64_t)1 << 46;                         // descriptor version
  d |= (uint64_t)2 << 61;                         // 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace mla

// Sign-split query rows of the latent geometry: qs[b][g] = [min(q,0) | max(q,0)] (bf16;
// the half that does not apply is +0).  One thread per 8 channels.
__global__ void __launch_bounds__(256) mla_qsplit_kernel(const uint4* __restrict__ q,
                                                         uint4* __restrict__ qs, int rows) {
  constexpr int CPR = mla::kD / 8;  // 72 chunks per query row
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  // the previous kernel of the stream may still read qs
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  if (i >= rows * CPR) return;
  const int r = i / CPR, c = i % CPR;
  const uint4 v = q[(size_t)r * CPR + c];
  uint32_t w[4] = {v.x, v.y, v.z, v.w}, lo[4], hi[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t neg = ((w[e] >> 15) & 0x00010001u) * 0xFFFFu;  // negative halves
    lo[e] = w[e] & neg;
    hi[e] = w[e] & ~neg;
  }
  qs[(size_t)r * 2 * CPR + c] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  qs[(size_t)r * 2 * CPR + CPR + c] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
}

struct MlaScoreArgs {
  const uint8_t* summ;  // [n_pool][1][2][576] bf16
  const uint8_t* qs;    // [B][128][1152] bf16, sign-split query rows
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;  // [B][1][max_pages]
  int32_t* status;
  int P, max_pages, n_pool;
};

__global__ void __launch_bounds__(mla::kThreads, 1) score_mla_kernel(const MlaScoreArgs a) {
  using namespace mla;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int row_ph[mla::kTile];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x, b = blockIdx.y;
  const int p0 = tile * kTile;

  if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;");
  const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
  const int nb = (L + a.P - 1) / a.P;
  float* srow = a.scores + (size_t)b * a.max_pages;
  if (p0 >= nb) {  // past the sequence: -inf scores, no tensor-core work
    for (int p = p0 + tid; p < min(a.max_pages, p0 + kTile); p += kThreads) srow[p] = -INFINITY;
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 128);  // the 128 producer threads
      mbar_init(&empty_bar[s], 1);   // one tcgen05.commit
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < kTile) {  // physical page of every row of the tile (-1: zero row)
    const int p = p0 + tid;
    int ph = -1;
    if (p < nb) {
      ph = a.page_table[(size_t)b * a.max_pages + p];
      if (ph < 0 || ph >= a.n_pool) {
        report(a.status, SA_ERR_DEVICE_CHECK);
        ph = -1;
      }
    }
    row_ph[tid] = ph;
  }
  if (warp == 4) {  // TMEM: 128 fp32 columns (one per head), 128 lanes (one per page)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base)),
                 "r"(128)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  mla::tc_fence_before();
  __syncthreads();
  mla::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t st0 = smem_u32(stages);

  if (warp < 4) {
    // ===================== producers: 16-byte copies into swizzled stages ==========
    // eight consecutive lanes copy one 128-byte row of a chunk (coalesced); a warp covers
    // four rows per pass, the four producer warps 16 rows, eight passes the 128 rows
    const int u = lane & 7;
    const int rsub = warp * 4 + (lane >> 3);
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % kStages;
      if (kc >= kStages) {
        bool ok = !*(volatile int*)&abort_flag;
        if (ok && !mbar_wait(&empty_bar[s], ((kc / kStages) - 1) & 1)) {
          report(a.status, SA_ERR_TIMEOUT);
          atomicExch(&abort_flag, 1);
        }
      }
      const uint32_t sa_ = st0 + s * kStageBytes;
#pragma unroll
      for (int i = 0; i < kTile / 16; ++i) {
        const int r = 16 * i + rsub;
        const int ph = row_ph[r];
        const uint32_t off = (uint32_t)(r * kRowBytes + ((u ^ (r & 7)) << 4));
        // rows outside the sequence are zero-filled (source size 0)
        cp_async16(sa_ + off, a.summ + (size_t)(ph < 0 ? 0 : ph) * (kK * 2) + kc * kRowBytes + u * 16,
                   ph < 0 ? 0u : 16u);
        cp_async16(sa_ + kOpBytes + off,
                   a.qs + ((size_t)b * kG + r) * (kK * 2) + kc * kRowBytes + u * 16, 16u);
      }
      cp_async_commit();
      // the stage issued kStages-1 chunks ago has landed: publish it to the MMA thread
      if (kc >= kStages - 1) {
        cp_async_wait<kStages - 1>();
        fence_proxy_async_smem();
        mbar_arrive(&full_bar[(kc - (kStages - 1)) % kStages]);
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    for (int kc = kChunks - (kStages - 1); kc < kChunks; ++kc) mbar_arrive(&full_bar[kc % kStages]);
  } else {
    // ===================== MMA issue (one thread) =====================
    if (warp == 4 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kTile, kG);
      bool ok = true;
      for (int kc = 0; kc < kChunks && ok; ++kc) {
        const int s = kc % kStages;
        if (*(volatile int*)&abort_flag || !mbar_wait(&full_bar[s], (kc / kStages) & 1)) {
          report(a.status, SA_ERR_TIMEOUT);
          atomicExch(&abort_flag, 1);
          ok = false;
          break;
        }
        mla::tc_fence_after();
        const uint32_t sa_ = st0 + s * kStageBytes;
#pragma unroll
        for (int k = 0; k < kChunk / 16; ++k) {
          // advancing K by 16 elements = 32 bytes inside the swizzled 128-byte rows
          umma_bf16(tmem, desc_sw128(sa_ + k * 32), desc_sw128(sa_ + kOpBytes + k * 32), idesc,
                    (kc | k) != 0);
        }
        umma_commit(&empty_bar[s]);  // the stage is free once these MMAs have read it
      }
      umma_commit(&done_bar);  // all issued MMAs complete -> accumulator ready
    }
    __syncwarp();
    // ===================== epilogue: lane (page) row max over 128 heads ==========
    const int wq = warp - 4;  // TMEM lanes 32*wq .. 32*wq + 31
    // warp-uniform: tcgen05.ld below is a .sync.aligned warp instruction
    const bool ready = __all_sync(0xffffffffu, mbar_wait(&done_bar, 0));
    mla::tc_fence_after();
    float m = -INFINITY;
    if (ready) {
#pragma unroll
      for (int c0 = 0; c0 < kG; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * wq) << 16) + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, v[i]);
      }
    } else if (lane == 0) {
      report(a.status, SA_ERR_TIMEOUT);
    }
    const int p = p0 + 32 * wq + lane;
    if (p < a.max_pages) srow[p] = (p < nb && !*(volatile int*)&abort_flag) ? m : -INFINITY;
  }
  mla::tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    mla::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128)
                 : "memory");
  }
}

static cudaError_t launch_pdl_mla(const void* fn, dim3 grid, dim3 block, size_t smem,
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

size_t mla_qsplit_bytes(const sa_geom& g) { return (size_t)g.B * mla::kG * mla::kK * 2; }

cudaError_t launch_score_mla(const sa_geom& g, const void* q, const void* summ, void* qs,
                             const int32_t* page_table, const int32_t* seq_lens, float* scores,
                             int32_t* status, cudaStream_t stream) {
  const int rows = g.B * mla::kG;
  const int n_thr = rows * (mla::kD / 8);
  const uint4* qv = static_cast<const uint4*>(q);
  uint4* qsv = static_cast<uint4*>(qs);
  void* qargs[] = {&qv, &qsv, const_cast<int*>(&rows)};
  cudaError_t e = launch_pdl_mla(reinterpret_cast<const void*>(mla_qsplit_kernel),
                                 dim3((n_thr + 255) / 256), dim3(256), 0, stream, qargs);
  if (e != cudaSuccess) return e;
  MlaScoreArgs a;
  a.summ = static_cast<const uint8_t*>(summ);
  a.qs = static_cast<const uint8_t*>(qs);
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.scores = scores;
  a.status = status;
  a.P = g.P;
  a.max_pages = g.max_pages;
  a.n_pool = g.n_pool;
  const void* kern = reinterpret_cast<const void*>(score_mla_kernel);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  const int tiles = (g.max_pages + mla::kTile - 1) / mla::kTile;
  return launch_pdl_mla(kern, dim3(tiles, g.B), dim3(mla::kThreads), mla::kSmem, stream, args);
}

// =====================================================================================
// Latent attention over the selected pages (tcgen05).
//
// Method: exact softmax attention of the 128 query heads over the tokens of the selected
// pages, V = the first 512 channels of each token's latent row (SubQ/SSA article, SSA
// section; Vortex summary, section 1: pages reached through the page table), split into
// chunks of 256 tokens per CTA and merged by log-sum-exp.
//
// Warps 0-3 stage operands, warp 8 issues the MMAs (it must not be one of the softmax
// warps: the P . V MMAs wait for their arrival), warps 4-7 (TMEM lane quarters 0-3) run
// the softmax and the epilogue.
// Per CTA (sequence b, chunk): S = Q K^T (M = 128 heads, N = 256 tokens, K = 576 in 9
// chunks of 64 channels) accumulates in TMEM columns [0, 256); the epilogue warps (one
// TMEM lane = one head each) take the exact softmax over the chunk and write P (bf16) to
// shared memory in the swizzled K-major layout; O = P V (M = 128, N = 64 channels per
// MMA, K = 256 tokens) then accumulates in TMEM columns [0, 512).  The V operand is
// MN-major: the bytes of a token's 64-channel slice sit at the same swizzled place as the
// K operand's chunk, so both phases use one staging routine (the second read of those
// rows comes from L2).  The chunk's (m, l) and unnormalised O are written to the
// workspace ([channel][head], coalesced) and attend_mla_merge_kernel combines the chunks.
// =====================================================================================

namespace mla {
constexpr int kDv = 512;
constexpr int kTok = 256;                       // tokens per CTA (UMMA N of Q K^T)
constexpr int kQChunk = kG * kRowBytes;         // 16 KB: 128 head rows x 128 B
constexpr int kKChunk = kTok * kRowBytes;       // 32 KB: 256 token rows x 128 B
constexpr int kAStage = kQChunk + kKChunk;      // 48 KB
constexpr int kAStages = 3;
constexpr int kPBytes = kG * kTok * 2;          // 64 KB: P, 4 chunks of 64 tokens
constexpr int kQkChunks = kD / kChunk;          // 9
constexpr int kPvChunks = kDv / kChunk;         // 8
constexpr size_t kAttnSmem = 1024 + (size_t)kAStages * kAStage + kPBytes;
constexpr int kAttnThreads = 288;  // 4 producer, 4 softmax/epilogue, 1 MMA-issue warps

// MN-major operand with 128-byte swizzle: 64 N-elements per 128-byte row, rows = K,
// 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(32768 >> 4) << 16;  // stride between 64-element N atoms (one atom here)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride between 8-row K groups
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
}  // namespace mla

struct MlaAttnArgs {
  const uint8_t* q;        // [B][128][576] bf16
  const uint8_t* kv;       // [n_pool][1][P][576] bf16 latent rows
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* sel;      // [B][1][sel_stride]
  const int32_t* sel_count;
  const int32_t* sel_phys;  // nullable
  float* part_o;            // [B][n_split][512][128]
  float* part_ml;           // [B][n_split][128][2]
  int32_t* status;
  int P, max_pages, n_pool, sel_stride, n_split;
  float scale_log2;
};

__global__ void __launch_bounds__(mla::kAttnThreads, 1) attend_mla_kernel(const MlaAttnArgs a) {
  using namespace mla;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* pbuf = stages + kAStages * kAStage;  // P, 1024-aligned
  __shared__ __align__(8) uint64_t full_bar[kAStages];
  __shared__ __align__(8) uint64_t empty_bar[kAStages];
  __shared__ __align__(8) uint64_t s_done, p_ready, o_done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ uint32_t valid_mask[kTok / 32];
  __shared__ int tok_row[kTok];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, b = blockIdx.y;
  const int ppc = kTok / a.P;  // pages per chunk

  if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;");
  const int L = min(max(a.seq_lens[b], 0), a.max_pages * a.P);
  const int nb = (L + a.P - 1) / a.P;
  const int cnt = min(max(a.sel_count[b], 0), a.sel_stride);
  const int i0 = split * ppc;
  float* pml = a.part_ml + ((size_t)b * a.n_split + split) * kG * 2;
  if (i0 >= cnt) {  // nothing selected in this chunk: an empty state
    if (tid < kG) {
      pml[tid * 2] = -INFINITY;
      pml[tid * 2 + 1] = 0.f;
    }
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&full_bar[s], 128);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&s_done, 1);
    mbar_init(&p_ready, 128);
    mbar_init(&o_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  // token rows of this chunk (thread r: tokens r and r + 128): latent row index in the
  // pool (-1: zero row) and the mask of valid tokens, before the barrier that publishes
  // them to the producers and the softmax warps
  if (warp < 4) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int t = tid + 128 * h2;
      const int i = i0 + t / a.P;
      const int slot = t % a.P;
      int row = -1;
      if (i < cnt) {
        const int lp = a.sel[(size_t)b * a.sel_stride + i];
        if (lp >= 0 && lp < nb) {
          const int ph = a.sel_phys ? a.sel_phys[(size_t)b * a.sel_stride + i]
                                    : a.page_table[(size_t)b * a.max_pages + lp];
          if (ph < 0 || ph >= a.n_pool)
            report(a.status, SA_ERR_DEVICE_CHECK);
          else if (lp * a.P + slot < L)
            row = ph * a.P + slot;
        }
      }
      tok_row[t] = row;
      const unsigned m = __ballot_sync(0xffffffffu, row >= 0);
      if (lane == 0) valid_mask[t >> 5] = m;
    }
  }
  if (warp == 8) {  // all 512 TMEM columns: S in [0,256), later O in [0,512)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t st0 = smem_u32(stages);
  const uint32_t pb0 = smem_u32(pbuf);

  if (warp < 4) {
    // ===================== producers =====================
    // eight consecutive lanes copy one 128-byte row of a chunk (coalesced): 8 passes of
    // 16 rows for the 128 query rows, 16 passes for the 256 token rows
    const int u = lane & 7;
    const int rsub = warp * 4 + (lane >> 3);
    // 9 chunks of (Q, K) for S, then 8 chunks of V (the first 512 channels) for O
    for (int it = 0; it < kQkChunks + kPvChunks; ++it) {
      const int s = it % kAStages;
      if (it >= kAStages) {
        if (!*(volatile int*)&abort_flag &&
            !mbar_wait(&empty_bar[s], ((it / kAStages) - 1) & 1)) {
          report(a.status, SA_ERR_TIMEOUT);
          atomicExch(&abort_flag, 1);
        }
      }
      const int kc = it < kQkChunks ? it : it - kQkChunks;
      const uint32_t sq = st0 + s * kAStage;
      const uint32_t sk = sq + kQChunk;
      if (it < kQkChunks) {
#pragma unroll
        for (int i = 0; i < kG / 16; ++i) {
          const int r = 16 * i + rsub;
          cp_async16(sq + r * kRowBytes + ((u ^ (r & 7)) << 4),
                     a.q + ((size_t)b * kG + r) * (kD * 2) + kc * kRowBytes + u * 16, 16u);
        }
      }
#pragma unroll 4
      for (int i = 0; i < kTok / 16; ++i) {
        const int t = 16 * i + rsub;
        const int row = tok_row[t];
        // tokens outside the selection are zero-filled (source size 0)
        cp_async16(sk + t * kRowBytes + ((u ^ (t & 7)) << 4),
                   a.kv + (size_t)(row < 0 ? 0 : row) * (kD * 2) + kc * kRowBytes + u * 16,
                   row < 0 ? 0u : 16u);
      }
      cp_async_commit();
      if (it >= kAStages - 1) {
        cp_async_wait<kAStages - 1>();
        fence_proxy_async_smem();
        mbar_arrive(&full_bar[(it - (kAStages - 1)) % kAStages]);
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    for (int it = kQkChunks + kPvChunks - (kAStages - 1); it < kQkChunks + kPvChunks; ++it)
      mbar_arrive(&full_bar[it % kAStages]);
  } else if (warp == 8) {
    // ===================== MMA issue (one thread of its own warp) =====================
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kG, kTok);
      constexpr uint32_t idesc_o = idesc_bf16(kG, 64) | (1u << 16);  // B (V) MN-major
      bool ok = true;
      for (int it = 0; it < kQkChunks + kPvChunks && ok; ++it) {
        const int s = it % kAStages;
        if (it == kQkChunks) {
          umma_commit(&s_done);  // S complete -> softmax
          if (!mbar_wait(&p_ready, 0)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (*(volatile int*)&abort_flag || !mbar_wait(&full_bar[s], (it / kAStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sq = st0 + s * kAStage;
        const uint32_t sk = sq + kQChunk;
        if (it < kQkChunks) {
#pragma unroll
          for (int k = 0; k < kChunk / 16; ++k)
            umma_bf16(tmem, desc_sw128(sq + k * 32), desc_sw128(sk + k * 32), idesc_s,
                      (it | k) != 0);
        } else {
          const int cb = it - kQkChunks;  // channels 64*cb .. 64*cb + 63
#pragma unroll 4
          for (int kk = 0; kk < kTok / 16; ++kk)
            umma_bf16(tmem + 64 * cb,
                      desc_sw128(pb0 + (kk >> 2) * (kG * kRowBytes) + (kk & 3) * 32),
                      desc_sw128_mn(sk + kk * 16 * kRowBytes), idesc_o, kk != 0);
        }
        umma_commit(&empty_bar[s]);
      }
      if (!ok) {
        report(a.status, SA_ERR_TIMEOUT);
        atomicExch(&abort_flag, 1);
        umma_commit(&s_done);  // never leave the epilogue waiting (bounded anyway)
      }
      umma_commit(&o_done);
    }
    __syncwarp();
  } else {
    const int wq = warp - 4;  // TMEM lanes 32*wq .. : heads 32*wq + lane
    const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
    // ===================== softmax over the chunk (one head per thread) ==========
    const int head = 32 * wq + lane;
    bool ready = __all_sync(0xffffffffu, mbar_wait(&s_done, 0));
    tc_fence_after();
    float m = -INFINITY, l = 0.f;
    if (ready) {
#pragma unroll 1
      for (int c0 = 0; c0 < kTok; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + c0, v);
        const uint32_t vm = valid_mask[c0 >> 5];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if ((vm >> i) & 1) m = fmaxf(m, v[i] * a.scale_log2);
      }
      // P = 2^(x - m) in bf16, K-major swizzled rows (row = head), and l = sum of P
#pragma unroll 1
      for (int c0 = 0; c0 < kTok; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + c0, v);
        const uint32_t vm = valid_mask[c0 >> 5];
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ((vm >> (2 * i)) & 1) ? fast_exp2(v[2 * i] * a.scale_log2 - m) : 0.f;
          const float p1 =
              ((vm >> (2 * i + 1)) & 1) ? fast_exp2(v[2 * i + 1] * a.scale_log2 - m) : 0.f;
          l += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        // tokens c0 .. c0+31 = chunk c0/64, 16-byte units (c0 % 64)/8 .. +3
        const uint32_t rowp = pb0 + (c0 >> 6) * (kG * kRowBytes) + head * kRowBytes;
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const int u = ((c0 & 63) >> 3) + u4;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           rowp + ((u ^ (head & 7)) << 4)),
                       "r"(pk[4 * u4]), "r"(pk[4 * u4 + 1]), "r"(pk[4 * u4 + 2]),
                       "r"(pk[4 * u4 + 3])
                       : "memory");
        }
      }
    }
    fence_proxy_async_smem();  // P (generic stores) -> tensor-core reads
    tc_fence_before();
    mbar_arrive(&p_ready);
    // ===================== O epilogue: the chunk's state to the workspace ==========
    ready = __all_sync(0xffffffffu, mbar_wait(&o_done, 0)) && ready;
    tc_fence_after();
    const bool good = ready && !*(volatile int*)&abort_flag;
    float* po = a.part_o + ((size_t)b * a.n_split + split) * kDv * kG;
    if (good) {
#pragma unroll 1
      for (int c0 = 0; c0 < kDv; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) po[(size_t)(c0 + i) * kG + head] = v[i];
      }
    } else if (lane == 0) {
      report(a.status, SA_ERR_TIMEOUT);
    }
    pml[head * 2] = good ? m : -INFINITY;
    pml[head * 2 + 1] = good ? l : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

// Combine the chunk states of each (sequence, head): out = sum_s 2^(m_s - M) O_s / L,
// lse = (M + log2 L) ln 2.  CTA = (sequence, 32 channels); thread = head.
constexpr int kMergeCh = 8;  // channels per merge CTA: B * 64 CTAs at the latent geometry

__global__ void __launch_bounds__(128) attend_mla_merge_kernel(const float* __restrict__ part_o,
                                                               const float* __restrict__ part_ml,
                                                               float* __restrict__ out,
                                                               float* __restrict__ lse,
                                                               int n_split) {
  using namespace mla;
  __shared__ float tile[kG][kMergeCh + 1];
  if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;");
  const int b = blockIdx.y, c0 = blockIdx.x * kMergeCh, h = threadIdx.x;
  const float* ml = part_ml + (size_t)b * n_split * kG * 2;
  // running maximum first (the splits' loads in flight together), then the weighted
  // sums in split order
  float M = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, ml[((size_t)s * kG + h) * 2]);
  float Lsum = 0.f, acc[kMergeCh];
#pragma unroll
  for (int i = 0; i < kMergeCh; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int s = 0; s < n_split; ++s) {
    const float ms = ml[((size_t)s * kG + h) * 2];
    if (ms == -INFINITY) continue;  // an empty chunk: its O is not read
    const float w = fast_exp2(ms - M);
    Lsum += w * ml[((size_t)s * kG + h) * 2 + 1];
    const float* po = part_o + (((size_t)b * n_split + s) * kDv + c0) * kG + h;
#pragma unroll
    for (int i = 0; i < kMergeCh; ++i) acc[i] += w * po[(size_t)i * kG];
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
  for (int i = 0; i < kMergeCh; ++i) tile[h][i] = acc[i] * inv;
  if (blockIdx.x == 0)
    lse[(size_t)b * kG + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
  __syncthreads();
  // write rows out[b][h][c0 .. c0+7]: 2 threads per head row, 4 floats each
  for (int e = h; e < kG * (kMergeCh / 4); e += 128) {
    const int hh = e / (kMergeCh / 4), q4 = (e % (kMergeCh / 4)) * 4;
    *reinterpret_cast<float4*>(out + ((size_t)b * kG + hh) * kDv + c0 + q4) =
        make_float4(tile[hh][q4], tile[hh][q4 + 1], tile[hh][q4 + 2], tile[hh][q4 + 3]);
  }
}

int mla_attend_splits(const sa_geom& g, int sel_stride) {
  const int ppc = mla::kTok / g.P;
  return (sel_stride + ppc - 1) / ppc;
}

size_t mla_attend_part_bytes(const sa_geom& g, int sel_stride) {
  const size_t ns = (size_t)mla_attend_splits(g, sel_stride);
  return (size_t)g.B * ns * mla::kG * (mla::kDv + 2) * 4;
}

cudaError_t launch_attend_mla(const sa_geom& g, const void* q, const void* kv,
                              const int32_t* page_table, const int32_t* seq_lens,
                              const int32_t* sel, const int32_t* sel_count,
                              const int32_t* sel_phys, int sel_stride, float scale, float* part,
                              float* out, float* lse, int32_t* status, cudaStream_t stream) {
  MlaAttnArgs a;
  a.q = static_cast<const uint8_t*>(q);
  a.kv = static_cast<const uint8_t*>(kv);
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.sel = sel;
  a.sel_count = sel_count;
  a.sel_phys = sel_phys;
  a.n_split = mla_attend_splits(g, sel_stride);
  a.part_o = part;
  a.part_ml = part + (size_t)g.B * a.n_split * mla::kDv * mla::kG;
  a.status = status;
  a.P = g.P;
  a.max_pages = g.max_pages;
  a.n_pool = g.n_pool;
  a.sel_stride = sel_stride;
  a.scale_log2 = scale * 1.4426950408889634f;
  const void* kern = reinterpret_cast<const void*>(attend_mla_kernel);
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::kAttnSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  e = launch_pdl_mla(kern, dim3(a.n_split, g.B), dim3(mla::kAttnThreads), mla::kAttnSmem,
                     stream, args);
  if (e != cudaSuccess) return e;
  const float* po = a.part_o;
  const float* pml = a.part_ml;
  int ns = a.n_split;
  void* margs[] = {&po, &pml, &out, &lse, &ns};
  return launch_pdl_mla(reinterpret_cast<const void*>(attend_mla_merge_kernel),
                        dim3(mla::kDv / kMergeCh, g.B), dim3(128), 0, stream, margs);
}

}  // namespace sa
