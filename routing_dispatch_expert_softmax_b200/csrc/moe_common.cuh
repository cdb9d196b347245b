// Shared definitions of the B200 MoE library: workspace layout, error word,
// and thin inline-PTX wrappers for mbarriers, TMA and the tcgen05 tensor
// cores (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ----------------------------------------------------------------- constants
constexpr int kTokensPerRouteBlock = 256;  // tokens per block in hist/scatter
constexpr int kGemmBM = 128;               // activation rows per GEMM tile
constexpr int kGemmBK = 64;                // K elements per pipeline stage
constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kMaxR = 64;
// Batches of at most this many tokens (so at most this many rows per expert)
// run the expert GEMMs in swap-AB form.
constexpr int kSwapMaxT = 256;

// Large batches whose experts average at least one full 128-row tile run the
// expert GEMMs on CTA pairs (256-row tiles); their work lists then split each
// expert's tiles into pairs and at most one leftover tile.  Between kSwapMaxT
// and this density the single-CTA kernel runs all 128-row tiles.
inline bool pair_tiles(const moe_shape& s) {
  return s.T > kSwapMaxT && (long long)s.T * s.k >= (long long)128 * s.E;
}

// Batches above this many tokens compute router logits on the tensor cores.
constexpr int kRouterTcMinT = 257;

// Tensor-core router: K = 3d (three bf16 planes of W_g) is split into P
// partitions of whole 64-wide blocks (at least 4 per part), each a separate
// work item writing an fp32 partial plane that a finish kernel adds in
// partition order.  P is the largest divisor of the block count that keeps
// tiles * P within one wave of kRouterTargetItems work items: a 128 x E
// logit tile streams 32 KB of operands per 64-deep K block, so one SM alone
// cannot feed its tensor cores and the tiles must be spread over all SMs.
constexpr int kRouterTargetItems = 148;
inline int router_tc_parts(const moe_shape& s) {
  if (s.T < kRouterTcMinT) return 0;
  const int bn = s.E <= 128 ? 128 : 256;
  const long long tiles = (long long)((s.T + 127) / 128) * ((s.E + bn - 1) / bn);
  const int nk = 3 * s.d / 64;  // 64-wide K blocks over the three planes
  int best = 1;
  for (int P = 2; P <= nk / 4; ++P) {
    if (nk % P != 0) continue;
    if (tiles * P > kRouterTargetItems) break;
    best = P;
  }
  return best;
}

// Workspace header (the 64 bytes the caller zeroes once): ws[0] = first error
// code, ws[1] = detail (kernel id), ws[2] = the fused routing kernel's block
// ticket (back to 0 at the end of every call).
enum : int { kErrSlot = 0, kErrDetail = 1, kRouteTicket = 2 };

// Every bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ void record_error(int* err, int code, int detail) {
  if (atomicCAS(err + kErrSlot, 0, code) == 0) err[kErrDetail] = detail;
}

// The shape limits every C-ABI entry point accepts (include/moe.h, moe_shape).
inline bool shape_valid(const moe_shape* s) {
  if (!s) return false;
  if (s->T < 0 || s->T > (1 << 20)) return false;
  if (s->d < 64 || s->d > 16384 || s->d % 64) return false;
  if (s->E < 1 || s->E > kMaxE) return false;
  if (s->k < 1 || s->k > kMaxK || s->k > s->E) return false;
  if (s->f < 64 || s->f > 32768 || s->f % 64) return false;
  if (s->R < 0 || s->R > kMaxR) return false;
  if (s->R > 1 && s->E % s->R) return false;
  return true;
}

// ----------------------------------------------------------------- workspace
struct WsLayout {
  size_t err, w3, logit_part, logits, idx, idx_phys, w, counts, offsets, blockhist, blockbase,
      blocksend, send, rank_off, perm, row_of, tiles, x_perm, h, z, xs, hq, hs, total;
  int nblocks;      // token blocks of kTokensPerRouteBlock
  int max_mtiles;   // upper bound of 128-row expert tiles
  long long P;      // T * k
  long long Ppad;   // rows of x_perm / h including the TMA padding
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Work lists the routing kernels build for the expert GEMMs, in one int
// buffer: [0] = number of 128-row tiles in the row-tile list, [1] = number of
// touched experts, [2] = number of leftover tiles; then E entries (row0,
// row_end, expert) for the touched experts in expert order, then E leftover
// entries, then the row tiles (row0, row_end, expert), 128 rows each.  When
// the expert GEMMs run on CTA pairs (pair_row_tiles), an expert's tile count
// is rounded up to an even number so pairs never span experts, except that an
// expert with a single tile goes to the leftover list, which a single-CTA
// kernel runs; otherwise every tile is a row tile and the leftover list is
// empty.
// Row tiles of an expert with nt 128-row tiles in the CTA-pair layout.  An
// odd count is padded to the next pair: the pair's empty half costs MMA work
// but the expert's weights stream through L2 once.  A lone tile (nt = 1)
// would be half empty, so it runs as a single-CTA leftover tile instead.
__host__ __device__ inline int pair_row_tiles(int nt) { return nt == 1 ? 0 : (nt + 1) & ~1; }

// Upper bound of the row-tile list: each expert one partial tile and, in the
// CTA-pair layout, one padding tile.
__host__ __device__ inline int max_mtiles_of(long long P, int E) {
  return (int)((P + kGemmBM - 1) / kGemmBM + 2 * E);
}
// After the lists: one ready counter per list entry (max_mtiles + E of them),
// zeroed by every kernel that writes the lists.  The small-batch GEMM1 adds 1
// to entry i's counter when one of its column tiles of that entry's rows is
// stored; GEMM2 starts an entry's work once the count is complete.
// One more int after them: the small-batch GEMM2's item queue; then a second
// array of counters and its queue, laid out the same way (the W8A8 layer's
// quantised entries, which its GEMM2 waits on).
__host__ __device__ inline size_t tile_list_ints(int max_mtiles, int E) {
  return 4 + 3 * ((size_t)max_mtiles + 2 * (size_t)E) + 2 * ((size_t)max_mtiles + E + 1);
}
__host__ __device__ inline int* ready_counters(int* tiles, int max_mtiles, int E) {
  return tiles + 4 + 3 * ((size_t)max_mtiles + 2 * (size_t)E);
}
// ints after ready_counters() that the list writers zero: both arrays and their queues
__host__ __device__ inline int ready_ints(int max_mtiles, int E) {
  return 2 * (max_mtiles + E + 1);
}
__host__ __device__ inline int* expert_entries(int* tiles) { return tiles + 4; }
__host__ __device__ inline int* leftover_entries(int* tiles, int E) { return tiles + 4 + 3 * E; }
__host__ __device__ inline int* row_tile_entries(int* tiles, int E) { return tiles + 4 + 6 * E; }

// E_tab: experts of the dispatch tables and expert GEMMs (the physical
// experts when replicas are used, moe_forward_eplb); the router regions use
// the s.E logical experts.  -1: E_tab = s.E.
inline WsLayout ws_layout(const moe_shape& s, int num_sms, int E_tab = -1) {
  WsLayout L{};
  const long long T = s.T, k = s.k, d = s.d, f = s.f;
  const long long E_log = s.E;
  const long long E = E_tab > 0 ? E_tab : s.E;
  const long long R = s.R > 1 ? s.R : 1;
  L.P = T * k;
  L.Ppad = L.P + kGemmBM;
  L.nblocks = (int)((T + kTokensPerRouteBlock - 1) / kTokensPerRouteBlock);
  // each expert: one partial tile and, in the CTA-pair layout, one padding tile
  L.max_mtiles = max_mtiles_of(L.P, (int)E);
  (void)num_sms;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.err = take(64);
  L.w3 = take(2 * 3 * (size_t)d * E_log);  // router weight split into 3 bf16 planes
  L.logit_part = take(sizeof(float) * (size_t)router_tc_parts(s) * T * E_log);

  L.logits = take(sizeof(float) * T * E_log);
  L.idx = take(sizeof(int) * T * k);
  L.idx_phys = take(sizeof(int) * T * k);
  L.w = take(sizeof(float) * T * k);
  L.counts = take(sizeof(int) * E);
  L.offsets = take(sizeof(int) * (E + 1));
  L.blockhist = take(sizeof(int) * (size_t)L.nblocks * E);
  L.blockbase = take(sizeof(int) * (size_t)L.nblocks * E);
  L.blocksend = take(sizeof(int) * (size_t)L.nblocks * R * R);
  L.send = take(sizeof(int) * R * R);
  L.rank_off = take(sizeof(int) * (R + 1));
  L.perm = take(sizeof(int) * L.P);
  L.row_of = take(sizeof(int) * L.P);
  L.tiles = take(sizeof(int) * tile_list_ints(L.max_mtiles, (int)E));
  L.x_perm = take(2 * (size_t)L.Ppad * d);
  L.h = take(2 * (size_t)L.Ppad * f);
  L.z = take(2 * (size_t)L.P * d);
  // FP8 activations: the token codes take the x_perm region (one byte per
  // element instead of two); their row scales, the SwiGLU output's codes and
  // its row scales have their own.
  L.xs = take(sizeof(float) * (size_t)L.Ppad);
  L.hq = take((size_t)L.Ppad * f);
  L.hs = take(sizeof(float) * (size_t)L.Ppad);
  L.total = o;
  return L;
}

// ----------------------------------------------------------------- PTX: misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch: every kernel of the layer lets the next one
// launch as soon as all of its own CTAs are running (trigger), and waits for
// its predecessor grid to complete and publish its memory before touching
// any global data (wait).  The next kernel's launch and prologue then overlap
// this kernel's tail.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ bool elect_one_lane() {
  return (threadIdx.x & 31) == 0;
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

// Raises the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete.  Gives up
// (returns false) once *abort is set by another thread or after kWaitLimitNs;
// in the latter case it sets *abort itself so every other wait gives up too.
__device__ __forceinline__ bool mbar_wait_bounded(
    uint64_t* bar, uint32_t parity, volatile int* abort,
    unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort = 1;
      return false;
    }
  }
}

// Orders this thread's generic-proxy global accesses with later async-proxy
// (TMA) accesses, in both directions.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Spins until *counter >= target (acquire, GPU scope), with the bounded-wait
// limit; on timeout sets *abort_flag and returns false.
__device__ __forceinline__ bool wait_count_bounded(const int* counter, int target,
                                                   volatile int* abort_flag) {
  const unsigned long long t0 = globaltimer();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= target) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
}

// ----------------------------------------------------------------- TMA
// 2-D tiled bulk tensor load into shared memory, completing on `bar`.
// c0 is the innermost (contiguous) coordinate in elements, c1 the row.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* tm,
                                            uint64_t* bar, int c0, int c1,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes.L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(c0), "r"(c1),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm))
               : "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
          smem_u32(smem_result)),
      "r"(ncols)
      : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D(tmem) (+)= A(smem) * B(smem)^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16_ss(uint32_t tmem_d, uint64_t adesc,
                                             uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D (+)= A * B^T with E4M3 A and B from shared memory (K = 32 per instruction).
__device__ __forceinline__ void umma_e4m3_ss(uint32_t tmem_d, uint64_t adesc,
                                             uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05.mma issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (quarter*32 + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]),
        "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 64 bf16 (128 B), 8-row groups 1024 B apart.
// Field layout (sm_100 UMMA descriptor): start address >> 4 in bits [0,14),
// leading byte offset >> 4 in [16,30) (1 for swizzled K-major), stride byte
// offset >> 4 in [32,46), descriptor version 1 in [46,48), layout type in
// [61,64) (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t desc = 0;
  desc |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  desc |= (uint64_t)1 << 16;
  desc |= (uint64_t)(1024 >> 4) << 32;
  desc |= (uint64_t)1 << 46;
  desc |= (uint64_t)2 << 61;
  return desc;
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D, both
// operands K-major, shape M x N.  Bits: D format [4,6) = 1 (f32); A format
// [7,10) = 1 (bf16); B format [10,13) = 1 (bf16); A/B major bits 15/16 = 0
// (K-major); N >> 3 in [17,23); M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// The same for kind::f8f6f4 with E4M3 A and B (format code 0 in both fields).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ----------------------------------------------------------------- bf16
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Launches `kern` on `st` with programmatic stream serialization (so the
// kernel may start while its predecessor finishes; it synchronises with
// pdl_wait) and, if cluster > 1, a 1-D thread-block cluster.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t st, int cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace moe
