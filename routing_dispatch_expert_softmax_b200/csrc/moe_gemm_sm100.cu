// Expert FFN grouped GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Serving MoE models with expert parallelism on 8xH200", section "Tensor
// parallel vs expert parallel": each expert's tokens go through full-size
// expert GEMMs; section "Batching ...": at small batch the expert GEMM streams
// the expert's weights from HBM for a handful of token rows.
//
// One persistent kernel template serves both GEMMs of the SwiGLU expert:
//   GEMM1 (SWIGLU = true):  A = x_perm rows, B = [Wg_e^T tile ; Wu_e^T tile],
//                           epilogue h = silu(g) * u  -> bf16 h
//   GEMM2 (SWIGLU = false): A = h rows, B = Wd_e^T tile -> bf16 z
// Work item = (128-row tile of one expert, BN-wide output tile).  The list of
// row tiles is built on the device from the expert offsets, so the launch
// needs no host synchronisation; the grid is one CTA per SM and each CTA
// strides through the work items.
//
// CTA = 6 warps: warp 0 issues TMA loads (one thread), warp 1 owns TMEM and
// issues tcgen05.mma (one thread), warps 2-5 drain the accumulator (TMEM lane
// quarter = warp % 4).  Shared memory holds STAGES (A, B) K-slices of 64
// elements in the 128-byte-swizzled K-major layout; TMEM holds two fp32
// accumulators of 128 x BN so the epilogue of one tile overlaps the MMAs of
// the next.  Every wait is bounded (error word MOE_ERR_TIMEOUT, then drain and
// return).
#include "moe_kernels.cuh"

namespace moe {

// Epilogues of the grouped GEMM.
enum : int {
  kEpiSwiGLU = 0,  // h = silu(gate) * up -> bf16 (columns [0,BN/2) gate, [BN/2,BN) up)
  kEpiStore = 1,   // bf16 copy of the accumulator
  kEpiLogits = 2   // fp32 accumulator + bias[col] (router logits)
};

// Where a GEMM kernel synchronises with the kernels before and after it
// (programmatic dependent launch):
//   kPdlStart:     lets the next kernel launch, then waits for the previous one
//                  before touching its outputs (the usual chain).
//   kPdlAfterWait: waits first, then lets the next kernel launch, so the next
//                  kernel may read everything complete before this one began.
//   kPdlTail:      reads only data complete before the previous kernel began
//                  (which must be kPdlAfterWait), so it starts without waiting
//                  and fills the SMs the previous kernel's tail leaves idle; it
//                  lets the next kernel launch at once (so that kernel's set-up
//                  is not exposed) and waits for the previous kernel at its
//                  end, so its own completion implies both.
enum : int { kPdlStart = 0, kPdlAfterWait = 1, kPdlTail = 2 };

struct GemmArgs {
  const int* tile_count;  // device number of row tiles; nullptr = dense rows [0, dense_rows)
  const int* tile_rows;   // (row0, row_end, expert) per 128-row tile
  int E;                  // experts
  int dense_rows;         // rows of A in dense mode
  int n_tiles;            // output tiles of width BN (BN/2 for SwiGLU) per row tile
  int K;                  // reduction length of B (multiple of 64)
  int a_kblocks;          // A's K coordinate is (kb mod a_kblocks) * 64
  int b_rows_per_expert;  // B rows owned by one expert
  int up_offset;          // SwiGLU: B row offset of the up half
  int n_out;              // valid output columns
  void* out;
  int ld_out;
  const float* bias;      // kEpiLogits only (may be null)
  int* err;
  int weights_once;       // 1: each B tile is read by one work item (hint evict_first)
  int kparts;             // K partitions per output tile (kEpiLogits; 1 otherwise)
  long long part_stride;  // elements between the partial outputs of two partitions
  int pdl;                // kPdlStart / kPdlAfterWait / kPdlTail
  const float* a_scale;   // E4M3 operands (the CTA-pair kernel's F8 form): one scale per A row
  const float* b_scale;   // and one per B row (weight row)
};

__device__ __forceinline__ void pdl_enter(int mode) {
  if (mode == kPdlStart) {
    pdl_trigger();
    pdl_wait();
  } else if (mode == kPdlAfterWait) {
    pdl_wait();
    pdl_trigger();
  } else {
    pdl_trigger();
  }
}

__device__ __forceinline__ void pdl_leave(int mode) {
  if (mode == kPdlTail) pdl_wait();
}

// Work-list entries another kernel wrote; read through L2 (not L1) so a
// kernel that starts without waiting never sees a stale line.
__device__ __forceinline__ int tile_ld(const int* p) { return __ldcg(p); }

template <int BN, int EPI>
struct GemmCfg {
  // The router (logits) epilogue's staging tile costs a K-stage: kernels of
  // a programmatic-launch chain measured slower above ~200 KB of shared memory.
  static constexpr int kStages = EPI == kEpiLogits ? ((BN == 256) ? 3 : 5) : ((BN == 256) ? 4 : 6);
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;  // 16 KB
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;  // double-buffered accumulator
  // Logits epilogue: per epilogue warp 32 rows x 32 fp32 staged for full-line stores.
  static constexpr int kOutStageBytes = EPI == kEpiLogits ? 4 * 32 * 128 : 0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kOutStageBytes + 1024 /*align*/ + 256;
  static constexpr int kThreads = 192;
};

__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity,
                                                unsigned long long limit_ns) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Grouped rasterization of the work items: row tiles are taken in groups of
// kRasterGroup; inside a group the output tile is the slow index, so the CTAs
// running at the same time share weight tiles (each read once from DRAM and
// reused by the group's row tiles from L2) and the group's activation tiles
// stay in L2 while the output tiles sweep past them.
constexpr int kRasterGroup = 16;

__device__ __forceinline__ void raster(int w, int n_tiles, int num_mtiles, int& mt, int& nt) {
  const int per_group = kRasterGroup * n_tiles;
  const int g = w / per_group;
  const int r = w - g * per_group;
  const int g0 = g * kRasterGroup;
  const int gsz = min(kRasterGroup, num_mtiles - g0);
  nt = r / gsz;
  mt = g0 + (r - nt * gsz);
}

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1) k_grouped_gemm(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const GemmArgs args) {
  using C = GemmCfg<BN, EPI>;
  constexpr int S = C::kStages;
  constexpr bool SWIGLU = (EPI == kEpiSwiGLU);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint4* out_stage = reinterpret_cast<uint4*>(smem + S * C::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kOutStageBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_enter(args.pdl);  // the work lists and operands come from earlier kernels

  const bool dense = args.tile_count == nullptr;
  const int num_mtiles =
      dense ? (args.dense_rows + kGemmBM - 1) / kGemmBM : tile_ld(args.tile_count);
  const int n_tiles = args.n_tiles * args.kparts;  // output tiles x K partitions
  const int ntn = args.n_tiles;
  const int total = num_mtiles * n_tiles;
  const int nk = args.K / kGemmBK;
  const int kpp = nk / args.kparts;  // K blocks per partition
  const int* tl = args.tile_rows;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      // Weight tiles used by a single row tile are streamed (evict first);
      // otherwise every row tile of the expert re-reads them from L2.
      const uint64_t pol_w = args.weights_once ? policy_evict_first() : policy_evict_normal();
      const uint64_t pol_a = policy_evict_normal();
      int fills[S];
#pragma unroll
      for (int s = 0; s < S; ++s) fills[s] = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        int mt, nt;
        raster(w, n_tiles, num_mtiles, mt, nt);
        const int part = nt / ntn, ntile = nt - part * ntn;
        const int row0 = dense ? mt * kGemmBM : tile_ld(tl + 3 * mt + 0);
        const int e = dense ? 0 : tile_ld(tl + 3 * mt + 2);
        const int brow = e * args.b_rows_per_expert + ntile * (SWIGLU ? BN / 2 : BN);
        const int kb0 = part * kpp;
        int ka = kb0 % args.a_kblocks;
        for (int kb = kb0; kb < kb0 + kpp; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + stage * C::kStageBytes;
          uint8_t* b_dst = a_dst + C::kABytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          tma_load_2d(a_dst, &tmA, &full[stage], ka * kGemmBK, row0, pol_a);
          if (++ka == args.a_kblocks) ka = 0;
          if (SWIGLU) {
            tma_load_2d(b_dst, &tmB, &full[stage], kb * kGemmBK, brow, pol_w);
            tma_load_2d(b_dst + (BN / 2) * 128, &tmB, &full[stage], kb * kGemmBK,
                        brow + args.up_offset, pol_w);
          } else {
            tma_load_2d(b_dst, &tmB, &full[stage], kb * kGemmBK, brow, pol_w);
          }
          ++fills[stage];
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // Let every copy already issued land before the CTA leaves.
#pragma unroll
        for (int s = 0; s < S; ++s)
          if (fills[s] > 0) mbar_wait_limit(&full[s], (uint32_t)((fills[s] - 1) & 1), 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t aph = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait_bounded(&tempty[ab], aph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(ab * BN);
        for (int kb = 0; kb < kpp; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk) {
            umma_bf16_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                         sw128_kmajor_desc(b_addr + kk * 32), idesc,
                         (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the smem slot when these MMAs finish
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[ab]);
      }
      if (*abort_flag) {
        umma_commit(drain);
        mbar_wait_limit(drain, 0, 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const int r_in_tile = q * 32 + lane;
    int it = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      int mt, nt_all;
      raster(w, n_tiles, num_mtiles, mt, nt_all);
      const int part = nt_all / ntn, nt = nt_all - part * ntn;
      const int row0 = dense ? mt * kGemmBM : tile_ld(tl + 3 * mt + 0);
      const int rowend = dense ? args.dense_rows : tile_ld(tl + 3 * mt + 1);
      const int ab = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      const bool got = mbar_wait_bounded(&tfull[ab], aph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + (uint32_t)(ab * BN) + ((uint32_t)(q * 32) << 16);
      const int row = row0 + r_in_tile;
      const bool row_ok = row < rowend;
      if (EPI == kEpiSwiGLU) {
        constexpr int H = BN / 2;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll 1
        for (int c = 0; c < H; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(t_addr + c, g);
          tmem_ld_32x32b_x32(t_addr + H + c, u);
          tmem_ld_wait();
          const int col = nt * H + c;
          if (row_ok && col < args.n_out) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              p[i] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * args.ld_out + col);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          }
        }
      } else if (EPI == kEpiStore) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t a[32];
          tmem_ld_32x32b_x32(t_addr + c, a);
          tmem_ld_wait();
          const int col = nt * BN + c;
          if (row_ok && col < args.n_out) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              p[i] = pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * args.ld_out + col);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          }
        }
      } else {
        float* out = static_cast<float*>(args.out) + (size_t)part * args.part_stride;
        // Rows of 16-byte-aligned fp32 vectors: stage each 32 x 32 slice in
        // the warp's tile (16-byte chunks XOR-swizzled by row) and store 4
        // whole 128-byte rows per instruction; otherwise one float at a time.
        const bool vec = (args.ld_out & 3) == 0 && (args.part_stride & 3) == 0 &&
                         (reinterpret_cast<uintptr_t>(args.out) & 15) == 0 &&
                         (!args.bias || (reinterpret_cast<uintptr_t>(args.bias) & 15) == 0);
        uint4* st_tile = out_stage + (size_t)(warp - 2) * 32 * 8;
        const int row_base = row0 + q * 32;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t a[32];
          tmem_ld_32x32b_x32(t_addr + c, a);
          tmem_ld_wait();
          const int col = nt * BN + c;
          if (vec) {
            if (col < args.n_out) {  // warp-uniform
#pragma unroll
              for (int v = 0; v < 8; ++v)
                st_tile[lane * 8 + (v ^ (lane & 7))] =
                    make_uint4(a[4 * v], a[4 * v + 1], a[4 * v + 2], a[4 * v + 3]);
              __syncwarp();
              const int v = lane & 7, cv = col + 4 * v;
              float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
              if (args.bias && cv < args.n_out)
                bv = __ldg(reinterpret_cast<const float4*>(args.bias + cv));
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int r = i * 4 + (lane >> 3);
                const uint4 u = st_tile[r * 8 + (v ^ (r & 7))];
                if (row_base + r < rowend && cv < args.n_out) {
                  const float4 o = make_float4(__uint_as_float(u.x) + bv.x,
                                               __uint_as_float(u.y) + bv.y,
                                               __uint_as_float(u.z) + bv.z,
                                               __uint_as_float(u.w) + bv.w);
                  *reinterpret_cast<float4*>(out + (size_t)(row_base + r) * args.ld_out + cv) =
                      o;
                }
              }
              __syncwarp();
            }
          } else if (row_ok && col < args.n_out) {
            float* dst = out + (size_t)row * args.ld_out + col;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (col + i < args.n_out) {
                const float bv = args.bias ? __ldg(args.bias + col + i) : 0.f;
                dst[i] = args.bias ? __uint_as_float(a[i]) + bv : __uint_as_float(a[i]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) record_error(args.err, MOE_ERR_TIMEOUT, 10);
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
  pdl_leave(args.pdl);
}

// ============================================================== large-batch kernel, CTA pairs
// Expert GEMMs for large batches on pairs of SMs (tcgen05 cta_group::2).  A
// 2-CTA cluster owns a 256-row x 256-column output tile; each CTA loads its
// own 128 activation rows and 128 of the 256 weight rows (GEMM1: the leader
// the gate rows, the peer the up rows), so a K-stage costs each CTA 32 KB of
// operand traffic instead of 48 KB for the same MMA work per SM.  The leader's
// single MMA thread issues M=256 x N=256 MMAs that read both CTAs' shared
// memory and write 128 rows x 256 columns into each CTA's TMEM.
//   full[s]   (leader only) armed by the leader with both CTAs' bytes; the
//             peer's TMA loads complete on it through the cluster address
//   empty[s]  (both) freed by the leader's multicast commit
//   tfull[a]  (both) accumulator ready, multicast commit
//   tempty[a] (leader only) 128 + 128 epilogue arrivals, the peer's remote
// Work lists give every expert an even number of 128-row tiles, so tile pair
// p = (2p, 2p+1) stays inside one expert.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* tm,
                                                 uint32_t leader_bar, int c0, int c1,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(leader_bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_ss_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with E4M3 A and B (K = 32 per instruction).
__device__ __forceinline__ void umma_e4m3_ss_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on the barrier at this offset in every CTA of `mask` when all
// tcgen05.mma issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Arrives on the barrier at the same offset in CTA `cta` of the cluster.  The
// default (CTA-scope) release is enough for its one use, the accumulator-free
// signal: the TMEM loads it guards have completed (tcgen05.wait::ld) before it,
// and the MMA issuer reads nothing else this thread wrote.  A cluster-scope
// release would also wait for the epilogue's global stores of the tile.
__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar, uint32_t cta) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
      "r"(cta)
      : "memory");
}

template <int EPI>
struct PairCfg {
  // GEMM2's staging tile costs it a K-stage: at 214 KB of shared memory the
  // pair GEMM2 measured 13 us slower than at 182 KB (same-box A/B, prefill).
  static constexpr int kStages = EPI == kEpiStore ? 5 : 6;
  static constexpr int kABytes = 128 * kGemmBK * 2;  // this CTA's 128 activation rows
  static constexpr int kBBytes = 128 * kGemmBK * 2;  // this CTA's 128 weight rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 512;  // two 128 x 256 fp32 accumulators
  // Epilogue warps: two per 32-lane TMEM quarter, each taking half of the
  // tile's columns, so that draining an accumulator keeps pace with the
  // MMAs of the next tile (short-K GEMM2 tiles especially).
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  // Per epilogue warp: 32 rows x 128 bytes of output staged for full-line
  // stores (the plain-store epilogue only).
  static constexpr int kOutStageBytes = EPI == kEpiStore ? kEpiWarps * 32 * 128 : 0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kOutStageBytes + 1024 + 256;
};

// F8: A (token rows) and B (weight rows) are E4M3 codes; a stage's 128-byte
// rows then hold 128 K elements (kind::f8f6f4 MMAs), and the epilogue
// multiplies each accumulator by args.a_scale[row] * args.b_scale[weight row].
template <int EPI, bool F8 = false>
__global__ void __launch_bounds__(PairCfg<EPI>::kThreads, 1) k_grouped_gemm_2sm(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const GemmArgs args) {
  using C = PairCfg<EPI>;
  constexpr int S = C::kStages;
  constexpr int kKb = F8 ? 128 : kGemmBK;  // K elements per stage
  constexpr int BN = 256;
  constexpr bool SWIGLU = (EPI == kEpiSwiGLU);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint4* out_stage = reinterpret_cast<uint4*>(smem + S * C::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kOutStageBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(&full[s2], 1);
      mbar_init(&empty[s2], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * C::kEpiWarps);  // every epilogue thread of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer signals the leader's barriers only after both are set up
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_enter(args.pdl);  // the work lists and operands come from earlier kernels

  const int num_pairs = tile_ld(args.tile_count) / 2;
  const int n_tiles = args.n_tiles;
  const int total = num_pairs * n_tiles;
  const int nk = (args.K + kKb - 1) / kKb;  // F8: a partial last block reads zeros past K
  const int* tl = args.tile_rows;
  const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      const uint64_t pol = policy_evict_normal();
      int fills[S];
#pragma unroll
      for (int s2 = 0; s2 < S; ++s2) fills[s2] = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int w = cluster_id; w < total && ok; w += num_clusters) {
        int mp, nt;
        raster(w, n_tiles, num_pairs, mp, nt);
        const int row0 = tile_ld(tl + 3 * (2 * mp) + 0);
        const int e = tile_ld(tl + 3 * (2 * mp) + 2);
        const int a_row = row0 + (int)rank * 128;
        const int b_row = SWIGLU ? e * args.b_rows_per_expert + nt * 128 + (int)rank * args.up_offset
                                 : e * args.b_rows_per_expert + nt * BN + (int)rank * 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + stage * C::kStageBytes;
          uint8_t* b_dst = a_dst + C::kABytes;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
          const uint32_t lbar = smem_u32(&full[stage]) & 0xFEFFFFFFu;  // the leader's barrier
          tma_load_2d_pair(a_dst, &tmA, lbar, kb * kKb, a_row, pol);
          tma_load_2d_pair(b_dst, &tmB, lbar, kb * kKb, b_row, pol);
          ++fills[stage];
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag && leader) {
#pragma unroll
        for (int s2 = 0; s2 < S; ++s2)
          if (fills[s2] > 0) mbar_wait_limit(&full[s2], (uint32_t)((fills[s2] - 1) & 1), 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader)
      constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(256, BN) : idesc_bf16_f32(256, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int w = cluster_id; w < total && ok; w += num_clusters, ++it) {
        const int ab = it & 1;
        const uint32_t aph = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait_bounded(&tempty[ab], aph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(ab * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b_addr = a_addr + C::kABytes;
          // four MMAs per stage: K = 16 bf16 or 32 E4M3 elements, 32 bytes each
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (F8)
              umma_e4m3_ss_pair(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                                sw128_kmajor_desc(b_addr + kk * 32), idesc,
                                (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16_ss_pair(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                                sw128_kmajor_desc(b_addr + kk * 32), idesc,
                                (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty[stage], 0x3);  // frees this stage in both CTAs
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit_pair_mc(&tfull[ab], 0x3);
      }
      if (*abort_flag) {
        umma_commit_pair(drain);
        mbar_wait_limit(drain, 0, 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2.., both CTAs)
    // Each warp owns TMEM lanes q*32.. (32 output rows; a warp reaches the
    // lanes of its index mod 4) and half of the accumulator's columns (hc).
    // GEMM2: a 64-column slice is packed to bf16, written row by row into the
    // warp's staging tile (16-byte chunks XOR-swizzled by row: no bank
    // conflicts either way) and read back so that every store instruction
    // writes 4 full 128-byte rows instead of half sectors of 32 rows.
    static_assert(C::kEpiWarps == 4 || C::kEpiWarps == 8, "one or two warps per lane quarter");
    constexpr int kColParts = C::kEpiWarps / 4;
    const int q = warp & 3;
    const int hc = (warp - 2) >> 2;
    uint4* st_tile = out_stage + (size_t)(warp - 2) * 32 * 8;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
    int it = 0;
    for (int w = cluster_id; w < total; w += num_clusters, ++it) {
      int mp, nt;
      raster(w, n_tiles, num_pairs, mp, nt);
      const int row0 = tile_ld(tl + 3 * (2 * mp) + 0);
      const int rowend = tile_ld(tl + 3 * (2 * mp) + 1);
      // F8: first weight row of the tile (SwiGLU: of its gate half)
      const int wrow0 = F8 ? tile_ld(tl + 3 * (2 * mp) + 2) * args.b_rows_per_expert +
                                 nt * (SWIGLU ? BN / 2 : BN)
                           : 0;
      const int ab = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      const bool got = mbar_wait_bounded(&tfull[ab], aph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + (uint32_t)(ab * BN) + ((uint32_t)(q * 32) << 16);
      const int row_base = row0 + (int)rank * 128 + q * 32;
      // Stores the staged 32 x 64 slice at output column col0 (a multiple of
      // 64; n_out is one too, so a slice is wholly inside or outside).
      auto drain_slice = [&](int col0) {
        __syncwarp();
        if (col0 < args.n_out) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = i * 4 + (lane >> 3), v = lane & 7;
            const uint4 val = st_tile[r * 8 + (v ^ (r & 7))];
            if (row_base + r < rowend)
              *reinterpret_cast<uint4*>(out + (size_t)(row_base + r) * args.ld_out + col0 + v * 8) =
                  val;
          }
        }
        __syncwarp();
      };
      if (SWIGLU) {
        // h is half as wide as the accumulator; direct 16-byte stores measured
        // faster here than the staged path.
        constexpr int H = BN / 2;
        const int row = row_base + lane;
        const bool row_ok = row < rowend;
        const float sa = (F8 && row_ok) ? __ldg(args.a_scale + row) : 1.0f;
#pragma unroll 1
        for (int c = hc * (H / kColParts); c < (hc + 1) * (H / kColParts); c += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(t_addr + c, g);
          tmem_ld_32x32b_x32(t_addr + H + c, u);
          tmem_ld_wait();
          const int col = nt * H + c;
          if (row_ok && col < args.n_out) {
            if (F8) {  // gate rows wrow0 + c + i, up rows up_offset further
              const float* sg = args.b_scale + wrow0 + c;
              const float* su = sg + args.up_offset;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                g[i] = __float_as_uint(__uint_as_float(g[i]) * sa * __ldg(sg + i));
                u[i] = __float_as_uint(__uint_as_float(u[i]) * sa * __ldg(su + i));
              }
            }
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              p[i] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * args.ld_out + col);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          }
        }
      } else {
        const int row = row_base + lane;
        const float sa = (F8 && row < rowend) ? __ldg(args.a_scale + row) : 1.0f;
#pragma unroll 1
        for (int c = hc * (BN / kColParts); c < (hc + 1) * (BN / kColParts); c += 64) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t a[32];
            tmem_ld_32x32b_x32(t_addr + c + 32 * half, a);
            tmem_ld_wait();
            if (F8 && nt * BN + c + 32 * half < args.n_out) {
              const float* sb = args.b_scale + wrow0 + c + 32 * half;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                a[i] = __float_as_uint(__uint_as_float(a[i]) * sa * __ldg(sb + i));
            }
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              p[i] = pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int chunk = 4 * half + v;
              st_tile[lane * 8 + (chunk ^ (lane & 7))] =
                  make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
            }
          }
          drain_slice(nt * BN + c);
        }
      }
      tc_fence_before();
      if (leader) mbar_arrive(&tempty[ab]);
      else mbar_arrive_cta(&tempty[ab], 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs read this CTA's shared memory until here
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) record_error(args.err, MOE_ERR_TIMEOUT, 13);
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::kTmemCols)
                 : "memory");
}

// ============================================================== small-batch kernel
// Swap-AB form for batches of at most NMAX tokens per expert (decode): the
// expert's weights are the M = 128 operand (128 weight rows per work item:
// 64 gate + 64 up rows of Wg/Wu for GEMM1, 128 rows of Wd for GEMM2) and the
// expert's n token rows are the N operand, N = 16 * ceil(n / 16) chosen per
// item in the instruction descriptor.  Every K-stage then moves 16 KB of
// weights and only 2 KB per 16 tokens, instead of a 128-row activation tile
// that is mostly other experts' rows.  Work item = (touched expert, 128-row
// weight tile).  D[weight row][token] sits in TMEM lanes x columns; GEMM1's
// epilogue pairs gate lane j with up lane 64 + j through shared memory.
template <int NMAX, bool SWIGLU>
struct SwapCfg {
  // One stage below what fits: the smaller footprint (177 / 169 KB at
  // NMAX = 64) measured slightly faster in the whole decode graph (same-box
  // A/B: 121.1 -> 120.4 us at T = 64, 235 -> 231 us at T = 256).
  static constexpr int kStages = NMAX <= 64 ? 7 : NMAX <= 128 ? 5 : 4;
  static constexpr int kABytes = 128 * kGemmBK * 2;   // weights, 16 KB
  static constexpr int kBBytes = NMAX * kGemmBK * 2;  // tokens
  static constexpr int kStageBytes = kABytes + kBBytes;
  // Accumulator buffers in TMEM: the MMA runs up to kAccBufs - 1 items ahead
  // of the epilogue (all 512 columns at NMAX = 128; a CTA of the other GEMM
  // cannot share the SM, its shared memory does not fit beside this one's).
  // Same-box A/B against two buffers: W8A8 T = 256 165.8 -> 161 us, the rest
  // unchanged.
  static constexpr int kAccBufs = 4;
  static constexpr int kTmemCols = kAccBufs * NMAX;
  static constexpr int kXchBytes = SWIGLU ? 2 * 64 * 16 * 4 : 0;
  // This CTA's first kMaxItems work items (row0, rows, expert, column tile),
  // read from the list once: a per-item L2 read in the producer and the MMA
  // loop stalls both at every item boundary.
  static constexpr int kMaxItems = 128;
  static constexpr int kItemBytes = 16 * kMaxItems;
  static constexpr int kSmemBytes = kStages * kStageBytes + kXchBytes + 1024 + 256 + kItemBytes;
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Work items come from a list of (row0, row_end, expert) entries: the
// touched-expert list (every item holds all of an expert's rows), or with
// row_tiles the 128-row tile list, whose entry i covers rows
// [row0, min(row_end, row0 + 128)).  An item with more than NMAX rows (only
// caller offsets that give one expert more rows than the batch has tokens
// make one) runs as several passes of at most NMAX rows, each streaming the
// item's weights again.
//
// early_w != 0 (an early launch): the producer issues the weight half of its
// first S stages before waiting for the previous kernel, and the token half
// after.  The caller guarantees that the work list is complete once this
// kernel may launch: the previous kernel lets its dependents launch only
// after its own wait, and the list comes from a kernel before it.  Every
// thread of this kernel likewise lets the next kernel launch only after its
// own wait, so the next expert GEMM may be an early launch.
//
// ready != nullptr: the GEMM1 / GEMM2 pair synchronises per work-list entry
// instead of per kernel.  GEMM1 (SWIGLU) adds 1 to ready[i] once it has
// stored an item's columns of entry i's rows; GEMM2 never waits for GEMM1 as
// a whole: before streaming an item of entry i it waits (bounded) until
// ready[i] == ready_target (GEMM1's column tiles), so GEMM2 CTAs on SMs that
// GEMM1's tail frees start at once.  GEMM2 waits for the previous kernel only
// at its end, so its completion still implies GEMM1's.
//
// A counted GEMM2 with ready_count > 0 takes its items from a queue
// (ready[ready_count], an int after the counters, zeroed with them) instead
// of every gridDim.x-th item:
// the producer claims item w with atomicAdd, in order, and passes (row0,
// rows, expert, w) to the MMA and epilogue warps through a ring of 8
// records with full / empty barriers; a record with rows < 0 ends the work.
// Its CTAs start as GEMM1's tail frees SMs, so the early ones take more items.
//
// F8: both operands are E4M3 codes (kind::f8f6f4 MMAs; a stage's 128-byte
// rows then hold 128 K elements), w_scale holds one fp32 scale per weight row
// (the TMA row index) and x_scale one per token row, and the epilogue
// multiplies each accumulator by its two scales.
template <int NMAX, bool SWIGLU, bool F8>
__global__ void __launch_bounds__(192, 1) k_expert_gemm_swap(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
    const int* __restrict__ list_count, const int* __restrict__ list, int row_tiles,
    int n_tiles, int K, int w_rows_per_expert,
    int up_offset, int n_out, __nv_bfloat16* __restrict__ out, int ld_out,
    int* __restrict__ err, int early_w, const float* __restrict__ w_scale,
    const float* __restrict__ x_scale, int* __restrict__ ready, int ready_target,
    int ready_count, const int* __restrict__ tok_row, int n_tok) {
  using C = SwapCfg<NMAX, SWIGLU>;
  constexpr int kKb = F8 ? 128 : kGemmBK;  // K elements per stage (128-byte rows)
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* xch = reinterpret_cast<float*>(smem + S * C::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kXchBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + C::kAccBufs;
  uint64_t* drain = tempty + C::kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* n_items_s = const_cast<int*>(abort_flag) + 1;
  int4* items_s = reinterpret_cast<int4*>(smem + S * C::kStageBytes + C::kXchBytes + 256);
  // dynamic items: the first 8 table slots are the ring, its barriers follow
  constexpr int kRing = 8;
  uint64_t* ifull = reinterpret_cast<uint64_t*>(items_s + kRing);
  uint64_t* iempty = ifull + kRing;
  const bool counted = !SWIGLU && ready != nullptr;  // GEMM2 of a counted pair
  // Direct tokens (GEMM1, at most 64 tokens): the token operand of every item
  // is all n_tok rows of the unpermuted x (one N <= 64 tile), and the
  // epilogue stores column t (token t) to the h row r of the item's entry
  // with tok_row[r] == t; the dispatch gather is not needed.
  const bool direct = SWIGLU && NMAX == 64 && tok_row != nullptr;
  const bool dyn = counted && ready_count > 0;       // ... taking items from the queue

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(&full[s2], 1);
      mbar_init(&empty[s2], 1);
    }
    for (int a = 0; a < C::kAccBufs; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    if (dyn) {
      for (int r = 0; r < kRing; ++r) {
        mbar_init(&ifull[r], 1);
        mbar_init(&iempty[r], 1);
      }
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Warp 0 (the producer's) of an early launch reads the work list before its
  // wait; every other thread waits here.
  const bool early = early_w != 0 && threadIdx.x == 0;  // the producer thread
  if (counted) {
    pdl_trigger();
  } else if (!(early_w != 0 && warp == 0)) {
    pdl_wait();  // the operands come from the previous kernels
    pdl_trigger();
  }
  const int nk = (K + kKb - 1) / kKb;  // a partial last block reads zeros past K
  // Work item w: (row0, rows, expert, w) of list entry w / n_tiles, column
  // tile w % n_tiles; a row tile holds at most 128 rows of its expert.  The
  // list is read around L1 (an early producer reads it before its wait).
  auto load_w = [&](int w) -> int4 {
    const int i = w / n_tiles;
    const int row0 = __ldcg(list + 3 * i + 0);
    const int r = __ldcg(list + 3 * i + 1) - row0;
    return make_int4(row0, row_tiles ? min(r, kGemmBM) : r, __ldcg(list + 3 * i + 2), w);
  };
  // Static items: this CTA's j-th is w = blockIdx.x + j * gridDim.x.
  auto load_item = [&](int j) -> int4 { return load_w(blockIdx.x + j * gridDim.x); };
  // Warp 0 fills the table, then arrives (without waiting) on named barrier 3,
  // which the other warps wait on.
  if (dyn) {
    if (warp != 0) named_bar_sync(3, 192);
    else asm volatile("bar.arrive 3, 192;" ::: "memory");
  } else if (warp == 0) {
    const int total = __ldcg(list_count) * n_tiles;
    const int my = total > (int)blockIdx.x ? (total - (int)blockIdx.x - 1) / (int)gridDim.x + 1
                                           : 0;
    for (int j = lane; j < min(my, C::kMaxItems); j += 32) items_s[j] = load_item(j);
    if (lane == 0) *n_items_s = my;
    __syncwarp();
    asm volatile("bar.arrive 3, 192;" ::: "memory");
    if (early_w != 0 && lane != 0) {
      pdl_wait();
      pdl_trigger();
    }
  } else {
    named_bar_sync(3, 192);
  }
  const int my_items = dyn ? 0 : *n_items_s;
  auto item = [&](int j) -> int4 { return j < C::kMaxItems ? items_s[j] : load_item(j); };
  // Item j of the MMA and epilogue warps: the table's, or (counted) the ring's
  // record; false at the end of the work.
  auto fetch = [&](int j, int4& itm) -> bool {
    if (!dyn) {
      if (j >= my_items) return false;
      itm = item(j);
      return true;
    }
    if (!mbar_wait_bounded(&ifull[j & (kRing - 1)], (uint32_t)((j / kRing) & 1), abort_flag))
      return false;
    itm = items_s[j & (kRing - 1)];
    return itm.y >= 0;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int fills[S];
#pragma unroll
      for (int s2 = 0; s2 < S; ++s2) fills[s2] = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // token tiles of stage s: expect their bytes, arrive, load them
      auto load_tokens = [&](int s2, int kb, int row0, int nb) {
        uint8_t* b_dst = smem + s2 * C::kStageBytes + C::kABytes;
        mbar_arrive_expect_tx(&full[s2], (uint32_t)(nb * 16 * 128));
        for (int b = 0; b < nb; ++b)
          tma_load_2d(b_dst + b * 16 * 128, &tmX, &full[s2], kb * kKb, row0 + 16 * b, pol_x);
      };
      // Token tiles that cannot be read yet are deferred: an early launch's
      // first S stages (until the previous kernel completes) and, in a
      // counted GEMM2, the stages of an item whose entry GEMM1 has not
      // finished.  A deferred stage gets its weights at once and its tokens
      // (with the stage's single arrival) when released, so its barrier
      // cannot complete before; at most S stages, of one item, are deferred.
      int deferred = 0;
      bool waited = !early;  // the previous kernel is complete (or need not be)
      int d_stage[S], d_kb[S], d_row0[S], d_nb[S];
      auto release_deferred = [&](const int* counter) -> bool {
        if (!waited) {
          pdl_wait();
          pdl_trigger();
          waited = true;
        }
        if (counter != nullptr) {  // entry's rows of h complete, then read by TMA
          if (!wait_count_bounded(counter, ready_target, abort_flag)) return false;
          fence_proxy_async_global();
        }
        for (int q = 0; q < deferred; ++q) load_tokens(d_stage[q], d_kb[q], d_row0[q], d_nb[q]);
        deferred = 0;
        return true;
      };
      // counted GEMM2: claim the next item, publish it to the ring
      const int total = dyn ? __ldcg(list_count) * n_tiles : 0;
      auto claim = [&](int j, int4& itm) -> bool {
        const int slot = j & (kRing - 1);
        if (j >= kRing &&
            !mbar_wait_bounded(&iempty[slot], (uint32_t)(((j / kRing) - 1) & 1), abort_flag))
          return false;
        const int w = atomicAdd(ready + ready_count, 1);
        itm = w < total ? load_w(w) : make_int4(0, -1, 0, 0);
        items_s[slot] = itm;
        mbar_arrive(&ifull[slot]);
        return itm.y >= 0;
      };
      for (int j = 0; ok; ++j) {
        int4 itm;
        if (dyn) {
          if (!claim(j, itm)) break;
        } else {
          if (j >= my_items) break;
          itm = item(j);
        }
        const int n = itm.y;
        const int wrow = itm.z * w_rows_per_expert + (itm.w % n_tiles) * (SWIGLU ? 64 : 128);
        // counted GEMM2: this item's entry counter, or nullptr once it is complete
        const int* pending = nullptr;
        if (counted && n > 0) {
          const int* c = ready + itm.w / n_tiles;
          int v;
          asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
          if (v >= ready_target)
            fence_proxy_async_global();
          else
            pending = c;
        }
        for (int p0 = 0; p0 < n && ok; p0 += NMAX) {  // n < 1: recorded by the epilogue
          const int row0 = direct ? 0 : itm.x + p0;
          const int nb = direct ? (n_tok + 15) >> 4 : (min(n - p0, NMAX) + 15) >> 4;
          for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* a_dst = smem + stage * C::kStageBytes;
            const bool now = waited && pending == nullptr;
            // One arrival per stage, with every byte of the stage expected by
            // then: the whole stage at once, or (deferred) the weights now and
            // the tokens with the arrival.
            if (now) {
              mbar_arrive_expect_tx(&full[stage], (uint32_t)(C::kABytes + nb * 16 * 128));
            } else {
              mbar_expect_tx(&full[stage], (uint32_t)C::kABytes);
            }
            if (SWIGLU) {
              tma_load_2d(a_dst, &tmW, &full[stage], kb * kKb, wrow, pol_w);
              tma_load_2d(a_dst + 64 * 128, &tmW, &full[stage], kb * kKb, wrow + up_offset,
                          pol_w);
            } else {
              tma_load_2d(a_dst, &tmW, &full[stage], kb * kKb, wrow, pol_w);
            }
            if (now) {
              for (int b = 0; b < nb; ++b)
                tma_load_2d(a_dst + C::kABytes + b * 16 * 128, &tmX, &full[stage], kb * kKb,
                            row0 + 16 * b, pol_x);
            } else {
              d_stage[deferred] = stage;
              d_kb[deferred] = kb;
              d_row0[deferred] = row0;
              d_nb[deferred] = nb;
              if (++deferred == S) {  // the ring is full of deferred stages
                ok = release_deferred(pending);
                pending = nullptr;
              }
            }
            ++fills[stage];
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
            if (!ok) break;
          }
        }
        // an item's deferred stages are released before the next item begins
        if (ok && pending != nullptr) ok = release_deferred(pending);
      }
      if (ok && (!waited || deferred > 0)) ok = release_deferred(nullptr);  // few stages, or none
      if (*abort_flag) {
#pragma unroll
        for (int s2 = 0; s2 < S; ++s2)
          if (fills[s2] > 0)
            mbar_wait_limit(&full[s2], (uint32_t)((fills[s2] - 1) & 1), 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        int4 itm;
        if (!fetch(j, itm)) break;
        const int n = itm.y;
        // one accumulator buffer per pass (an empty item has none; the same in the epilogue)
        for (int p0 = 0; p0 < n && ok; p0 += NMAX, ++it) {
          const int ncol = (((direct ? n_tok : min(n - p0, NMAX)) + 15) >> 4) * 16;
          const uint32_t idesc = F8 ? idesc_e4m3_f32(128, ncol) : idesc_bf16_f32(128, ncol);
          const int ab = it % C::kAccBufs;
          const uint32_t aph = (uint32_t)((it / C::kAccBufs) & 1);
          if (!mbar_wait_bounded(&tempty[ab], aph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(ab * NMAX);
          for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
            const uint32_t b_addr = a_addr + C::kABytes;
            // four MMAs per stage: K = 16 bf16 or 32 E4M3 elements, 32 bytes each
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (F8)
                umma_e4m3_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                             sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
              else
                umma_bf16_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                             sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) umma_commit(&tfull[ab]);
        }
      }
      if (*abort_flag) {
        umma_commit(drain);
        mbar_wait_limit(drain, 0, 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lanes q*32 .. q*32+31 = weight rows
    int it = 0;
    int chunk_parity = 0;
    bool stop = false;
    for (int j = 0; !stop; ++j) {
      int4 itm;
      if (!fetch(j, itm)) break;
      const int n_item = itm.y, nt = itm.w % n_tiles;
      if (n_item < 1 && threadIdx.x == 64) record_error(err, MOE_ERR_DEVICE_CHECK, 12);
      for (int p0 = 0; p0 < n_item; p0 += NMAX, ++it) {
        const int row0 = itm.x + p0;
        const int n = min(n_item - p0, NMAX);
        const int ncols = (((direct ? n_tok : n) + 15) >> 4) * 16;
        const int ab = it % C::kAccBufs;
        const uint32_t aph = (uint32_t)((it / C::kAccBufs) & 1);
        // F8: the item's token scales, lane l holding those of columns l,
        // l + 32, ... (one parallel load per lane instead of one dependent load
        // per column).  A counted GEMM2's scales come from a kernel that may
        // still run: read through L2 once the item's accumulator is complete
        // (its producer waited for the entry); otherwise before the wait.
        float xsr[F8 ? (NMAX + 31) / 32 : 1];
        auto load_scales = [&]() {
#pragma unroll
          for (int i = 0; i < (F8 ? (NMAX + 31) / 32 : 1); ++i) {
            const float* p = x_scale + row0 + lane + 32 * i;
            xsr[i] = (F8 && lane + 32 * i < n) ? (counted ? __ldcg(p) : __ldg(p)) : 0.0f;
          }
        };
        if (!counted) load_scales();
        mbar_wait_bounded(&tfull[ab], aph, abort_flag);
        // The four epilogue warps decide together whether to go on, so none is
        // left waiting at the exchange barrier below.
        named_bar_sync(2, 128);
        if (*abort_flag) {
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t t_addr = tmem_base + (uint32_t)(ab * NMAX) + ((uint32_t)(q * 32) << 16);
        // first weight row of the item (the TMA row index; the F8 scales' index)
        const int wrow0 = itm.z * w_rows_per_expert + nt * (SWIGLU ? 64 : 128);
        if (counted) load_scales();
        // token c0 + cc's scale for the 16 columns from c0 (warp-wide shuffles)
        auto chunk_scales = [&](int c0, float* xv) {
          if (!F8) return;
          float xsel = xsr[0];
#pragma unroll
          for (int i = 1; i < (F8 ? (NMAX + 31) / 32 : 1); ++i)
            if ((c0 >> 5) == i) xsel = xsr[i];
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) xv[cc] = __shfl_sync(0xffffffffu, xsel, (c0 + cc) & 31);
        };
        // accumulator of token column c times its scales (F8), else as is
        auto scaled = [&](uint32_t bits, float sw, int c, float xc) {
          const float a = __uint_as_float(bits);
          if (!F8) return a;
          return c < n ? a * sw * xc : 0.0f;
        };
        if (SWIGLU) {
          // lanes 0..63: gate rows j, lanes 64..127: up rows j (j = lane & 63)
          const int j = (q & 1) * 32 + lane;
          const int col = nt * 64 + j;
          const float sw = F8 ? __ldg(w_scale + wrow0 + (q >= 2 ? up_offset : 0) + j) : 1.0f;
          // h row of accumulator column c: row0 + c for c < n, or (direct)
          // the entry row holding token c (lane l keeps columns l and l + 32),
          // -1 for a column with no row
          int map0 = -1, map1 = -1;
          if (direct) {
            const int pv0 = lane < n ? __ldg(tok_row + row0 + lane) : -1;
            const int pv1 = lane + 32 < n ? __ldg(tok_row + row0 + lane + 32) : -1;
            for (int i = 0; i < n; ++i) {
              const int t = __shfl_sync(0xffffffffu, i < 32 ? pv0 : pv1, i & 31);
              if (t == lane) map0 = row0 + i;
              if (t == lane + 32) map1 = row0 + i;
            }
          }
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            float* x = xch + chunk_parity * (64 * 16);
            uint32_t v[16];
            float xv[16];
            int rr[16];
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const int c = c0 + cc;
              rr[cc] = direct ? __shfl_sync(0xffffffffu, c < 32 ? map0 : map1, c & 31)
                              : (c < n ? row0 + c : -1);
            }
            chunk_scales(c0, xv);
            tmem_ld_32x32b_x16(t_addr + c0, v);
            tmem_ld_wait();
            if (q >= 2) {
#pragma unroll
              for (int cc = 0; cc < 16; ++cc) x[cc * 64 + j] = scaled(v[cc], sw, c0 + cc, xv[cc]);
            }
            named_bar_sync(1, 128);
            if (q < 2 && col < n_out) {
#pragma unroll
              for (int cc = 0; cc < 16; ++cc) {
                const int c = c0 + cc;
                if (rr[cc] >= 0) {
                  const float g = scaled(v[cc], sw, c, xv[cc]);
                  const float u = x[cc * 64 + j];
                  out[(size_t)rr[cc] * ld_out + col] = __float2bfloat16_rn(silu_f(g) * u);
                }
              }
            }
            chunk_parity ^= 1;
          }
        } else {
          const int col = nt * 128 + q * 32 + lane;
          const float sw = (F8 && col < n_out) ? __ldg(w_scale + wrow0 + q * 32 + lane) : 1.0f;
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            uint32_t v[16];
            float xv[16];
            chunk_scales(c0, xv);
            tmem_ld_32x32b_x16(t_addr + c0, v);
            tmem_ld_wait();
            if (col < n_out) {
#pragma unroll
              for (int cc = 0; cc < 16; ++cc) {
                const int c = c0 + cc;
                if (c < n)
                  out[(size_t)(row0 + c) * ld_out + col] =
                      __float2bfloat16_rn(scaled(v[cc], sw, c, xv[cc]));
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[ab]);
      }
      if (SWIGLU && ready != nullptr && !stop) {
        // every epilogue thread's stores of this item, then one release add
        fence_proxy_async_global();
        named_bar_sync(4, 128);
        if (threadIdx.x == 64) {
          __threadfence();
          atomicAdd(ready + itm.w / n_tiles, 1);
        }
      }
      if (dyn && threadIdx.x == 64) mbar_arrive(&iempty[j & (kRing - 1)]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) record_error(err, MOE_ERR_TIMEOUT, 11);
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
  if (counted) pdl_wait();  // completion implies the previous kernel's
}

// ============================================================== host side
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                    void*, const cuuint64_t*, const cuuint64_t*,
                                    const cuuint32_t*, const cuuint32_t*,
                                    CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix; box = 64 columns
// (128 bytes, the swizzle span) x box_rows rows, 128-byte swizzle.
static bool make_tmap(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kGemmBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint8 tensor map (E4M3 codes) over a row-major [rows, cols] byte
// matrix; box = 128 columns (128 bytes, the swizzle span) x box_rows rows.
static bool make_tmap_u8(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int EPI>
static cudaError_t launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb,
                                 const GemmArgs& args, int max_work, int num_sms,
                                 cudaStream_t st) {
  using C = GemmCfg<BN, EPI>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<BN, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int grid = max_work < num_sms ? max_work : num_sms;
  if (grid < 1) grid = 1;
  return launch_kernel(k_grouped_gemm<BN, EPI>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, st,
                       1, ta, tb, args);
}

template <int NMAX, bool SWIGLU, bool F8 = false>
static cudaError_t launch_swap_t(const CUtensorMap& tw, const CUtensorMap& tx,
                                 const int* list_count, const int* list, int row_tiles,
                                 int max_work, int n_tiles, int K,
                                 int w_rows, int up_off, int n_out, __nv_bfloat16* out,
                                 int ld_out, int* err, int early, int num_sms,
                                 cudaStream_t st, const float* w_scale = nullptr,
                                 const float* x_scale = nullptr, int* ready = nullptr,
                                 int ready_target = 0, int ready_count = 0,
                                 const int* tok_row = nullptr, int n_tok = 0) {
  using C = SwapCfg<NMAX, SWIGLU>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_expert_gemm_swap<NMAX, SWIGLU, F8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int grid = max_work < num_sms ? max_work : num_sms;
  if (grid < 1) grid = 1;
  return launch_kernel(k_expert_gemm_swap<NMAX, SWIGLU, F8>, dim3(grid), dim3(192),
                       C::kSmemBytes, st, 1, tw, tx, list_count, list, row_tiles, n_tiles, K,
                       w_rows, up_off, n_out, out, ld_out, err, early, w_scale, x_scale, ready,
                       ready_target, ready_count, tok_row, n_tok);
}

// Small batches (T <= 256): both GEMMs in swap-AB form.  GEMM2 waits for
// GEMM1 per work-list entry (ready counters), so its CTAs start as GEMM1's
// tail frees SMs; GEMM1 is an early launch when the caller says so.
static int launch_expert_ffn_swap(const __nv_bfloat16* x_perm, long long x_rows,
                                  const __nv_bfloat16* w13, const __nv_bfloat16* w2,
                                  const moe_shape& s, const WsLayout& L, char* ws,
                                  __nv_bfloat16* z, int num_sms, cudaStream_t st,
                                  void* const* events, bool early1, const int* tok_row) {
  const int e1 = early1 ? 1 : 0;
  auto mark = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st,
                                    cudaEventRecordExternal);
  };
  int* err = reinterpret_cast<int*>(ws + L.err);
  const int* tiles = reinterpret_cast<const int*>(ws + L.tiles);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  CUtensorMap tW1, tX1, tW2, tX2;
  if (!make_tmap(&tW1, w13, (uint64_t)s.E * 2 * s.f, (uint64_t)s.d, 64) ||
      !make_tmap(&tX1, x_perm, (uint64_t)x_rows, (uint64_t)s.d, 16) ||
      !make_tmap(&tW2, w2, (uint64_t)s.E * s.d, (uint64_t)s.f, 128) ||
      !make_tmap(&tX2, h, (uint64_t)L.Ppad, (uint64_t)s.f, 16))
    return MOE_ERR_CUDA;
  const int nt1 = s.f / 64;               // 64 gate + 64 up rows per item
  const int nt2 = (s.d + 127) / 128;      // 128 output columns per item
  const int E = s.E;
  // GEMM2 starts each list entry once GEMM1 has stored all nt1 column tiles of
  // it, taking its items from the queue after the counters unless at most one
  // wave of items can exist (then every CTA has one item at most anyway)
  int* ready = ready_counters(const_cast<int*>(tiles), L.max_mtiles, E);
  const long long max_items2 =
      s.T <= 64 ? (long long)std::min<long long>(E, (long long)s.T * s.k) * nt2
                : (long long)L.max_mtiles * nt2;
  const int rq = max_items2 <= num_sms ? 0 : L.max_mtiles + E;
  cudaError_t e;
  if (s.T <= 64) {
    // one item per touched expert (at most 64 rows)
    const int* cnt = tiles + 1;
    const int* ents = expert_entries(const_cast<int*>(tiles));
    // tok_row: x_perm is the unpermuted x (T rows) and GEMM1 maps its rows
    // itself; the work list then comes from the kernel just before, so no
    // early start
    e = launch_swap_t<64, true>(tW1, tX1, cnt, ents, 0, E * nt1, nt1, s.d, 2 * s.f, s.f, s.f, h,
                                s.f, err, tok_row ? 0 : e1, num_sms, st, nullptr, nullptr, ready,
                                0, 0, tok_row, s.T);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_swap_t<64, false>(tW2, tX2, cnt, ents, 0, E * nt2, nt2, s.f, s.d, 0, s.d, z,
                                   s.d, err, 0, num_sms, st, nullptr, nullptr, ready, nt1, rq);
  } else {
    // one item per 128-row tile: 5 K-stages of weights in flight instead of
    // the 4 that 256-row items leave room for
    const int* cnt = tiles;
    const int* ents = row_tile_entries(const_cast<int*>(tiles), E);
    e = launch_swap_t<128, true>(tW1, tX1, cnt, ents, 1, L.max_mtiles * nt1, nt1, s.d, 2 * s.f,
                                 s.f, s.f, h, s.f, err, e1, num_sms, st, nullptr, nullptr, ready);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_swap_t<128, false>(tW2, tX2, cnt, ents, 1, L.max_mtiles * nt2, nt2, s.f, s.d,
                                    0, s.d, z, s.d, err, 0, num_sms, st, nullptr, nullptr, ready,
                                    nt1, rq);
  }
  if (e == cudaSuccess) e = mark(1);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int EPI, bool F8 = false>
static cudaError_t launch_gemm_2sm(const CUtensorMap& ta, const CUtensorMap& tb,
                                   const GemmArgs& args, int max_pairs_work, int num_sms,
                                   cudaStream_t st) {
  using C = PairCfg<EPI>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm_2sm<EPI, F8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int clusters = max_pairs_work < num_sms / 2 ? max_pairs_work : num_sms / 2;
  if (clusters < 1) clusters = 1;
  return launch_kernel(k_grouped_gemm_2sm<EPI, F8>, dim3(2 * clusters), dim3(C::kThreads),
                       C::kSmemBytes, st, 2, ta, tb, args);
}

// The W8A8 expert GEMMs in the swap-AB form over the touched-expert list
// (NMAX = 64: T <= 64) or the 128-row tile list (NMAX = 128).  overlap: GEMM1
// counts each entry's stored column tiles (first counter array), the entry
// quantiser waits for complete entries and counts them (second array), and
// GEMM2 waits per entry, taking its items from the second array's queue when
// they can exceed one wave.  Otherwise the row quantiser runs between the
// GEMMs and GEMM2 is an early launch.  mark(0) after GEMM1.
template <int NMAX, typename Mark>
static cudaError_t swap_ffn_w8a8(const CUtensorMap& tW1, const CUtensorMap& tX1,
                                 const CUtensorMap& tW2, const CUtensorMap& tX2,
                                 const moe_shape& s, const WsLayout& L, const int* tiles,
                                 __nv_bfloat16* h, uint8_t* hq, float* hs, const float* xs,
                                 const float* w13_scale, const float* w2_scale,
                                 __nv_bfloat16* z, int* err, int e1, bool overlap, int num_sms,
                                 cudaStream_t st, Mark&& mark) {
  const int nt1 = s.f / 64, nt2 = (s.d + 127) / 128, E = s.E;
  const bool experts = NMAX == 64;  // one entry per touched expert
  const int* cnt = experts ? tiles + 1 : tiles;
  const int* ents = experts ? expert_entries(const_cast<int*>(tiles))
                            : row_tile_entries(const_cast<int*>(tiles), E);
  const int row_tiles = experts ? 0 : 1;
  const int max_entries = experts ? E : L.max_mtiles;
  int* ready1 = overlap ? ready_counters(const_cast<int*>(tiles), L.max_mtiles, E) : nullptr;
  const int rq_at = L.max_mtiles + E;  // each counter array's queue, after its counters
  int* ready2 = overlap ? ready1 + rq_at + 1 : nullptr;
  cudaError_t e = launch_swap_t<NMAX, true, true>(
      tW1, tX1, cnt, ents, row_tiles, max_entries * nt1, nt1, s.d, 2 * s.f, s.f, s.f, h, s.f,
      err, e1, num_sms, st, w13_scale, xs, ready1);
  if (e == cudaSuccess) e = mark(0);
  if (!overlap) {
    if (e == cudaSuccess) e = launch_quant_rows(h, nullptr, L.P, 0, s.f, hq, hs, err, st);
    if (e == cudaSuccess)
      e = launch_swap_t<NMAX, false, true>(tW2, tX2, cnt, ents, row_tiles, max_entries * nt2,
                                           nt2, s.f, s.d, 0, s.d, z, s.d, err, 1, num_sms, st,
                                           w2_scale, hs);
    return e;
  }
  if (e == cudaSuccess)
    e = launch_quant_entries(h, s.f, cnt, ents, row_tiles, max_entries, ready1, nt1, ready2, hq,
                             hs, err, st);
  const long long max_items2 =
      (experts ? std::min<long long>(E, (long long)s.T * s.k) : (long long)L.max_mtiles) * nt2;
  if (e == cudaSuccess)
    e = launch_swap_t<NMAX, false, true>(tW2, tX2, cnt, ents, row_tiles, max_entries * nt2, nt2,
                                         s.f, s.d, 0, s.d, z, s.d, err, 0, num_sms, st, w2_scale,
                                         hs, ready2, 1, max_items2 <= num_sms ? 0 : rq_at);
  return e;
}

// Both GEMMs with E4M3 operands on both sides, at every batch size, and
// between them the SwiGLU output quantised: the swap-AB kernels over the
// touched-expert list (T <= 64) or the 128-row tile list (swap_ffn_w8a8: the
// quantisation per list entry beside GEMM1 when the entries are small or
// many, else row by row between the GEMMs with GEMM2 an early launch); for
// large dense batches (the CTA-pair tile layout, pair_tiles) the CTA-pair
// kernels over the tile pairs, with the lone-tile experts' leftover list on
// the swap-AB kernels (their tokens fit one 128-row item) and the row
// quantiser between the GEMMs.
int launch_expert_ffn_w8a8(const uint8_t* xq, const float* xs, long long x_rows,
                           const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                           const float* w2_scale, const moe_shape& s, const WsLayout& L,
                           char* ws, __nv_bfloat16* z, int num_sms, cudaStream_t st,
                           void* const* events, bool early_gemm1) {
  auto mark = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st,
                                    cudaEventRecordExternal);
  };
  int* err = reinterpret_cast<int*>(ws + L.err);
  const int* tiles = reinterpret_cast<const int*>(ws + L.tiles);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  uint8_t* hq = reinterpret_cast<uint8_t*>(ws + L.hq);
  float* hs = reinterpret_cast<float*>(ws + L.hs);
  CUtensorMap tW1, tX1, tW2, tX2;
  if (!make_tmap_u8(&tW1, w13, (uint64_t)s.E * 2 * s.f, (uint64_t)s.d, 64) ||
      !make_tmap_u8(&tX1, xq, (uint64_t)x_rows, (uint64_t)s.d, 16) ||
      !make_tmap_u8(&tW2, w2, (uint64_t)s.E * s.d, (uint64_t)s.f, 128) ||
      !make_tmap_u8(&tX2, hq, (uint64_t)L.Ppad, (uint64_t)s.f, 16))
    return MOE_ERR_CUDA;
  const int nt1 = s.f / 64, nt2 = (s.d + 127) / 128, E = s.E;
  const int e1 = early_gemm1 ? 1 : 0;
  auto quant_h = [&]() {
    return launch_quant_rows(h, nullptr, L.P, 0, s.f, hq, hs, err, st);
  };
  cudaError_t e;
  if (!pair_tiles(s)) {
    // The swap-AB forms: one item per touched expert (T <= 64) or per 128-row
    // tile.  They overlap the three kernels (GEMM1 counting each list entry's
    // stored column tiles, the entry quantiser turning complete entries into
    // codes and counting them, GEMM2 waiting per entry) when an entry is
    // small or there are enough entries for them to complete while GEMM1
    // runs; a few large entries complete only near GEMM1's end, and then the
    // row quantiser between the kernels is cheaper.
    const bool small = s.T <= 64;
    const long long entries = std::min<long long>(E, (long long)s.T * s.k);
    const bool overlap = (long long)s.T * s.k <= 64 || entries >= 16;
    e = small ? swap_ffn_w8a8<64>(tW1, tX1, tW2, tX2, s, L, tiles, h, hq, hs, xs, w13_scale,
                                  w2_scale, z, err, e1, overlap, num_sms, st, mark)
              : swap_ffn_w8a8<128>(tW1, tX1, tW2, tX2, s, L, tiles, h, hq, hs, xs, w13_scale,
                                   w2_scale, z, err, e1, overlap, num_sms, st, mark);
  } else {
    CUtensorMap pA1, pB1, pA2, pB2;  // 128-row boxes: each CTA of a pair loads 128 rows
    if (!make_tmap_u8(&pA1, xq, (uint64_t)x_rows, (uint64_t)s.d, 128) ||
        !make_tmap_u8(&pB1, w13, (uint64_t)s.E * 2 * s.f, (uint64_t)s.d, 128) ||
        !make_tmap_u8(&pA2, hq, (uint64_t)L.Ppad, (uint64_t)s.f, 128) ||
        !make_tmap_u8(&pB2, w2, (uint64_t)s.E * s.d, (uint64_t)s.f, 128))
      return MOE_ERR_CUDA;
    const int* count = tiles;
    const int* rows = row_tile_entries(const_cast<int*>(tiles), E);
    const int* lcount = tiles + 2;
    const int* lrows = leftover_entries(const_cast<int*>(tiles), E);
    const int pnt1 = (s.f + 127) / 128, pnt2 = (s.d + 255) / 256;  // 256-wide output tiles
    GemmArgs g1{count, rows, E, 0, pnt1, s.d, 0, 2 * s.f, s.f, s.f, h, s.f, nullptr, err, 0, 1,
                0, kPdlStart, xs, w13_scale};
    GemmArgs g2{count, rows, E, 0, pnt2, s.f, 0, s.d, 0, s.d, z, s.d, nullptr, err, 0, 1, 0,
                kPdlStart, hs, w2_scale};
    const int max_pairs = (L.max_mtiles + 1) / 2;
    e = launch_gemm_2sm<kEpiSwiGLU, true>(pA1, pB1, g1, max_pairs * pnt1, num_sms, st);
    if (e == cudaSuccess)
      e = launch_swap_t<128, true, true>(tW1, tX1, lcount, lrows, 1, E * nt1, nt1, s.d, 2 * s.f,
                                         s.f, s.f, h, s.f, err, 0, num_sms, st, w13_scale, xs);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess) e = quant_h();
    if (e == cudaSuccess)
      e = launch_gemm_2sm<kEpiStore, true>(pA2, pB2, g2, max_pairs * pnt2, num_sms, st);
    if (e == cudaSuccess)
      e = launch_swap_t<128, false, true>(tW2, tX2, lcount, lrows, 1, E * nt2, nt2, s.f, s.d, 0,
                                          s.d, z, s.d, err, 0, num_sms, st, w2_scale, hs);
  }
  if (e == cudaSuccess) e = mark(1);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Both expert GEMMs over the rows described by the device tile list.
//   x_rows: rows of x_perm visible to TMA (P for a caller buffer, Ppad inside
//   the workspace); h has Ppad rows (workspace).
int launch_expert_ffn(const __nv_bfloat16* x_perm, long long x_rows,
                      const __nv_bfloat16* w13, const __nv_bfloat16* w2,
                      const moe_shape& s, const WsLayout& L, char* ws,
                      __nv_bfloat16* z, int num_sms, cudaStream_t st,
                      void* const* events, bool early_gemm1, const int* tok_row) {
  // events (optional): [0] recorded after GEMM1, [1] after GEMM2.
  auto mark = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st,
                                    cudaEventRecordExternal);
  };
  if (s.T <= kSwapMaxT)
    return launch_expert_ffn_swap(x_perm, x_rows, w13, w2, s, L, ws, z, num_sms, st, events,
                                  early_gemm1, s.T <= 64 ? tok_row : nullptr);
  int* err = reinterpret_cast<int*>(ws + L.err);
  const int* tiles = reinterpret_cast<const int*>(ws + L.tiles);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  const bool pairs = pair_tiles(s);  // the work lists hold tile pairs
  const bool wide = pairs || (L.P >= 64LL * s.E);  // many rows per expert: 256-wide tiles
  CUtensorMap tA1, tB1, tA2, tB2;
  const uint32_t bn = wide ? 256 : 128;
  // Each CTA of a pair loads 128 of the 256 weight rows of a tile.
  const uint32_t b1_box = pairs ? 128 : bn / 2, b2_box = pairs ? 128 : bn;
  if (!make_tmap(&tA1, x_perm, (uint64_t)x_rows, (uint64_t)s.d, kGemmBM) ||
      !make_tmap(&tB1, w13, (uint64_t)s.E * 2 * s.f, (uint64_t)s.d, b1_box) ||
      !make_tmap(&tA2, h, (uint64_t)L.Ppad, (uint64_t)s.f, kGemmBM) ||
      !make_tmap(&tB2, w2, (uint64_t)s.E * s.d, (uint64_t)s.f, b2_box))
    return MOE_ERR_CUDA;
  const int nt1 = (int)((s.f + bn / 2 - 1) / (bn / 2));
  const int nt2 = (int)((s.d + bn - 1) / bn);
  const int* count = tiles;                          // row tiles
  const int* rows = row_tile_entries(const_cast<int*>(tiles), s.E);
  GemmArgs g1{count, rows, s.E, 0, nt1, s.d, s.d / kGemmBK, 2 * s.f, s.f, s.f, h, s.f, nullptr,
              err, 0, 1, 0, kPdlStart};
  GemmArgs g2{count, rows, s.E, 0, nt2, s.f, s.f / kGemmBK, s.d, 0, s.d, z, s.d, nullptr,
              err, 0, 1, 0, kPdlStart};
  cudaError_t e;
  if (pairs) {
    // Pairs first; each expert's odd last tile runs in a single-CTA kernel
    // that starts on the SMs the pair kernel's tail frees (kPdlTail).
    CUtensorMap tB2w;  // 256-row boxes for the single-CTA GEMM2
    if (!make_tmap(&tB2w, w2, (uint64_t)s.E * s.d, (uint64_t)s.f, 256)) return MOE_ERR_CUDA;
    const int* lcount = tiles + 2;
    const int* lrows = leftover_entries(const_cast<int*>(tiles), s.E);
    GemmArgs l1 = g1, l2 = g2;
    l1.tile_count = l2.tile_count = lcount;
    l1.tile_rows = l2.tile_rows = lrows;
    l1.pdl = l2.pdl = kPdlTail;
    g1.pdl = g2.pdl = kPdlAfterWait;
    const int max_pairs = (L.max_mtiles + 1) / 2;
    e = launch_gemm_2sm<kEpiSwiGLU>(tA1, tB1, g1, max_pairs * nt1, num_sms, st);
    if (e == cudaSuccess) e = launch_gemm_t<256, kEpiSwiGLU>(tA1, tB1, l1, s.E * nt1, num_sms, st);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_gemm_2sm<kEpiStore>(tA2, tB2, g2, max_pairs * nt2, num_sms, st);
    if (e == cudaSuccess) e = launch_gemm_t<256, kEpiStore>(tA2, tB2w, l2, s.E * nt2, num_sms, st);
  } else if (wide) {
    e = launch_gemm_t<256, kEpiSwiGLU>(tA1, tB1, g1, L.max_mtiles * nt1, num_sms, st);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_gemm_t<256, kEpiStore>(tA2, tB2, g2, L.max_mtiles * nt2, num_sms, st);
  } else {
    e = launch_gemm_t<128, kEpiSwiGLU>(tA1, tB1, g1, L.max_mtiles * nt1, num_sms, st);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_gemm_t<128, kEpiStore>(tA2, tB2, g2, L.max_mtiles * nt2, num_sms, st);
  }
  if (e == cudaSuccess) e = mark(1);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ============================================================== router, large T
// W_g (d x E, fp32) -> three bf16 planes W3 (E rows x 3d, K-major) with
// W = hi + mid + lo exactly to 24 significant bits: hi = bf16(W),
// mid = bf16(W - hi), lo = bf16(W - hi - mid) (each difference is exact in
// fp32).  x is bf16, so x . W_g = x . [hi | mid | lo] over K = 3d on the bf16
// tensor cores with fp32 accumulation.
__global__ void __launch_bounds__(256) k_router_split(const float* __restrict__ w_g, int d,
                                                      int E, __nv_bfloat16* __restrict__ w3) {
  pdl_trigger();
  pdl_wait();
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int k = k0 + r, e = e0 + tx;
    tile[r][tx] = (k < d && e < E) ? w_g[(size_t)k * E + e] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r, k = k0 + tx;
    if (e < E && k < d) {
      const float v = tile[tx][r];
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(hi);
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(mid);
      const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
      __nv_bfloat16* row = w3 + (size_t)e * 3 * d;
      row[k] = hi;
      row[d + k] = mid;
      row[2 * d + k] = lo;
    }
  }
}

__global__ void __launch_bounds__(256) k_router_finish(const float* __restrict__ part, int P,
                                                       long long n, int E,
                                                       const float* __restrict__ bias,
                                                       float* __restrict__ logits) {
  pdl_trigger();
  pdl_wait();
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long i0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const bool vec = (E & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0 &&
                   (!bias || (reinterpret_cast<uintptr_t>(bias) & 15) == 0);
  if (vec) {
    // 4 logits per thread step; every partial plane's load in flight at once
    // (P <= 84: the partitions hold at least 4 of the 3d/64 <= 768 K blocks).
    const long long n4 = n / 4;
    const float4* p4 = reinterpret_cast<const float4*>(part);
    for (long long i = i0; i < n4; i += stride) {
      float4 v = __ldcs(p4 + i);
      for (int p = 1; p < P; ++p) {
        const float4 u = __ldcs(p4 + (size_t)p * n4 + i);
        v.x += u.x;
        v.y += u.y;
        v.z += u.z;
        v.w += u.w;
      }
      if (bias) {
        const float4 b = __ldg(reinterpret_cast<const float4*>(bias) + (i % (E / 4)));
        v.x += b.x;
        v.y += b.y;
        v.z += b.z;
        v.w += b.w;
      }
      reinterpret_cast<float4*>(logits)[i] = v;
    }
    return;
  }
  for (long long i = i0; i < n; i += stride) {
    float v = part[i];
    for (int p = 1; p < P; ++p) v += part[(size_t)p * n + i];
    logits[i] = bias ? v + bias[i % E] : v;
  }
}

cudaError_t launch_router_tc(const __nv_bfloat16* x, const float* w_g, const float* bias,
                             const moe_shape& s, float* logits, __nv_bfloat16* w3,
                             float* part, int* err, int num_sms, cudaStream_t st) {
  dim3 g((s.d + 31) / 32, (s.E + 31) / 32);
  cudaError_t e = launch_kernel(k_router_split, g, dim3(256), 0, st, 1, w_g, s.d, s.E, w3);
  if (e != cudaSuccess) return e;
  const uint32_t bn = s.E <= 128 ? 128 : 256;
  CUtensorMap tA, tB;
  if (!make_tmap(&tA, x, (uint64_t)s.T, (uint64_t)s.d, kGemmBM) ||
      !make_tmap(&tB, w3, (uint64_t)s.E, (uint64_t)3 * s.d, bn))
    return cudaErrorInvalidValue;
  const int nt = (s.E + bn - 1) / bn;
  const int P = router_tc_parts(s);
  const long long n = (long long)s.T * s.E;
  // Each partition writes its own fp32 plane; k_router_finish adds them in
  // partition order and adds the bias.
  // P == 1: the GEMM writes the logits (with the bias) directly.
  GemmArgs a{nullptr, nullptr, 0, s.T, nt, 3 * s.d, s.d / kGemmBK, 0, 0, s.E,
             P == 1 ? logits : part, s.E, P == 1 ? bias : nullptr, err, 0, P, n, kPdlStart};
  const int work = ((s.T + kGemmBM - 1) / kGemmBM) * nt * P;
  e = (bn == 128) ? launch_gemm_t<128, kEpiLogits>(tA, tB, a, work, num_sms, st)
                  : launch_gemm_t<256, kEpiLogits>(tA, tB, a, work, num_sms, st);
  if (e != cudaSuccess || P == 1) return e;
  const int blocks = (int)std::min<long long>((n + 255) / 256, 4L * num_sms);
  return launch_kernel(k_router_finish, dim3(blocks), dim3(256), 0, st, 1, part, P, n, s.E,
                       bias, logits);
}

}  // namespace moe
