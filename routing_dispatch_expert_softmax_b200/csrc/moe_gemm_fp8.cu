// Small-batch expert GEMMs with FP8 (E4M3) expert weights.
//
// "Serving MoE models with expert parallelism on 8xH200", section
// "Memory math for 8xH200": DeepSeek-V3 and the Qwen3 FP8 variants ship their
// weights at one byte per parameter; section "Quantization choices": native FP8
// checkpoints are the default; and its FAQ: each expert sees a small slice of
// the batch, so the expert GEMMs are bound by streaming the expert's weights.
// Halving the bytes of every weight halves that stream.
//
// Weight format (the pages name FP8 but no encoding or scale granularity):
// every weight is an OCP FP8 E4M3 code, and every output row of an expert's
// matrix (a row of W_gate, W_up or W_down in the same [rows, K] K-major storage
// the bf16 path uses) carries one fp32 scale:  W[r, c] = e4m3(code[r, c]) * scale[r].
// A row scale factors out of the row's dot products, so the kernel multiplies
// the fp32 accumulator by it in the epilogue.
//
// Same work items and roles as the bf16 swap-AB kernel (weights are the M = 128
// operand, the expert's token rows the N operand), plus a converter warpgroup:
//   warp 0      TMA producer: each raw stage receives the e4m3 weight tile
//               (128 rows x 64 bytes, unswizzled) and, beside it, the stage's
//               bf16 token tile (128-byte swizzled, the MMA layout), so both
//               stream through the same deep ring;
//   warps 6-9   widen each raw weight tile to bf16 (exact: every E4M3 value is
//               a bf16 value) and write it 128-byte swizzled, K-major, into a
//               short ring of converted-weight stages;
//   warp 1      owns TMEM and issues tcgen05.mma kind::f16 with A = converted
//               weights, B = the token tile still in its raw stage; a raw
//               stage is free once the four converter warps and the MMA are
//               done with it;
//   warps 2-5   drain the accumulator, apply the row scales (and SwiGLU), store.
// Activations stay bf16, so the result is the bf16 path's arithmetic applied to
// the dequantised weights.  Every wait is bounded (error word MOE_ERR_TIMEOUT,
// then drain and return).
#include <cuda_fp8.h>

#include "moe_kernels.cuh"

namespace moe {
namespace {

template <int NMAX, bool SWIGLU>
struct F8Cfg {
  // Raw stages in flight: 9 x (8 KB e4m3 + 8 KB tokens) at NMAX = 64,
  // 6 x (8 + 16 KB) at NMAX = 128; two converted-weight stages.
  static constexpr int kRawStages = NMAX <= 64 ? 9 : 6;
  static constexpr int kMmaStages = 2;
  static constexpr int kRawWBytes = 128 * kGemmBK;        // 8 KB of e4m3
  static constexpr int kXBytes = NMAX * kGemmBK * 2;      // token rows, bf16
  static constexpr int kRawBytes = kRawWBytes + kXBytes;  // one raw stage
  static constexpr int kWBytes = 128 * kGemmBK * 2;       // 16 KB of bf16
  static constexpr int kMmaBytes = kWBytes;
  static constexpr int kTmemCols = 2 * NMAX;
  static constexpr int kXchBytes = SWIGLU ? 2 * 64 * 16 * 4 : 0;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes =
      kMmaStages * kMmaBytes + kRawStages * kRawBytes + kXchBytes + kBarBytes + 1024;
  static constexpr int kThreads = 320;
  static_assert(8 * (2 * kRawStages + 2 * kMmaStages + 5) + 8 <= kBarBytes, "barriers");
  static_assert(kRawBytes % 1024 == 0 && kWBytes % 1024 == 0, "swizzled tiles 1024-aligned");
};

__device__ __forceinline__ bool wait_limit(uint64_t* bar, uint32_t parity,
                                           unsigned long long limit_ns) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ void bar_sync_named(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (tensor core) reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ float silu_fast(float g) { return g / (1.0f + __expf(-g)); }

// Two E4M3 codes (low byte first) -> a bf16x2 word (low half first).  The
// hardware e4m3x2 -> f16x2 conversion is exact, and so are f16 -> f32 and an
// f32 holding a 4-bit-significand value -> bf16.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two_codes) {
  const __half2_raw hr =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
  return pack_bf16x2(f.x, f.y);
}

// Work items as in the bf16 swap-AB kernel: list entries (row0, row_end,
// expert); with row_tiles an entry covers at most 128 of its expert's rows.
template <int NMAX, bool SWIGLU>
__global__ void __launch_bounds__(320, 1) k_expert_gemm_swap_f8(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
    const float* __restrict__ w_scale, const int* __restrict__ list_count,
    const int* __restrict__ list, int row_tiles, int n_tiles, int K, int w_rows_per_expert,
    int up_offset, int n_out, __nv_bfloat16* __restrict__ out, int ld_out,
    int* __restrict__ err) {
  using C = F8Cfg<NMAX, SWIGLU>;
  constexpr int RS = C::kRawStages;
  constexpr int MS = C::kMmaStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* mma_st = smem;                                  // MS x bf16 W
  uint8_t* raw_st = smem + MS * C::kMmaBytes;              // RS x (e4m3 W | bf16 tokens)
  float* xch = reinterpret_cast<float*>(raw_st + RS * C::kRawBytes);
  uint64_t* rfull = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xch) + C::kXchBytes);
  uint64_t* rempty = rfull + RS;   // 4 converter warps + the MMA commit
  uint64_t* wfull = rempty + RS;   // converted weights written (4 converter warps)
  uint64_t* mempty = wfull + MS;   // converted-weight stage free (tcgen05.commit)
  uint64_t* tfull = mempty + MS;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < RS; ++s2) {
      mbar_init(&rfull[s2], 1);
      mbar_init(&rempty[s2], 5);
    }
    for (int s2 = 0; s2 < MS; ++s2) {
      mbar_init(&wfull[s2], 4);
      mbar_init(&mempty[s2], 1);
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
  pdl_trigger();
  pdl_wait();  // the work lists and the token rows come from the previous kernels
  const int total = list_count[0] * n_tiles;
  const int nk = K / kGemmBK;
  const int* et = list;
  auto item_rows = [&](int i) {
    const int r = et[3 * i + 1] - et[3 * i + 0];
    return row_tiles ? min(r, kGemmBM) : r;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ producer: e4m3 weights + tokens
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int fills[RS];
#pragma unroll
      for (int s2 = 0; s2 < RS; ++s2) fills[s2] = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int i = w / n_tiles, nt = w - (w / n_tiles) * n_tiles;
        const int row0 = et[3 * i + 0];
        const int n = item_rows(i);
        const int e = et[3 * i + 2];
        if (n < 1 || n > NMAX) continue;  // recorded by the epilogue
        const int nb = (n + 15) >> 4;
        const int wrow = e * w_rows_per_expert + nt * (SWIGLU ? 64 : 128);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&rempty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* dst = raw_st + stage * C::kRawBytes;
          uint8_t* xdst = dst + C::kRawWBytes;
          mbar_arrive_expect_tx(&rfull[stage], (uint32_t)(C::kRawWBytes + nb * 16 * 128));
          if (SWIGLU) {
            tma_load_2d(dst, &tmW, &rfull[stage], kb * kGemmBK, wrow, pol_w);
            tma_load_2d(dst + 64 * kGemmBK, &tmW, &rfull[stage], kb * kGemmBK, wrow + up_offset,
                        pol_w);
          } else {
            tma_load_2d(dst, &tmW, &rfull[stage], kb * kGemmBK, wrow, pol_w);
          }
          for (int b = 0; b < nb; ++b)
            tma_load_2d(xdst + b * 16 * 128, &tmX, &rfull[stage], kb * kGemmBK, row0 + 16 * b,
                        pol_x);
          ++fills[stage];
          if (++stage == RS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
#pragma unroll
        for (int s2 = 0; s2 < RS; ++s2)
          if (fills[s2] > 0) wait_limit(&rfull[s2], (uint32_t)((fills[s2] - 1) & 1), 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0, rs = 0;
      uint32_t phase = 0, rph = 0;
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
        const int i = w / n_tiles;
        const int n = item_rows(i);
        if (n < 1 || n > NMAX) {
          --it;
          continue;
        }
        const uint32_t idesc = idesc_bf16_f32(128, ((n + 15) >> 4) * 16);
        const int ab = it & 1;
        const uint32_t aph = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait_bounded(&tempty[ab], aph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(ab * NMAX);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&wfull[stage], phase, abort_flag) ||
              !mbar_wait_bounded(&rfull[rs], rph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(mma_st + stage * C::kMmaBytes);
          const uint32_t b_addr = smem_u32(raw_st + rs * C::kRawBytes + C::kRawWBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            umma_bf16_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                         sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&mempty[stage]);
          umma_commit(&rempty[rs]);  // the raw stage's token tile is read
          if (++stage == MS) {
            stage = 0;
            phase ^= 1u;
          }
          if (++rs == RS) {
            rs = 0;
            rph ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[ab]);
      }
      if (*abort_flag) {
        umma_commit(drain);
        wait_limit(drain, 0, 100000000ull);
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------ converters (warps 6..9)
    const int ct = threadIdx.x - 192;  // 0..127
    int rs = 0, ms = 0;
    uint32_t rph = 0, mph = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int i = w / n_tiles;
      const int n = item_rows(i);
      if (n < 1 || n > NMAX) continue;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_bounded(&mempty[ms], mph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* wdst = mma_st + ms * C::kMmaBytes;
        if (!mbar_wait_bounded(&rfull[rs], rph, abort_flag)) {
          ok = false;
          break;
        }
        // 128 rows x 4 chunks of 16 codes; chunk j of row r becomes bf16
        // chunks 2j and 2j+1 of the row, at 16-byte slots (2j)^(r&7) and
        // (2j+1)^(r&7) (the 128-byte swizzle).
        const uint8_t* src = raw_st + rs * C::kRawBytes;
#pragma unroll
        for (int c = ct; c < 512; c += 128) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + c * 16);
          const int r = c >> 2, j = c & 3, sw = r & 7;
          uint4 lo, hi;
          lo.x = e4m3x2_to_bf16x2(v.x & 0xFFFFu);
          lo.y = e4m3x2_to_bf16x2(v.x >> 16);
          lo.z = e4m3x2_to_bf16x2(v.y & 0xFFFFu);
          lo.w = e4m3x2_to_bf16x2(v.y >> 16);
          hi.x = e4m3x2_to_bf16x2(v.z & 0xFFFFu);
          hi.y = e4m3x2_to_bf16x2(v.z >> 16);
          hi.z = e4m3x2_to_bf16x2(v.w & 0xFFFFu);
          hi.w = e4m3x2_to_bf16x2(v.w >> 16);
          uint8_t* rowp = wdst + r * 128;
          *reinterpret_cast<uint4*>(rowp + (((2 * j) ^ sw) << 4)) = lo;
          *reinterpret_cast<uint4*>(rowp + (((2 * j + 1) ^ sw) << 4)) = hi;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[rs]);
          mbar_arrive(&wfull[ms]);
        }
        if (++rs == RS) {
          rs = 0;
          rph ^= 1u;
        }
        if (++ms == MS) {
          ms = 0;
          mph ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lanes q*32 .. q*32+31 = weight rows of the item
    int it = 0;
    int chunk_parity = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      const int i = w / n_tiles, nt = w - (w / n_tiles) * n_tiles;
      const int row0 = et[3 * i + 0];
      const int n = item_rows(i);
      const int e = et[3 * i + 2];
      if (n < 1 || n > NMAX) {
        if (threadIdx.x == 64) record_error(err, MOE_ERR_DEVICE_CHECK, 15);
        --it;
        continue;
      }
      // this thread's weight row and its scale
      int col, srow;
      if (SWIGLU) {
        col = nt * 64 + (q & 1) * 32 + lane;
        srow = e * w_rows_per_expert + col + (q >= 2 ? up_offset : 0);
      } else {
        col = nt * 128 + q * 32 + lane;
        srow = e * w_rows_per_expert + col;
      }
      const float sc = col < n_out ? __ldg(w_scale + srow) : 0.0f;
      const int ncols = ((n + 15) >> 4) * 16;
      const int ab = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      mbar_wait_bounded(&tfull[ab], aph, abort_flag);
      bar_sync_named(2, 128);
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + (uint32_t)(ab * NMAX) + ((uint32_t)(q * 32) << 16);
      if (SWIGLU) {
        // lanes 0..63: gate rows j, lanes 64..127: up rows j (j = lane & 63)
        const int j = (q & 1) * 32 + lane;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float* x = xch + chunk_parity * (64 * 16);
          uint32_t v[16];
          tmem_ld_x16(t_addr + c0, v);
          tmem_ld_wait();
          if (q >= 2) {
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) x[cc * 64 + j] = __uint_as_float(v[cc]) * sc;
          }
          bar_sync_named(1, 128);
          if (q < 2 && col < n_out) {
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const int c = c0 + cc;
              if (c < n) {
                const float g = __uint_as_float(v[cc]) * sc;
                const float u = x[cc * 64 + j];
                out[(size_t)(row0 + c) * ld_out + col] = __float2bfloat16_rn(silu_fast(g) * u);
              }
            }
          }
          chunk_parity ^= 1;
        }
      } else {
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          uint32_t v[16];
          tmem_ld_x16(t_addr + c0, v);
          tmem_ld_wait();
          if (col < n_out) {
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const int c = c0 + cc;
              if (c < n)
                out[(size_t)(row0 + c) * ld_out + col] =
                    __float2bfloat16_rn(__uint_as_float(v[cc]) * sc);
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
  if (threadIdx.x == 0 && *abort_flag) record_error(err, MOE_ERR_TIMEOUT, 14);
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ============================================================== host side
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

PFN_encodeTiled_t encode_fn() {
  static PFN_encodeTiled_t fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled_t>(p);
  }
  return fn;
}

// Row-major [rows, cols] matrix, box = 64 elements x box_rows.  bf16 tiles are
// 128-byte swizzled (the MMA layout); e4m3 tiles (64 bytes a row) are left
// unswizzled for the converters, which read them row by row.
bool tmap_2d(CUtensorMap* tm, const void* base, bool e4m3, uint64_t rows, uint64_t cols,
             uint32_t box_rows) {
  PFN_encodeTiled_t enc = encode_fn();
  if (!enc) return false;
  const uint64_t esz = e4m3 ? 1 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {(cuuint32_t)kGemmBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   e4m3 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int NMAX, bool SWIGLU>
cudaError_t launch_swap_f8(const CUtensorMap& tw, const CUtensorMap& tx, const float* scale,
                           const int* list_count, const int* list, int row_tiles, int max_work,
                           int n_tiles, int K, int w_rows, int up_off, int n_out,
                           __nv_bfloat16* out, int ld_out, int* err, int num_sms,
                           cudaStream_t st) {
  using C = F8Cfg<NMAX, SWIGLU>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_expert_gemm_swap_f8<NMAX, SWIGLU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int grid = max_work < num_sms ? max_work : num_sms;
  if (grid < 1) grid = 1;
  return launch_kernel(k_expert_gemm_swap_f8<NMAX, SWIGLU>, dim3(grid), dim3(C::kThreads),
                       C::kSmemBytes, st, 1, tw, tx, scale, list_count, list, row_tiles, n_tiles,
                       K, w_rows, up_off, n_out, out, ld_out, err);
}

}  // namespace

int launch_expert_ffn_fp8(const __nv_bfloat16* x_perm, long long x_rows, const uint8_t* w13,
                          const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                          const moe_shape& s, const WsLayout& L, char* ws, __nv_bfloat16* z,
                          int num_sms, cudaStream_t st, void* const* events) {
  auto mark = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st,
                                    cudaEventRecordExternal);
  };
  int* err = reinterpret_cast<int*>(ws + L.err);
  const int* tiles = reinterpret_cast<const int*>(ws + L.tiles);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  CUtensorMap tW1, tX1, tW2, tX2;
  if (!tmap_2d(&tW1, w13, true, (uint64_t)s.E * 2 * s.f, (uint64_t)s.d, 64) ||
      !tmap_2d(&tX1, x_perm, false, (uint64_t)x_rows, (uint64_t)s.d, 16) ||
      !tmap_2d(&tW2, w2, true, (uint64_t)s.E * s.d, (uint64_t)s.f, 128) ||
      !tmap_2d(&tX2, h, false, (uint64_t)L.Ppad, (uint64_t)s.f, 16))
    return MOE_ERR_CUDA;
  const int nt1 = s.f / 64;           // 64 gate + 64 up rows per item
  const int nt2 = (s.d + 127) / 128;  // 128 output columns per item
  const int E = s.E;
  cudaError_t e;
  if (s.T <= 64) {
    const int* cnt = tiles + 1;  // touched experts, one item each (<= 64 rows)
    const int* ents = expert_entries(const_cast<int*>(tiles));
    e = launch_swap_f8<64, true>(tW1, tX1, w13_scale, cnt, ents, 0, E * nt1, nt1, s.d, 2 * s.f,
                                 s.f, s.f, h, s.f, err, num_sms, st);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_swap_f8<64, false>(tW2, tX2, w2_scale, cnt, ents, 0, E * nt2, nt2, s.f, s.d, 0,
                                    s.d, z, s.d, err, num_sms, st);
  } else {
    const int* cnt = tiles;  // 128-row tiles
    const int* ents = row_tile_entries(const_cast<int*>(tiles), E);
    e = launch_swap_f8<128, true>(tW1, tX1, w13_scale, cnt, ents, 1, L.max_mtiles * nt1, nt1,
                                  s.d, 2 * s.f, s.f, s.f, h, s.f, err, num_sms, st);
    if (e == cudaSuccess) e = mark(0);
    if (e == cudaSuccess)
      e = launch_swap_f8<128, false>(tW2, tX2, w2_scale, cnt, ents, 1, L.max_mtiles * nt2, nt2,
                                     s.f, s.d, 0, s.d, z, s.d, err, num_sms, st);
  }
  if (e == cudaSuccess) e = mark(1);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
