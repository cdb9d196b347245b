// Row quantisation of bf16 activations to E4M3 codes with one power-of-two
// scale per row, for the expert GEMMs whose operands are both E4M3
// (tcgen05 kind::f8f6f4).
//
// "Serving MoE models with expert parallelism on 8xH200", sections "Memory
// math for 8xH200" and "Quantization choices": one-byte FP8 weights are the
// native format of the large MoE checkpoints.  The pages fix no activation
// format; the one taken here: row r gets the scale 2^e_r, e_r the smallest
// integer with max_c |a[r,c]| <= 448 * 2^e_r (0 for an all-zero row), and
// code[r,c] is the E4M3 value nearest to a[r,c] * 2^-e_r, ties to even.
// Scaling by a power of two is exact, so the codes depend on the input only.
#include "moe_kernels.cuh"

#include <cuda_fp8.h>

namespace moe {

// 2^k as an fp32 for -126 <= k <= 127 (a normal number: exponent field k+127).
__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }

// Smallest e with (bf16 magnitude bits m) <= 448 * 2^e; 0 for m == 0.
// A normal bf16 magnitude is (1 + f/128) * 2^(x-127) with x = m >> 7 and
// f = m & 127; 448 = 1.75 * 2^8, so e = x - 135 when f <= 96 (1 + f/128 <=
// 1.75) and x - 134 otherwise.  A subnormal one is f * 2^-133; with p the
// top bit of f, f = (f / 2^p) * 2^p and the same comparison reads 4f <= 7 * 2^p.
__device__ __forceinline__ int pow2_exponent_of_bf16_mag(uint32_t m) {
  if (m == 0) return 0;
  const int x = (int)(m >> 7), f = (int)(m & 127);
  if (x > 0) return x - 135 + (f > 96 ? 1 : 0);
  const int p = 31 - __clz(f);
  return p - 141 + (4 * f > (7 << p) ? 1 : 0);
}

// One row of cols elements (a multiple of 8) to codes and (lane 0) its
// scale, one warp cooperating.  L2: read around L1 (rows another CTA of a
// running kernel wrote); else through the read-only path.
template <bool L2>
__device__ __forceinline__ void quant_row(const __nv_bfloat16* src, int cols, uint8_t* codes,
                                          float* scale, int lane) {
  const uint4* in = reinterpret_cast<const uint4*>(src);
  auto ld = [&](int c) { return L2 ? __ldcg(in + c) : __ldg(in + c); };
  const int nv = cols / 8;
  // the largest magnitude: bf16 magnitude bits order like the magnitudes
  uint32_t m = 0;
  for (int c = lane; c < nv; c += 32) {
    const uint4 v = ld(c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  const int e = pow2_exponent_of_bf16_mag(m);
  // multiply by 2^-e in two exact steps (each factor a normal fp32)
  const int k1 = (-e) >> 1, k2 = -e - k1;
  const float s1 = pow2f(k1), s2 = pow2f(k2);
  uint2* out = reinterpret_cast<uint2*>(codes);
  for (int c = lane; c < nv; c += 32) {
    const uint4 v = ld(c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(w[i] << 16) * s1 * s2;
      const float hi = __uint_as_float(w[i] & 0xFFFF0000u) * s1 * s2;
      const uint32_t pair =
          __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
      if (i & 1)
        q[i >> 1] |= pair << 16;
      else
        q[i >> 1] = pair;
    }
    out[c] = make_uint2(q[0], q[1]);
  }
  if (lane == 0) *scale = pow2f(e >> 1) * pow2f(e - (e >> 1));
}

// One warp per row.  GATHER: output row r quantises input row perm[r] (the
// dispatch gather fused in), else input row r.
template <bool GATHER>
__global__ void __launch_bounds__(256) k_quant_rows_e4m3(
    const __nv_bfloat16* __restrict__ a, const int* __restrict__ perm, long long rows,
    int n_src, int cols, uint8_t* __restrict__ codes, float* __restrict__ scales,
    int* __restrict__ err) {
  // The next kernel (an expert GEMM) may read the work lists before its own
  // wait only if this kernel lets it launch after this wait.
  pdl_wait();
  pdl_trigger();
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  long long src = row;
  if (GATHER) {
    const int t = perm[row];
    if (t < 0 || t >= n_src) {
      if (lane == 0) record_error(err, MOE_ERR_DEVICE_CHECK, 13);
      return;
    }
    src = t;
  }
  quant_row<false>(a + src * cols, cols, codes + row * cols, scales + row, lane);
}

// One row of cols <= 32 * 8 * kRegVecs elements held in registers (loaded
// once through L2, then the maximum and the codes as quant_row computes them).
// Same-box A/B against the two-pass quant_row: Qwen3 W8A8 T = 256 163 -> 156
// us with 768-column rows; 2048-column rows (DeepSeek-V3) were slower this way.
constexpr int kRegVecs = 4;  // 16-byte vectors per lane: rows of up to 1024 bf16
__device__ __forceinline__ void quant_row_regs(const __nv_bfloat16* src, int cols,
                                               uint8_t* codes, float* scale, int lane) {
  const uint4* in = reinterpret_cast<const uint4*>(src);
  const int nv = cols / 8;
  uint4 v[kRegVecs];
#pragma unroll
  for (int i = 0; i < kRegVecs; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < nv ? __ldcg(in + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kRegVecs; ++i) {
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  const int e = pow2_exponent_of_bf16_mag(m);
  const int k1 = (-e) >> 1, k2 = -e - k1;
  const float s1 = pow2f(k1), s2 = pow2f(k2);
  uint2* out = reinterpret_cast<uint2*>(codes);
#pragma unroll
  for (int i = 0; i < kRegVecs; ++i) {
    const int c = lane + 32 * i;
    if (c < nv) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t q[2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = __uint_as_float(w[j] << 16) * s1 * s2;
        const float hi = __uint_as_float(w[j] & 0xFFFF0000u) * s1 * s2;
        const uint32_t pair =
            __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
        if (j & 1)
          q[j >> 1] |= pair << 16;
        else
          q[j >> 1] = pair;
      }
      out[c] = make_uint2(q[0], q[1]);
    }
  }
  if (lane == 0) *scale = pow2f(e >> 1) * pow2f(e - (e >> 1));
}

// The SwiGLU output of the small-batch W8A8 GEMM1, quantised per work-list
// entry while GEMM1 runs: block i takes entry i (list entries: row0, row_end,
// expert; row_tiles caps an entry at 128 rows), waits (bounded) until GEMM1
// has stored all `target1` column tiles of the entry's rows (ready1[i]),
// quantises those rows as k_quant_rows_e4m3 does (the reads go through L2:
// GEMM1 wrote them while this kernel ran), then sets ready2[i] for GEMM2.  It
// lets GEMM2 launch at once and waits for GEMM1 only at its end, so its
// completion still implies GEMM1's.
__global__ void __launch_bounds__(256) k_quant_entries_e4m3(
    const __nv_bfloat16* __restrict__ h, int cols, const int* __restrict__ list_count,
    const int* __restrict__ list, int row_tiles, const int* __restrict__ ready1, int target1,
    int* __restrict__ ready2, uint8_t* __restrict__ codes, float* __restrict__ scales,
    int* __restrict__ err) {
  pdl_trigger();
  __shared__ int go;
  const int i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (i < __ldcg(list_count)) {
    const int row0 = __ldcg(list + 3 * i + 0);
    const int rows = __ldcg(list + 3 * i + 1) - row0;
    const int n = row_tiles ? min(rows, kGemmBM) : rows;
    if (threadIdx.x == 0) {
      int flag = 0;
      go = wait_count_bounded(ready1 + i, target1, &flag) ? 1 : 0;
      if (!go) record_error(err, MOE_ERR_TIMEOUT, 16);
    }
    __syncthreads();
    if (go) {
      __threadfence();
      const int nw = blockDim.x >> 5;
      for (int r = warp; r < n; r += nw) {  // one row per warp
        const size_t o = (size_t)(row0 + r) * cols;
        if (cols <= 256 * kRegVecs)
          quant_row_regs(h + o, cols, codes + o, scales + row0 + r, lane);
        else
          quant_row<true>(h + o, cols, codes + o, scales + row0 + r, lane);
      }
      fence_proxy_async_global();  // the codes before GEMM2's TMA reads
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ready2 + i, 1);
      }
    }
  }
  pdl_wait();
}

// Threads per entry block: one warp per row of the entry, 8 rows at once (a
// block of 1024 threads does not fit beside a GEMM1 CTA's registers).
constexpr int kQuantEntryThreads = 256;

cudaError_t launch_quant_entries(const __nv_bfloat16* h, int cols, const int* list_count,
                                 const int* list, int row_tiles, int max_entries,
                                 const int* ready1, int target1, int* ready2, uint8_t* codes,
                                 float* scales, int* err, cudaStream_t st) {
  if (max_entries < 1) return cudaSuccess;
  return launch_kernel(k_quant_entries_e4m3, dim3((unsigned)max_entries), dim3(kQuantEntryThreads), 0, st, 1,
                       h, cols, list_count, list, row_tiles, ready1, target1, ready2, codes,
                       scales, err);
}

cudaError_t launch_quant_rows(const __nv_bfloat16* a, const int* perm, long long rows, int n_src,
                              int cols, uint8_t* codes, float* scales, int* err,
                              cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + 7) / 8;
  if (perm)
    return launch_kernel(k_quant_rows_e4m3<true>, dim3((unsigned)blocks), dim3(256), 0, st, 1, a,
                         perm, rows, n_src, cols, codes, scales, err);
  return launch_kernel(k_quant_rows_e4m3<false>, dim3((unsigned)blocks), dim3(256), 0, st, 1, a,
                       perm, rows, n_src, cols, codes, scales, err);
}

}  // namespace moe
