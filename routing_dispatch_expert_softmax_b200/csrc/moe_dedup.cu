// Token-deduplicated per-rank dispatch: a token travels once to every rank
// that owns at least one of its selected experts ("Serving MoE models with
// expert parallelism on 8xH200", section "Tensor parallel vs expert
// parallel"; "Expert Parallelism for MoE Models", section "Mechanics of Token
// Routing and All-to-All Communication").  Ranks own contiguous expert
// blocks, owner(e) = e / (E/R); source rank src(t) = t / ceil(T/R).  The send
// buffer is rank-major with tokens ascending inside a rank; each row carries
// the token and a k-bit mask of its slots that rank owns.
//   k_dedup_hist:    per block of tokens, rows per destination rank and per
//                    (source, destination) pair
//   k_dedup_scan:    rank offsets, per-block bases, send counts
//   k_dedup_scatter: stable rows (per-warp ballots per rank), token, mask,
//                    rank_row_of
//   k_dedup_gather:  x rows into the send buffer
#include "moe_kernels.cuh"

namespace moe {
namespace {

constexpr int kDedupBlock = 256;  // tokens per block
constexpr int kDedupWarps = kDedupBlock / 32;

// Bit r set when one of token t's slots lands on rank r (R <= 64); invalid
// ids are recorded and skipped.
__device__ __forceinline__ uint64_t token_ranks(const int* __restrict__ idx, int t, int k,
                                                int E, int per, int* err) {
  uint64_t m = 0;
  for (int j = 0; j < k; ++j) {
    const int e = idx[(size_t)t * k + j];
    if (e < 0 || e >= E) {
      record_error(err, MOE_ERR_DEVICE_CHECK, 40);
      continue;
    }
    m |= 1ull << (e / per);
  }
  return m;
}

__global__ void __launch_bounds__(kDedupBlock) k_dedup_hist(
    const int* __restrict__ idx, int T, int E, int k, int R, int src_chunk,
    int* __restrict__ blockcnt, int* __restrict__ blocksend, int* err) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  int* cnt = sm;       // [R]
  int* send = sm + R;  // [R*R]
  for (int i = threadIdx.x; i < R + R * R; i += blockDim.x) sm[i] = 0;
  __syncthreads();
  const int t = blockIdx.x * kDedupBlock + threadIdx.x;
  if (t < T) {
    const int src = t / src_chunk;
    uint64_t m = token_ranks(idx, t, k, E, E / R, err);
    while (m) {
      const int r = __ffsll((long long)m) - 1;
      m &= m - 1;
      atomicAdd(&cnt[r], 1);
      atomicAdd(&send[src * R + r], 1);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < R; i += blockDim.x) blockcnt[(size_t)blockIdx.x * R + i] = cnt[i];
  for (int i = threadIdx.x; i < R * R; i += blockDim.x)
    blocksend[(size_t)blockIdx.x * R * R + i] = send[i];
}

// One block of 1024 threads.
__global__ void __launch_bounds__(1024) k_dedup_scan(const int* __restrict__ blockcnt,
                                                     int nblocks, int R,
                                                     const int* __restrict__ blocksend,
                                                     int* __restrict__ blockbase,
                                                     int* __restrict__ send_out,
                                                     int* __restrict__ rank_off) {
  pdl_trigger();
  pdl_wait();
  __shared__ int tot[65];
  const int r = threadIdx.x;
  if (r < R) {
    int c = 0;
    for (int b = 0; b < nblocks; ++b) c += blockcnt[(size_t)b * R + r];
    tot[r] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0;
    for (int q = 0; q < R; ++q) {
      const int c = tot[q];
      tot[q] = a;
      a += c;
    }
    tot[R] = a;
  }
  __syncthreads();
  if (r <= R) rank_off[r] = tot[r];
  if (r < R) {
    int a = tot[r];
    for (int b = 0; b < nblocks; ++b) {
      blockbase[(size_t)b * R + r] = a;
      a += blockcnt[(size_t)b * R + r];
    }
  }
  for (int i = threadIdx.x; i < R * R; i += blockDim.x) {
    int c = 0;
    for (int b = 0; b < nblocks; ++b) c += blocksend[(size_t)b * R * R + i];
    send_out[i] = c;
  }
}

__global__ void __launch_bounds__(kDedupBlock) k_dedup_scatter(
    const int* __restrict__ idx, int T, int E, int k, int R,
    const int* __restrict__ blockbase, int* __restrict__ token_of,
    uint32_t* __restrict__ slot_mask, int* __restrict__ rank_row_of) {
  pdl_trigger();
  pdl_wait();
  __shared__ int wcnt[kDedupWarps][64];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int t = blockIdx.x * kDedupBlock + threadIdx.x;
  const bool valid = t < T;
  const int per = E / R;
  uint64_t m = 0;  // ranks this token goes to (0 for lanes past T)
  if (valid)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) m |= 1ull << (e / per);  // invalid ids: recorded by k_dedup_hist
    }
  for (int r = 0; r < R; ++r) {
    const uint32_t b = __ballot_sync(0xffffffffu, (m >> r) & 1ull);
    if (lane == 0) wcnt[wid][r] = __popc(b);
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int r = 0; r < R; ++r) {
    // every lane votes, so the ballot is the same in both loops
    const uint32_t b = __ballot_sync(0xffffffffu, (m >> r) & 1ull);
    if (!valid) continue;
    int row = -1;
    if ((m >> r) & 1ull) {
      row = blockbase[(size_t)blockIdx.x * R + r] + __popc(b & lt);
      for (int w2 = 0; w2 < wid; ++w2) row += wcnt[w2][r];
      uint32_t mask = 0;
      for (int j = 0; j < k; ++j) {
        const int e = idx[(size_t)t * k + j];
        if (e >= 0 && e < E && e / per == r) mask |= 1u << j;
      }
      token_of[row] = t;
      slot_mask[row] = mask;
    }
    if (rank_row_of) rank_row_of[(size_t)t * R + r] = row;
  }
}

// x_dedup[row] = x[token_of[row]] for the rows that exist (rank_off[R] of
// them, known only on the device): a warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) k_dedup_gather(const __nv_bfloat16* __restrict__ x,
                                                      const int* __restrict__ token_of,
                                                      const int* __restrict__ rank_off, int R,
                                                      int T, int d,
                                                      __nv_bfloat16* __restrict__ x_dedup,
                                                      int* err) {
  pdl_trigger();
  pdl_wait();
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rank_off[R]) return;
  const int lane = threadIdx.x & 31;
  const int t = token_of[row];
  if (t < 0 || t >= T) {
    if (lane == 0) record_error(err, MOE_ERR_DEVICE_CHECK, 41);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(x_dedup + (size_t)row * d);
  for (int c = lane; c < d / 8; c += 32) dst[c] = __ldg(src + c);
}

}  // namespace
}  // namespace moe

using namespace moe;

namespace {
bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

extern "C" int moe_dispatch_dedup(const int32_t* idx, const moe_bf16* x, const moe_shape* s,
                                  int32_t* send_counts, int32_t* rank_offsets,
                                  int32_t* token_of, uint32_t* slot_mask,
                                  int32_t* rank_row_of, moe_bf16* x_dedup, void* ws,
                                  void* stream) {
  if (!shape_valid(s) || s->R < 2) return MOE_ERR_INVALID_ARG;
  if (!ws || !al(ws, 256) || !send_counts || !rank_offsets || !al(send_counts, 4) ||
      !al(rank_offsets, 4))
    return MOE_ERR_INVALID_ARG;
  if (s->T > 0 && (!idx || !token_of || !slot_mask || !al(idx, 4) || !al(token_of, 4) ||
                   !al(slot_mask, 4) || (rank_row_of && !al(rank_row_of, 4)) ||
                   (x_dedup && (!x || !al(x, 16) || !al(x_dedup, 16)))))
    return MOE_ERR_INVALID_ARG;
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int R = s->R, T = s->T;
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(send_counts, 0, sizeof(int) * R * R, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(rank_offsets, 0, sizeof(int) * (R + 1), st);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  const WsLayout L = ws_layout(*s, sms);
  char* w = static_cast<char*>(ws);
  int* err = reinterpret_cast<int*>(w + L.err);
  int* blockcnt = reinterpret_cast<int*>(w + L.blockhist);   // nblocks x R <= nblocks x E
  int* blockbase = reinterpret_cast<int*>(w + L.blockbase);
  int* blocksend = reinterpret_cast<int*>(w + L.blocksend);  // nblocks x R x R
  static_assert(kDedupBlock == kTokensPerRouteBlock, "blocks match the workspace carve");
  const int nblocks = (T + kDedupBlock - 1) / kDedupBlock;
  const int chunk = (T + R - 1) / R;
  const size_t hist_smem = sizeof(int) * (R + R * R);
  cudaError_t e = launch_kernel(k_dedup_hist, dim3(nblocks), dim3(kDedupBlock), hist_smem, st,
                                1, idx, T, s->E, s->k, R, chunk, blockcnt, blocksend, err);
  if (e == cudaSuccess)
    e = launch_kernel(k_dedup_scan, dim3(1), dim3(1024), 0, st, 1, (const int*)blockcnt,
                      nblocks, R, (const int*)blocksend, blockbase, send_counts, rank_offsets);
  if (e == cudaSuccess)
    e = launch_kernel(k_dedup_scatter, dim3(nblocks), dim3(kDedupBlock), 0, st, 1, idx, T,
                      s->E, s->k, R, (const int*)blockbase, token_of, slot_mask, rank_row_of);
  if (e == cudaSuccess && x_dedup) {
    const long long rows = (long long)T * (s->k < R ? s->k : R);
    e = launch_kernel(k_dedup_gather, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st, 1,
                      reinterpret_cast<const __nv_bfloat16*>(x), (const int*)token_of,
                      (const int*)rank_offsets, R, T, s->d,
                      reinterpret_cast<__nv_bfloat16*>(x_dedup), err);
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
