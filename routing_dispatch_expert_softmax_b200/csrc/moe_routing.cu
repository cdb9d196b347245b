// Routing, dispatch and combine kernels of the routed MoE layer (sm_100a).
//
// Steps (the layer of "Wide Expert Parallelism", section "What is an MoE
// layer?", and "Serving MoE models with expert parallelism on 8xH200",
// sections "Tensor parallel vs expert parallel" and "Routing imbalance"):
//   router partial GEMM -> fused partial-sum + softmax top-k selection
//   -> per-block expert histogram -> one-block scan (counts, offsets, GEMM
//   tile list, virtual-EP send counts) -> stable scatter (row_of, perm)
//   -> row gather into the expert-major buffer ... expert FFNs ...
//   -> gate-weighted combine.
#include "moe_kernels.cuh"

namespace moe {

// ============================================================== router GEMM
// logit_part[s][t][e] = sum over the s-th K slice of x[t,i] * w_g[i,e].
// Block: 16 tokens x 32 experts, 256 threads; thread = (2 tokens, 1 expert).
constexpr int kRtT = 16, kRtE = 32, kRtK = 64;

__global__ void __launch_bounds__(256) k_router_partial(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ w_g, int T,
    int d, int E, int k_per_split, float* __restrict__ part) {
  __shared__ float xs[kRtT][kRtK + 1];
  __shared__ float ws[kRtK][kRtE];
  const int t0 = blockIdx.x * kRtT;
  const int e0 = blockIdx.y * kRtE;
  const int split = blockIdx.z;
  const int kbeg = split * k_per_split;
  const int kend = min(d, kbeg + k_per_split);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // ty in 0..7
  float acc0 = 0.f, acc1 = 0.f;
  for (int kc = kbeg; kc < kend; kc += kRtK) {
    // x tile: 16 x 64 bf16
    for (int i = threadIdx.x; i < kRtT * kRtK; i += 256) {
      int r = i / kRtK, c = i % kRtK;
      int t = t0 + r;
      xs[r][c] = (t < T) ? __bfloat162float(x[(size_t)t * d + kc + c]) : 0.f;
    }
    // w tile: 64 x 32 fp32
    for (int i = threadIdx.x; i < kRtK * kRtE; i += 256) {
      int r = i / kRtE, c = i % kRtE;
      int e = e0 + c;
      ws[r][c] = (e < E) ? w_g[(size_t)(kc + r) * E + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 16
    for (int kk = 0; kk < kRtK; ++kk) {
      const float wv = ws[kk][tx];
      acc0 = fmaf(xs[2 * ty][kk], wv, acc0);
      acc1 = fmaf(xs[2 * ty + 1][kk], wv, acc1);
    }
    __syncthreads();
  }
  const int e = e0 + tx;
  if (e < E) {
    const int ta = t0 + 2 * ty, tb = ta + 1;
    float* base = part + (size_t)split * T * E;
    if (ta < T) base[(size_t)ta * E + e] = acc0;
    if (tb < T) base[(size_t)tb * E + e] = acc1;
  }
}

// logits[t,e] = sum_s part[s][t][e] (+ bias[e]), fixed order s = 0..S-1.
__global__ void k_router_finish(const float* __restrict__ part, int S,
                                const float* __restrict__ bias, int T, int E,
                                float* __restrict__ logits) {
  const size_t n = (size_t)T * E;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float v = part[i];
    for (int s = 1; s < S; ++s) v += part[(size_t)s * n + i];
    if (bias) v += bias[i % E];
    logits[i] = v;
  }
}

// ============================================================== top-k
// One warp per token.  Lane l holds logits l, l+32, ... .  k rounds of a
// warp-wide arg-max under the order (value desc, index asc) pick the slots in
// order; the winner of round j is kept by lane j.  Gates are the softmax over
// the k selected logits (equal to the full softmax renormalised over them).
template <int VPL>
__global__ void __launch_bounds__(256) k_topk(
    const float* __restrict__ part, int S, const float* __restrict__ bias,
    int T, int E, int k, float* __restrict__ logits_out, int* __restrict__ idx,
    float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const size_t n = (size_t)T * E;
  float v[VPL];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    float s = 0.f;
    if (e < E) {
      const size_t o = (size_t)t * E + e;
      s = part[o];
      for (int sp = 1; sp < S; ++sp) s += part[(size_t)sp * n + o];
      if (bias) s += bias[e];
      if (logits_out) logits_out[o] = s;
    } else {
      taken |= 1u << i;  // not a candidate
    }
    v[i] = s;
  }
  float my_v = 0.f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = 0.f;
    int be = INT_MAX;  // INT_MAX = no candidate
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (taken & (1u << i)) continue;
      const int e = lane + 32 * i;
      if (be == INT_MAX || v[i] > bv) {  // ascending e: equal keeps lower index
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      const bool take =
          oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be));
      if (take) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      my_v = bv;
      my_e = be;
    }
  }
  const float top = __shfl_sync(0xffffffffu, my_v, 0);
  float ex = (lane < k) ? expf(my_v - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_e;
    w[(size_t)t * k + lane] = ex / sum;
  }
}

// ============================================================== histogram
// blockhist[b][e] = rows of expert e among the tokens of block b.
// blocksend[b][s][r] = rows of those tokens with source rank s going to rank r.
__global__ void __launch_bounds__(kTokensPerRouteBlock) k_hist(
    const int* __restrict__ idx, int T, int E, int k, int R, int src_chunk,
    int* __restrict__ blockhist, int* __restrict__ blocksend, int* err) {
  extern __shared__ int sm[];
  int* hist = sm;            // [E]
  int* send = sm + E;        // [R*R] when R > 1
  const int RR = R > 1 ? R * R : 0;
  for (int i = threadIdx.x; i < E + RR; i += blockDim.x) sm[i] = 0;
  __syncthreads();
  const int t = blockIdx.x * kTokensPerRouteBlock + threadIdx.x;
  if (t < T) {
    const int per = R > 1 ? E / R : 1;
    const int src = R > 1 ? t / src_chunk : 0;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      bool ok = (e >= 0 && e < E);
      for (int j2 = 0; j2 < j && ok; ++j2) ok = idx[(size_t)t * k + j2] != e;
      if (!ok) {
        record_error(err, MOE_ERR_DEVICE_CHECK, 1);
        continue;
      }
      atomicAdd(&hist[e], 1);
      if (R > 1) atomicAdd(&send[src * R + e / per], 1);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    blockhist[(size_t)blockIdx.x * E + i] = hist[i];
  for (int i = threadIdx.x; i < RR; i += blockDim.x)
    blocksend[(size_t)blockIdx.x * RR + i] = send[i];
}

// Exclusive scan over a 1024-thread block; returns the exclusive prefix and
// writes the block total to *total.
__device__ int block_exclusive_scan_1024(int v, int* scratch /*[32]*/, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) scratch[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    int s = scratch[lane];
    int si = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, si, off);
      if (lane >= off) si += o;
    }
    scratch[lane] = si - s;  // exclusive warp offsets
    if (lane == 31) *total = si;
  }
  __syncthreads();
  const int r = scratch[wid] + inc - v;
  __syncthreads();
  return r;
}

// ============================================================== scan
// One block of 1024 threads.  counts, offsets, per-block bases, the GEMM
// tile list (one entry per 128 rows of an expert) and the virtual-EP layout.
__global__ void __launch_bounds__(1024) k_scan(
    const int* __restrict__ blockhist, int nblocks, int E, int R,
    const int* __restrict__ blocksend, int* __restrict__ blockbase,
    int* __restrict__ counts, int* __restrict__ offsets, int* __restrict__ tiles,
    int* __restrict__ send, int* __restrict__ rank_off) {
  __shared__ int scratch[32];
  __shared__ int total;
  const int e = threadIdx.x;  // E <= 1024
  int c = 0;
  if (e < E) {
    for (int b = 0; b < nblocks; ++b) {
      const int h = blockhist[(size_t)b * E + e];
      blockbase[(size_t)b * E + e] = c;
      c += h;
    }
  }
  const int off = block_exclusive_scan_1024(e < E ? c : 0, scratch, &total);
  const int P = total;
  if (e < E) {
    counts[e] = c;
    offsets[e] = off;
    for (int b = 0; b < nblocks; ++b) blockbase[(size_t)b * E + e] += off;
  }
  if (e == 0) offsets[E] = P;
  // GEMM tiles: (row0, row_end, expert) per 128-row tile of each expert.
  const int nt = (e < E) ? (c + kGemmBM - 1) / kGemmBM : 0;
  const int tb = block_exclusive_scan_1024(nt, scratch, &total);
  if (e == 0) tiles[0] = total;
  int* tl = tiles + 4;
  for (int i = 0; i < nt; ++i) {
    tl[3 * (tb + i) + 0] = off + i * kGemmBM;
    tl[3 * (tb + i) + 1] = off + c;
    tl[3 * (tb + i) + 2] = e;
  }
  if (R > 1) {
    for (int i = threadIdx.x; i < R * R; i += blockDim.x) {
      int s = 0;
      for (int b = 0; b < nblocks; ++b) s += blocksend[(size_t)b * R * R + i];
      send[i] = s;
    }
    __syncthreads();
    const int per = E / R;
    // offsets[] written above by other threads; re-read after the barrier.
    if (threadIdx.x <= R) rank_off[threadIdx.x] = (threadIdx.x == R) ? P : offsets[threadIdx.x * per];
  }
}

// Tile list from caller-provided offsets (moe_ffn); checks the offsets.
__global__ void __launch_bounds__(1024) k_tiles_from_offsets(
    const int* __restrict__ offsets, int E, int P, int* __restrict__ tiles, int* err) {
  __shared__ int scratch[32];
  __shared__ int total;
  const int e = threadIdx.x;
  int a = 0, c = 0;
  if (e < E) {
    a = offsets[e];
    const int b = offsets[e + 1];
    c = b - a;
    if (c < 0 || a < 0 || b > P || (e == 0 && a != 0) || (e == E - 1 && b != P)) {
      record_error(err, MOE_ERR_DEVICE_CHECK, 2);
      c = 0;
    }
  }
  const int nt = (c + kGemmBM - 1) / kGemmBM;
  const int tb = block_exclusive_scan_1024(nt, scratch, &total);
  if (e == 0) tiles[0] = total;
  int* tl = tiles + 4;
  for (int i = 0; i < nt; ++i) {
    tl[3 * (tb + i) + 0] = a + i * kGemmBM;
    tl[3 * (tb + i) + 1] = a + c;
    tl[3 * (tb + i) + 2] = e;
  }
}

// ============================================================== scatter
// Stable counting-sort placement: row(t,j) = blockbase[b][e] + rows of e from
// earlier warps of the block + rows of e from lower lanes of this warp.
__global__ void __launch_bounds__(kTokensPerRouteBlock) k_scatter(
    const int* __restrict__ idx, int T, int E, int k,
    const int* __restrict__ blockbase, int* __restrict__ row_of,
    int* __restrict__ perm) {
  extern __shared__ uint32_t masks[];  // [8][E]
  constexpr int W = kTokensPerRouteBlock / 32;
  for (int i = threadIdx.x; i < W * E; i += blockDim.x) masks[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int t = blockIdx.x * kTokensPerRouteBlock + threadIdx.x;
  const bool valid = t < T;
  if (valid) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) atomicOr(&masks[wid * E + e], 1u << lane);
    }
  }
  __syncthreads();
  if (valid) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) continue;  // recorded by k_hist
      int r = blockbase[(size_t)blockIdx.x * E + e];
      for (int w2 = 0; w2 < wid; ++w2) r += __popc(masks[w2 * E + e]);
      r += __popc(masks[wid * E + e] & lt);
      row_of[(size_t)t * k + j] = r;
      perm[r] = t;
    }
  }
}

// ============================================================== gather
// x_perm[row] = x[perm[row]]; one warp per row, 16-byte vectors.  A token
// index outside [0, T) (left by a rejected expert id) is skipped and recorded.
__global__ void __launch_bounds__(256) k_gather_rows(
    const __nv_bfloat16* __restrict__ x, const int* __restrict__ perm, long long P,
    int T, int d, __nv_bfloat16* __restrict__ x_perm, int* err) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= P) return;
  const int lane = threadIdx.x & 31;
  const int t = perm[row];
  if (t < 0 || t >= T) {
    if (lane == 0) record_error(err, MOE_ERR_DEVICE_CHECK, 3);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)row * d);
  const int nv = d / 8;
  for (int c = lane; c < nv; c += 32) dst[c] = __ldg(src + c);
}

// ============================================================== combine
// y[t] = sum_j w[t,j] * z[row_of[t,j]] in fp32, slot order; one warp per token.
// A row index outside [0, T*k) contributes nothing (never dereferenced).
__global__ void __launch_bounds__(256) k_combine(
    const __nv_bfloat16* __restrict__ z, const int* __restrict__ row_of,
    const float* __restrict__ w, int T, int d, int k,
    __nv_bfloat16* __restrict__ y) {
  const long long P = (long long)T * k;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int c = lane; c < nv; c += 32) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int r = row_of[(size_t)t * k + j];
      if (r < 0 || r >= P) continue;
      const float wj = w[(size_t)t * k + j];
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(z + (size_t)r * d) + c);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = __bfloat1622float2(p[i]);
        acc[2 * i] = fmaf(wj, f2.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj, f2.y, acc[2 * i + 1]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4*>(y + (size_t)t * d)[c] = o;
  }
}

// ============================================================== self-test
// Waits on an mbarrier that nothing ever arrives on, through the same bounded
// wait the GEMM pipeline uses, with a caller-chosen limit: the wait must give
// up and the kernel must record MOE_ERR_TIMEOUT and return.
__global__ void k_selftest_bounded_wait(unsigned long long limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns);
  if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) record_error(err, MOE_ERR_TIMEOUT, 20);
}

cudaError_t launch_selftest_bounded_wait(unsigned long long limit_ns, int* err,
                                         cudaStream_t st) {
  k_selftest_bounded_wait<<<1, 32, 0, st>>>(limit_ns, err);
  return cudaGetLastError();
}

// ============================================================== launchers
cudaError_t launch_router_partial(const __nv_bfloat16* x, const float* w_g,
                                  const moe_shape& s, int split, float* part,
                                  cudaStream_t st) {
  const int kchunks = s.d / kRtK;
  const int per = (kchunks + split - 1) / split;
  dim3 grid((s.T + kRtT - 1) / kRtT, (s.E + kRtE - 1) / kRtE, split);
  k_router_partial<<<grid, 256, 0, st>>>(x, w_g, s.T, s.d, s.E, per * kRtK, part);
  return cudaGetLastError();
}

cudaError_t launch_router_finish(const float* part, int split, const float* bias,
                                 const moe_shape& s, float* logits, cudaStream_t st) {
  const long long n = (long long)s.T * s.E;
  const int blocks = (int)std::min<long long>((n + 255) / 256, 4096);
  k_router_finish<<<blocks, 256, 0, st>>>(part, split, bias, s.T, s.E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* part, int split, const float* bias,
                        const moe_shape& s, float* logits_out, int* idx, float* w,
                        cudaStream_t st) {
  const int blocks = (s.T + 7) / 8;
  const int vpl = (s.E + 31) / 32;
#define MOE_TOPK_CASE(V)                                                     \
  case V:                                                                    \
    k_topk<V><<<blocks, 256, 0, st>>>(part, split, bias, s.T, s.E, s.k,      \
                                      logits_out, idx, w);                   \
    break;
  if (vpl <= 4) {
    switch (vpl) { MOE_TOPK_CASE(1) MOE_TOPK_CASE(2) MOE_TOPK_CASE(3) MOE_TOPK_CASE(4) }
  } else if (vpl <= 8) {
    k_topk<8><<<blocks, 256, 0, st>>>(part, split, bias, s.T, s.E, s.k, logits_out, idx, w);
  } else if (vpl <= 16) {
    k_topk<16><<<blocks, 256, 0, st>>>(part, split, bias, s.T, s.E, s.k, logits_out, idx, w);
  } else {
    k_topk<32><<<blocks, 256, 0, st>>>(part, split, bias, s.T, s.E, s.k, logits_out, idx, w);
  }
#undef MOE_TOPK_CASE
  return cudaGetLastError();
}

cudaError_t launch_route_tables(const int* idx, const moe_shape& s, const WsLayout& L,
                                char* ws, int* counts, int* offsets, int* row_of,
                                int* perm, int* send, int* rank_off, cudaStream_t st) {
  int* err = reinterpret_cast<int*>(ws + L.err);
  int* blockhist = reinterpret_cast<int*>(ws + L.blockhist);
  int* blockbase = reinterpret_cast<int*>(ws + L.blockbase);
  int* blocksend = reinterpret_cast<int*>(ws + L.blocksend);
  int* tiles = reinterpret_cast<int*>(ws + L.tiles);
  const int R = s.R > 1 ? s.R : 0;
  const int chunk = R ? (s.T + R - 1) / R : 1;
  const size_t hist_smem = sizeof(int) * (s.E + (R ? R * R : 0));
  k_hist<<<L.nblocks, kTokensPerRouteBlock, hist_smem, st>>>(
      idx, s.T, s.E, s.k, R, chunk, blockhist, blocksend, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_scan<<<1, 1024, 0, st>>>(blockhist, L.nblocks, s.E, R, blocksend, blockbase,
                             counts, offsets, tiles, send, rank_off);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t scat_smem = sizeof(uint32_t) * (kTokensPerRouteBlock / 32) * s.E;
  k_scatter<<<L.nblocks, kTokensPerRouteBlock, scat_smem, st>>>(
      idx, s.T, s.E, s.k, blockbase, row_of, perm);
  return cudaGetLastError();
}

cudaError_t launch_tiles_from_offsets(const int* offsets, const moe_shape& s,
                                      int* tiles, int* err, cudaStream_t st) {
  k_tiles_from_offsets<<<1, 1024, 0, st>>>(offsets, s.E, (int)((long long)s.T * s.k),
                                           tiles, err);
  return cudaGetLastError();
}

cudaError_t launch_gather(const __nv_bfloat16* x, const int* perm, long long P, int T,
                          int d, __nv_bfloat16* x_perm, int* err, cudaStream_t st) {
  if (P == 0) return cudaSuccess;
  const long long blocks = (P + 7) / 8;
  k_gather_rows<<<(unsigned)blocks, 256, 0, st>>>(x, perm, P, T, d, x_perm, err);
  return cudaGetLastError();
}

cudaError_t launch_combine(const __nv_bfloat16* z, const int* row_of, const float* w,
                           const moe_shape& s, __nv_bfloat16* y, cudaStream_t st) {
  const int blocks = (s.T + 7) / 8;
  k_combine<<<blocks, 256, 0, st>>>(z, row_of, w, s.T, s.d, s.k, y);
  return cudaGetLastError();
}

}  // namespace moe
