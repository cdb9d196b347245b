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
#include <cooperative_groups.h>

#include "moe_kernels.cuh"

namespace moe {

// ============================================================== router GEMM
// logits[t,e] = sum_i x[t,i] * w_g[i,e] (+ bias[e]), fp32.
// A thread-block cluster of CS CTAs owns a 32-token x RE-expert tile (RE = 32
// or 64); CTA r of the cluster accumulates the K slice [r*d/CS, (r+1)*d/CS)
// in fp32 FMA order, the partial tiles meet in distributed shared memory,
// and CTA r then sums output slice r over the CS partials in rank order
// 0..CS-1.  Each logit's sequence of operations depends on d and CS only (not
// on RE or the K chunking), so every call with the same d gives the same
// bits, and nothing leaves the SMs but the logits.
constexpr int kRtT = 32;

// Chunk loads of the router: every thread issues all of its 16-byte loads for
// a KC-deep K chunk before using any of them (W: KC x RE fp32 = KC*RE/1024
// float4 per thread; x: 32 x KC bf16 = KC/64 uint4 per thread), so a chunk
// costs one memory latency, and the next chunk's loads are in flight while
// this one is multiplied.
template <int RE, int KC>
struct RouterRegs {
  static constexpr int NW = KC * RE / 1024, NX = KC / 64;
  float4 w[NW];
  uint4 x[NX];
};

template <int RE, int KC>
__device__ __forceinline__ void router_load(RouterRegs<RE, KC>& r,
                                            const __nv_bfloat16* __restrict__ x,
                                            const float* __restrict__ w_g, int T, int d, int E,
                                            int t0, int e0, int kc, int chunk) {
  const int vpr = chunk / 8;  // 16-byte x vectors per token row
#pragma unroll
  for (int u = 0; u < RouterRegs<RE, KC>::NX; ++u) {
    const int v = threadIdx.x + 256 * u;
    r.x[u] = make_uint4(0, 0, 0, 0);
    if (v < kRtT * vpr) {
      const int row = v / vpr, c8 = (v - row * vpr) * 8;
      if (t0 + row < T)
        r.x[u] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + row) * d + kc + c8));
    }
  }
#pragma unroll
  for (int u = 0; u < RouterRegs<RE, KC>::NW; ++u) {
    const int v = threadIdx.x + 256 * u;  // RE/4 float4 per K row
    const int row = v / (RE / 4), c4 = (v % (RE / 4)) * 4;
    r.w[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < chunk) {
      const int e = e0 + c4;
      const float* src = w_g + (size_t)(kc + row) * E + e;
      if ((E & 3) == 0 && e + 3 < E) {
        r.w[u] = __ldg(reinterpret_cast<const float4*>(src));
      } else {
        float t4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) t4[q] = (e + q < E) ? __ldg(src + q) : 0.f;
        r.w[u] = make_float4(t4[0], t4[1], t4[2], t4[3]);
      }
    }
  }
}

template <int RE, int KC>
__device__ __forceinline__ void router_store(const RouterRegs<RE, KC>& r, float (*xs)[KC],
                                             float (*ws)[RE], int chunk) {
  const int vpr = chunk / 8;
#pragma unroll
  for (int u = 0; u < RouterRegs<RE, KC>::NX; ++u) {
    const int v = threadIdx.x + 256 * u;
    if (v < kRtT * vpr) {
      const int row = v / vpr, c8 = (v - row * vpr) * 8;
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.x[u]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        xs[row][c8 + 2 * i] = f.x;
        xs[row][c8 + 2 * i + 1] = f.y;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < RouterRegs<RE, KC>::NW; ++u) {
    const int v = threadIdx.x + 256 * u;
    const int row = v / (RE / 4), c4 = (v % (RE / 4)) * 4;
    if (row < chunk) *reinterpret_cast<float4*>(&ws[row][c4]) = r.w[u];
  }
}

// RE = 32 with 128-deep K chunks, or RE = 64 (half the CTAs: large grids
// fit fewer waves) with 64-deep ones; thread (ty, tx) accumulates tokens
// ty + 8i and experts tx + 32ee of the tile.
template <int RE, int KC>
__global__ void __launch_bounds__(256) k_router_cluster(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ w_g,
    const float* __restrict__ bias, int T, int d, int E, float* __restrict__ logits) {
  pdl_trigger();
  pdl_wait();
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  constexpr int NE = RE / 32;
  const int CS = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  __shared__ __align__(16) float xs[kRtT][KC];
  __shared__ __align__(16) float ws[KC][RE];
  __shared__ float part[kRtT * RE];
  const int e0 = (blockIdx.x / CS) * RE;
  const int t0 = blockIdx.y * kRtT;
  const int kslice = d / CS;
  const int kbeg = rank * kslice, kend = kbeg + kslice;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  float acc[4][NE];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int ee = 0; ee < NE; ++ee) acc[i][ee] = 0.f;
  // warp ty's token rows ty + 8i hold tokens for i < ni; with one such row
  // (at most 8 tokens in the tile) the warp multiplies only that row, and a
  // warp with none multiplies nothing (the other rows' sums stay zero and are
  // not stored)
  const int ni = min(4, max(0, (min(kRtT, T - t0) - ty + 7) / 8));
  RouterRegs<RE, KC> regs;
  router_load<RE, KC>(regs, x, w_g, T, d, E, t0, e0, kbeg, min(KC, kend - kbeg));
  for (int kc = kbeg; kc < kend; kc += KC) {
    const int chunk = min(KC, kend - kc);  // a multiple of 64
    router_store<RE, KC>(regs, xs, ws, chunk);
    __syncthreads();
    if (kc + KC < kend)
      router_load<RE, KC>(regs, x, w_g, T, d, E, t0, e0, kc + KC, min(KC, kend - kc - KC));
    if (ni >= 2) {
      for (int kk = 0; kk < chunk; kk += 4) {  // same FMA order as one kk at a time
        float4 xv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          xv[i] = *reinterpret_cast<const float4*>(&xs[ty + 8 * i][kk]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int ee = 0; ee < NE; ++ee) {
            const float wv = ws[kk + j][tx + 32 * ee];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float xe = j == 0 ? xv[i].x : j == 1 ? xv[i].y : j == 2 ? xv[i].z : xv[i].w;
              acc[i][ee] = fmaf(xe, wv, acc[i][ee]);
            }
          }
        }
      }
    } else if (ni == 1) {  // at most 8 tokens in the tile: warp ty's one row
      for (int kk = 0; kk < chunk; kk += 4) {
        const float4 xv = *reinterpret_cast<const float4*>(&xs[ty][kk]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float xe = j == 0 ? xv.x : j == 1 ? xv.y : j == 2 ? xv.z : xv.w;
#pragma unroll
          for (int ee = 0; ee < NE; ++ee)
            acc[0][ee] = fmaf(xe, ws[kk + j][tx + 32 * ee], acc[0][ee]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int ee = 0; ee < NE; ++ee) part[(ty + 8 * i) * RE + tx + 32 * ee] = acc[i][ee];
  cl.sync();
  const int per = (kRtT * RE) / CS;
  for (int o = rank * per + threadIdx.x; o < (rank + 1) * per; o += 256) {
    // all CS remote loads in flight at once, then the sum in rank order
    float pv[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) pv[r] = r < CS ? *cl.map_shared_rank(&part[o], r) : 0.f;
    float v = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < CS) v += pv[r];
    const int t = t0 + o / RE, e = e0 + (o % RE);
    if (t < T && e < E) logits[(size_t)t * E + e] = bias ? v + bias[e] : v;
  }
  cl.sync();  // partial tiles stay alive until every CTA has read them
}

// ============================================================== top-k
// One warp per token.  Lane l holds logits l, l+32, ... .  k rounds of a
// warp-wide arg-max under the order (value desc, index asc) pick the slots in
// order; the winner of round j is kept by lane j.  Gates are the softmax over
// the k selected logits (equal to the full softmax renormalised over them).
// Shared by k_topk and the fused small-batch routing kernel so both take the
// same decisions.
// Order-preserving 32-bit key of a float: a < b  <=>  key(a) < key(b).
// -0.0 is first turned into +0.0 so the two zeros get one key and tie.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

template <int VPL>
__device__ __forceinline__ void warp_topk_scan(const float* __restrict__ row, int E, int k,
                                          int lane, int* __restrict__ idx_row,
                                          float* __restrict__ w_row) {
  uint32_t key[VPL];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < E) key[i] = order_key(row[e]);
    else taken |= 1u << i;  // not a candidate
  }
  uint32_t my_key = 0;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    // this lane's best remaining candidate: largest key, lowest index
    uint32_t bk = 0;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (taken & (1u << i)) continue;
      if (bi < 0 || key[i] > bk) {  // ascending index: an equal key keeps the lower index
        bk = key[i];
        bi = i;
      }
    }
    // Lanes with no candidate left take part with key 0 and index 0xffffffff;
    // real keys are never 0 (0 would be the key of a negative NaN pattern).
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const uint32_t cand = (bi >= 0 && bk == wk) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
    const uint32_t we = __reduce_min_sync(0xffffffffu, cand);
    if ((int)(we & 31) == lane) taken |= 1u << (we >> 5);
    if (lane == j) {
      my_key = wk;
      my_e = (int)we;
    }
  }
  const float my_v = key_value(my_key);
  const float top = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = (lane < k) ? expf(my_v - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    idx_row[lane] = my_e;
    w_row[lane] = ex / sum;
  }
}

// Compare-exchange of two (key, slot) candidates so that position a ends up
// with the one that ranks first: larger key, or equal key and lower slot
// (the slot order within a lane is the expert-index order).
__device__ __forceinline__ void cmpx(uint32_t& ka, int& ia, uint32_t& kb, int& ib) {
  const bool keep = ka > kb || (ka == kb && ia < ib);
  if (!keep) {
    const uint32_t tk = ka;
    ka = kb;
    kb = tk;
    const int ti = ia;
    ia = ib;
    ib = ti;
  }
}

template <int VPL>
__device__ __forceinline__ void sort_candidates(uint32_t* k, int* i) {
  if (VPL == 2) {
    cmpx(k[0], i[0], k[1], i[1]);
  } else if (VPL == 4) {
    cmpx(k[0], i[0], k[1], i[1]);
    cmpx(k[2], i[2], k[3], i[3]);
    cmpx(k[0], i[0], k[2], i[2]);
    cmpx(k[1], i[1], k[3], i[3]);
    cmpx(k[1], i[1], k[2], i[2]);
  } else if (VPL == 8) {
    // odd-even merge sorting network, 19 comparators
    const int net[19][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}, {0, 2}, {1, 3}, {4, 6},
                            {5, 7}, {1, 2}, {5, 6}, {0, 4}, {3, 7}, {1, 5}, {2, 6},
                            {1, 4}, {3, 6}, {2, 4}, {3, 5}, {3, 4}};
#pragma unroll
    for (int c = 0; c < 19; ++c) cmpx(k[net[c][0]], i[net[c][0]], k[net[c][1]], i[net[c][1]]);
  }
}

// Up to 256 experts (at most 8 per lane): each lane sorts its candidates
// once, then every round compares only the lanes' heads -- one redux.sync for
// the largest key, one for the lowest index holding it -- and the winning lane
// drops its head.  A lane's head is its best candidate and, among equal keys,
// its lowest index, so the round picks the same expert as the rank order.
template <int V>
__device__ __forceinline__ void topk_load(const float* __restrict__ row, int E, int lane,
                                          uint32_t* key, int* slot) {
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? order_key(row[e]) : 0u;  // 0: below every finite key
    slot[i] = i;
  }
}

// One selection round: the winner's key and expert, and the winning lane
// drops its head.
template <int V>
__device__ __forceinline__ void topk_round(uint32_t* key, int* slot, int lane, uint32_t& wk,
                                           uint32_t& we) {
  wk = __reduce_max_sync(0xffffffffu, key[0]);
  const uint32_t cand = (key[0] == wk) ? (uint32_t)(lane + 32 * slot[0]) : 0xffffffffu;
  we = __reduce_min_sync(0xffffffffu, cand);
  if ((int)(we & 31) == lane) {
#pragma unroll
    for (int i = 0; i + 1 < V; ++i) {
      key[i] = key[i + 1];
      slot[i] = slot[i + 1];
    }
    key[V - 1] = 0u;
  }
}

// Gate of slot `lane` (< k): softmax over the k selected logits.
__device__ __forceinline__ float topk_gate(uint32_t my_key, int k, int lane) {
  const float my_v = key_value(my_key);
  const float top = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = (lane < k) ? expf(my_v - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  return ex / sum;
}

// idx_s_row (optional): a shared-memory copy of the selected ids.
template <int VPL>
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, int E, int k, int lane,
                                          int* __restrict__ idx_row, float* __restrict__ w_row,
                                          int* idx_s_row = nullptr) {
  if (VPL > 8) {
    warp_topk_scan<VPL>(row, E, k, lane, idx_row, w_row);
    if (idx_s_row && lane < k) idx_s_row[lane] = idx_row[lane];  // this lane's own store
    return;
  }
  constexpr int V = VPL > 8 ? 8 : VPL;
  uint32_t key[V];
  int slot[V];
  topk_load<V>(row, E, lane, key, slot);
  sort_candidates<V>(key, slot);
  uint32_t my_key = 0;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t wk, we;
    topk_round<V>(key, slot, lane, wk, we);
    if (lane == j) {
      my_key = wk;
      my_e = (int)we;
    }
  }
  const float g = topk_gate(my_key, k, lane);
  if (lane < k) {
    idx_row[lane] = my_e;
    w_row[lane] = g;
    if (idx_s_row) idx_s_row[lane] = my_e;
  }
}

template <int VPL>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits, int T, int E,
                                              int k, int* __restrict__ idx,
                                              float* __restrict__ w) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  warp_topk<VPL>(logits + (size_t)t * E, E, k, threadIdx.x & 31, idx + (size_t)t * k,
                 w + (size_t)t * k);
}

// ============================================================== histogram
// blockhist[b][e] = rows of expert e among the tokens of block b.
// blocksend[b][s][r] = rows of those tokens with source rank s going to rank r.
__global__ void __launch_bounds__(kTokensPerRouteBlock) k_hist(
    const int* __restrict__ idx, int T, int E, int k, int R, int src_chunk,
    int* __restrict__ blockhist, int* __restrict__ blocksend, int* err) {
  pdl_trigger();
  pdl_wait();
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

// The expert GEMMs' work lists (layout in tile_list_ints): every thread of a
// 1024-thread block calls this; thread e < E passes expert e's row count c
// and first row off.  pair: tile pairs for CTA-pair GEMMs (see
// pair_row_tiles).
__device__ void write_work_lists(int e, int E, int c, int off, int* tiles, int* scratch,
                                 int* total, bool pair, int max_mtiles) {
  int* ready = ready_counters(tiles, max_mtiles, E);
  for (int i = threadIdx.x; i < ready_ints(max_mtiles, E); i += blockDim.x) ready[i] = 0;
  const int nt = (e < E) ? (c + kGemmBM - 1) / kGemmBM : 0;
  const int nrow = pair ? pair_row_tiles(nt) : nt;  // tiles in the row-tile list
  const int left = (pair && nt == 1) ? 1 : 0;       // a lone tile: leftover list
  const int tb = block_exclusive_scan_1024(nrow, scratch, total);
  if (threadIdx.x == 0) tiles[0] = *total;
  int* rt = row_tile_entries(tiles, E);
  for (int i = 0; i < nrow; ++i) {
    rt[3 * (tb + i) + 0] = off + i * kGemmBM;
    rt[3 * (tb + i) + 1] = off + c;
    rt[3 * (tb + i) + 2] = e;
  }
  const int touched = (e < E && c > 0) ? 1 : 0;
  const int eb = block_exclusive_scan_1024(touched, scratch, total);
  if (threadIdx.x == 0) tiles[1] = *total;
  if (touched) {
    int* et = expert_entries(tiles);
    et[3 * eb + 0] = off;
    et[3 * eb + 1] = off + c;
    et[3 * eb + 2] = e;
  }
  const int lb = block_exclusive_scan_1024(left, scratch, total);
  if (threadIdx.x == 0) tiles[2] = *total;
  if (left) {
    int* lt = leftover_entries(tiles, E);
    lt[3 * lb + 0] = off;
    lt[3 * lb + 1] = off + c;
    lt[3 * lb + 2] = e;
  }
}

// ============================================================== scan
// One block of 1024 threads.  counts, offsets, per-block bases, the GEMM
// tile list (one entry per 128 rows of an expert) and the virtual-EP layout.
__global__ void __launch_bounds__(1024) k_scan(
    const int* __restrict__ blockhist, int nblocks, int E, int R,
    const int* __restrict__ blocksend, int* __restrict__ blockbase,
    int* __restrict__ counts, int* __restrict__ offsets, int* __restrict__ tiles,
    int* __restrict__ send, int* __restrict__ rank_off, int pair, int max_mtiles) {
  pdl_trigger();
  pdl_wait();
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
  write_work_lists(e, E, c, off, tiles, scratch, &total, pair != 0, max_mtiles);
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
    const int* __restrict__ offsets, int E, int P, int* __restrict__ tiles, int* err,
    int pair) {
  pdl_trigger();
  pdl_wait();
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
  write_work_lists(e, E, c, a, tiles, scratch, &total, pair != 0, max_mtiles_of(P, E));
}

// ============================================================== fused routing, T <= 1024
// Selection and the whole dispatch table for a batch of at most 1024 tokens
// in one launch.  Blocks of 1024 threads each select kFusedSelTokens tokens
// (one warp per token: selection throughput is bounded per SM, so the tokens
// are spread over ceil(T / kFusedSelTokens) SMs); the last block to take a
// ticket (a counter in the workspace's zeroed header, reset by that block)
// then builds the tables: histogram, one block scan of (rows, row tiles,
// touched, leftover) per expert, work lists, virtual-EP counts and the
// stable scatter (one token per thread).  Same results as k_topk + k_hist +
// k_scan + k_scatter.
constexpr int kFusedSmemIdx = 8192;  // T*k up to this keeps the ids in shared memory
constexpr int kFusedSelTokens = 8;   // tokens selected per block

// Exclusive block scan of four ints over 1024 threads (two barriers).
__device__ __forceinline__ int4 block_exclusive_scan4_1024(int4 v, int4* warp_tot, int4* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int4 inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, inc.x, off);
    const int b = __shfl_up_sync(0xffffffffu, inc.y, off);
    const int c = __shfl_up_sync(0xffffffffu, inc.z, off);
    const int d = __shfl_up_sync(0xffffffffu, inc.w, off);
    if (lane >= off) {
      inc.x += a;
      inc.y += b;
      inc.z += c;
      inc.w += d;
    }
  }
  if (lane == 31) warp_tot[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    const int4 t = warp_tot[lane];
    int4 si = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, si.x, off);
      const int b = __shfl_up_sync(0xffffffffu, si.y, off);
      const int c = __shfl_up_sync(0xffffffffu, si.z, off);
      const int d = __shfl_up_sync(0xffffffffu, si.w, off);
      if (lane >= off) {
        si.x += a;
        si.y += b;
        si.z += c;
        si.w += d;
      }
    }
    warp_tot[lane] = make_int4(si.x - t.x, si.y - t.y, si.z - t.z, si.w - t.w);
    if (lane == 31) *total = si;
  }
  __syncthreads();
  const int4 base = warp_tot[wid];
  return make_int4(base.x + inc.x - v.x, base.y + inc.y - v.y, base.z + inc.z - v.z,
                   base.w + inc.w - v.w);
}

template <int VPL>
__global__ void __launch_bounds__(1024) k_route_fused(
    const float* __restrict__ logits, int T, int E, int k, int R, int src_chunk,
    int* __restrict__ idx, float* __restrict__ w, int* __restrict__ counts,
    int* __restrict__ offsets, int* __restrict__ tiles, int* __restrict__ send_out,
    int* __restrict__ rank_off, int* __restrict__ row_of, int* __restrict__ perm, int* err,
    int* ticket, int pair, int max_mtiles) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  int* hist = sm;                                  // [E]
  int* off_s = hist + E;                           // [E]
  int* send = off_s + E;                           // [R*R]
  const int RR = R > 1 ? R * R : 0;
  uint32_t* masks = reinterpret_cast<uint32_t*>(send + RR);  // [32][E]
  int* idx_s = reinterpret_cast<int*>(masks + 32 * E);         // [T*k] when it fits
  __shared__ int4 warp_tot[32];
  __shared__ int4 total;
  __shared__ int is_last;
  const bool ids_in_smem = T * k <= kFusedSmemIdx;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const bool single = gridDim.x == 1;  // one block: no ticket, ids straight to smem
  for (int i = threadIdx.x; i < 2 * E + RR + 32 * E; i += 1024) sm[i] = 0;
  // Selection: block b, warp w < kFusedSelTokens takes token b*kFusedSelTokens + w.
  {
    const int t = blockIdx.x * kFusedSelTokens + wid;
    if (wid < kFusedSelTokens && t < T) {
      warp_topk<VPL>(logits + (size_t)t * E, E, k, lane, idx + (size_t)t * k,
                     w + (size_t)t * k, single && ids_in_smem ? idx_s + t * k : nullptr);
      if (!single) __threadfence();  // this lane's ids and gates before the block's ticket
    }
  }
  __syncthreads();
  if (!single) {
    if (threadIdx.x == 0) {
      __threadfence();
      is_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (!is_last) return;
    // The last block to finish selection builds the tables for the whole batch.
    __threadfence();
    if (threadIdx.x == 0) *ticket = 0;  // ready for the next call
    if (ids_in_smem)
      for (int i = threadIdx.x; i < T * k; i += 1024) idx_s[i] = __ldcg(idx + i);
    __syncthreads();
  }
  const int* ids = ids_in_smem ? idx_s : idx;
  {
    int* ready = ready_counters(tiles, max_mtiles, E);
    for (int i = threadIdx.x; i < ready_ints(max_mtiles, E); i += 1024) ready[i] = 0;
  }
  const int t = threadIdx.x;
  const bool valid = t < T;
  // The ids come from this kernel's own selection: distinct per token by
  // construction, and in range unless a logit is a NaN whose bits sort below
  // every candidate (an out-of-range pick is recorded and skipped).  Bit j of
  // okmask marks slot j as usable.
  uint32_t okmask = 0;
  if (valid) {
    const int per = R > 1 ? E / R : 1;
    const int src = R > 1 ? t / src_chunk : 0;
    for (int j = 0; j < k; ++j) {
      const int e = ids_in_smem ? ids[t * k + j] : __ldcg(ids + t * k + j);
      if (e < 0 || e >= E) {
        record_error(err, MOE_ERR_DEVICE_CHECK, 4);
        continue;
      }
      okmask |= 1u << j;
      atomicAdd(&hist[e], 1);
      atomicOr(&masks[wid * E + e], 1u << lane);
      if (R > 1) atomicAdd(&send[src * R + e / per], 1);
    }
  }
  __syncthreads();
  const int e = threadIdx.x;
  const int c = (e < E) ? hist[e] : 0;
  const int nt = (c + kGemmBM - 1) / kGemmBM;
  // CTA-pair GEMMs: pairs of row tiles; a lone tile goes to the leftover list
  const int nrow = pair ? pair_row_tiles(nt) : nt;
  const int left = (pair && nt == 1) ? 1 : 0;
  const int4 pre =
      block_exclusive_scan4_1024(make_int4(c, nrow, c > 0 ? 1 : 0, left), warp_tot, &total);
  const int4 tot = total;
  if (e < E) {
    counts[e] = c;
    offsets[e] = pre.x;
    off_s[e] = pre.x;
    int* rt = row_tile_entries(tiles, E);
    for (int i = 0; i < nrow; ++i) {
      rt[3 * (pre.y + i) + 0] = pre.x + i * kGemmBM;
      rt[3 * (pre.y + i) + 1] = pre.x + c;
      rt[3 * (pre.y + i) + 2] = e;
    }
    if (c > 0) {
      int* et = expert_entries(tiles);
      et[3 * pre.z + 0] = pre.x;
      et[3 * pre.z + 1] = pre.x + c;
      et[3 * pre.z + 2] = e;
    }
    if (left) {
      int* lt = leftover_entries(tiles, E);
      lt[3 * pre.w + 0] = pre.x;
      lt[3 * pre.w + 1] = pre.x + c;
      lt[3 * pre.w + 2] = e;
    }
  }
  if (threadIdx.x == 0) {
    offsets[E] = tot.x;
    tiles[0] = tot.y;
    tiles[1] = tot.z;
    tiles[2] = tot.w;
  }
  if (R > 1)
    for (int i = threadIdx.x; i < RR; i += 1024) send_out[i] = send[i];
  __syncthreads();  // off_s complete
  if (R > 1 && threadIdx.x <= R)
    rank_off[threadIdx.x] = (threadIdx.x == R) ? tot.x : off_s[threadIdx.x * (E / R)];
  if (valid) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      if (!((okmask >> j) & 1u)) continue;
      const int ej = ids_in_smem ? ids[t * k + j] : __ldcg(ids + t * k + j);
      int r = off_s[ej];
      for (int w2 = 0; w2 < wid; ++w2) r += __popc(masks[w2 * E + ej]);
      r += __popc(masks[wid * E + ej] & lt);
      row_of[(size_t)t * k + j] = r;
      perm[r] = t;
    }
  }
}

// ============================================================== scatter
// Stable counting-sort placement: row(t,j) = blockbase[b][e] + rows of e from
// earlier warps of the block + rows of e from lower lanes of this warp.
__global__ void __launch_bounds__(kTokensPerRouteBlock) k_scatter(
    const int* __restrict__ idx, int T, int E, int k,
    const int* __restrict__ blockbase, int* __restrict__ row_of,
    int* __restrict__ perm) {
  pdl_trigger();
  pdl_wait();
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
  // Lets the expert GEMMs launch only after this wait: they may then read the
  // work lists (written before this kernel) before their own wait.
  pdl_wait();
  pdl_trigger();
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
  // Up to 8 vectors per lane in flight; x_perm is written with streaming
  // stores so it does not push x (read k times) out of L2.
  for (int c0 = 0; c0 < nv; c0 += 256) {
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = c0 + lane + 32 * i;
      if (c < nv) v[i] = __ldg(src + c);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = c0 + lane + 32 * i;
      if (c < nv) __stcs(dst + c, v[i]);
    }
  }
}

// ============================================================== combine
// y[t] = sum_j w[t,j] * z[row_of[t,j]] in fp32, slot order.  One warp per
// (token, 256*V-column chunk): each lane owns V 16-byte vectors (8 columns
// each, 256 columns apart), so a warp reads V*512 contiguous bytes of each of
// the token's k rows with all k*V loads in flight.  A row index outside
// [0, T*k) contributes nothing (never dereferenced).
template <int V>
__global__ void __launch_bounds__(256) k_combine(
    const __nv_bfloat16* __restrict__ z, const int* __restrict__ row_of,
    const float* __restrict__ w, int T, int d, int k, __nv_bfloat16* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const long long P = (long long)T * k;
  const int span = 256 * V;
  const int nchunk = (d + span - 1) / span;
  const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (gw >= (long long)T * nchunk) return;
  const int lane = threadIdx.x & 31;
  const int t = (int)(gw / nchunk);
  const int col0 = (int)(gw - (long long)t * nchunk) * span + lane * 8;
  // lane j < k holds slot j's row and gate; broadcast them with shuffles so
  // the row loads below are all independent.
  int my_r = -1;
  float my_w = 0.f;
  if (lane < k) {
    my_r = __ldg(row_of + (size_t)t * k + lane);
    my_w = __ldg(w + (size_t)t * k + lane);
  }
  float acc[V][8];
#pragma unroll
  for (int v = 0; v < V; ++v)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[v][i] = 0.f;
  for (int j0 = 0; j0 < k; j0 += 8) {
    uint4 val[8][V];
    float wj[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int r = __shfl_sync(0xffffffffu, my_r, (j0 + jj) & 31);
      wj[jj] = __shfl_sync(0xffffffffu, my_w, (j0 + jj) & 31);
      const bool ok = (j0 + jj < k) && r >= 0 && r < P;
      if (!ok) wj[jj] = 0.f;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int col = col0 + 256 * v;
        val[jj][v] = (ok && col < d)
                         ? __ldcs(reinterpret_cast<const uint4*>(z + (size_t)r * d + col))
                         : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      if (j0 + jj >= k) break;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&val[jj][v]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f2 = __bfloat1622float2(p[i]);
          acc[v][2 * i] = fmaf(wj[jj], f2.x, acc[v][2 * i]);
          acc[v][2 * i + 1] = fmaf(wj[jj], f2.y, acc[v][2 * i + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const int col = col0 + 256 * v;
    if (col >= d) continue;
    uint4 o;
    o.x = pack_bf16x2(acc[v][0], acc[v][1]);
    o.y = pack_bf16x2(acc[v][2], acc[v][3]);
    o.z = pack_bf16x2(acc[v][4], acc[v][5]);
    o.w = pack_bf16x2(acc[v][6], acc[v][7]);
    *reinterpret_cast<uint4*>(y + (size_t)t * d + col) = o;
  }
}

// ============================================================== copy
// dst[i] = src[i] for n 16-byte vectors, grid-stride.  It lets the next
// kernel launch at once (that one waits for this one) and waits for a
// previous kernel only before its reads.
__global__ void __launch_bounds__(256) k_copy16(const uint4* __restrict__ src,
                                                uint4* __restrict__ dst, long long n) {
  pdl_trigger();
  pdl_wait();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

cudaError_t launch_copy(void* dst, const void* src, long long bytes, int num_sms,
                        cudaStream_t st) {
  const long long n = bytes / 16;
  if (n == 0) return cudaSuccess;
  long long blocks = (n + 255) / 256;
  if (blocks > 4LL * num_sms) blocks = 4LL * num_sms;
  return launch_kernel(k_copy16, dim3((unsigned)blocks), dim3(256), 0, st, 1,
                       reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), n);
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
// Largest cluster (16 if the device allows non-portable cluster sizes, else
// 8) whose K slices are whole 64-element chunks.
static int router_max_cluster() {
  static int max_cs = 0;
  if (max_cs == 0) {
    max_cs = 8;
    if (cudaFuncSetAttribute(k_router_cluster<32, 128>,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(k_router_cluster<64, 64>,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(256, 1, 1);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_router_cluster<32, 128>, &cfg) == cudaSuccess &&
          n > 0)
        max_cs = 16;
    }
    cudaGetLastError();
  }
  return max_cs;
}

static int router_cluster_size(int d) {
  for (int cs = router_max_cluster(); cs > 1; cs >>= 1)
    if (d % (64 * cs) == 0) return cs;
  return 1;
}

cudaError_t launch_router(const __nv_bfloat16* x, const float* w_g, const float* bias,
                          const moe_shape& s, float* logits, cudaStream_t st) {
  const int cs = router_cluster_size(s.d);
  const unsigned ty = (unsigned)((s.T + kRtT - 1) / kRtT);
  // 64-expert tiles when 32-expert ones would need more than 128 CTAs (a
  // second wave of clusters)
  const long long ctas32 = (long long)cs * ((s.E + 31) / 32) * ty;
  if (ctas32 > 128 && s.E > 32)
    return launch_kernel(k_router_cluster<64, 64>, dim3((unsigned)(cs * ((s.E + 63) / 64)), ty, 1),
                         dim3(256), 0, st, cs, x, w_g, bias, s.T, s.d, s.E, logits);
  return launch_kernel(k_router_cluster<32, 128>, dim3((unsigned)(cs * ((s.E + 31) / 32)), ty, 1),
                       dim3(256), 0, st, cs, x, w_g, bias, s.T, s.d, s.E, logits);
}

#define MOE_VPL_DISPATCH(VPL_VAR, CALL) \
  do {                                  \
    if ((VPL_VAR) <= 1) { CALL(1); }    \
    else if ((VPL_VAR) <= 2) { CALL(2); } \
    else if ((VPL_VAR) <= 4) { CALL(4); } \
    else if ((VPL_VAR) <= 8) { CALL(8); } \
    else if ((VPL_VAR) <= 16) { CALL(16); } \
    else { CALL(32); }                  \
  } while (0)

cudaError_t launch_topk(const float* logits, const moe_shape& s, int* idx, float* w,
                        cudaStream_t st) {
  const int blocks = (s.T + 7) / 8;
  const int vpl = (s.E + 31) / 32;
#define MOE_TOPK_CALL(V) \
  return launch_kernel(k_topk<V>, dim3(blocks), dim3(256), 0, st, 1, logits, s.T, s.E, s.k, idx, w)
  MOE_VPL_DISPATCH(vpl, MOE_TOPK_CALL);
#undef MOE_TOPK_CALL
}

template <int VPL>
static cudaError_t route_fused_t(const float* logits, const moe_shape& s, int R, int chunk,
                                 size_t smem, int* idx, float* w, int* counts, int* offsets,
                                 int* tiles, int* send, int* rank_off, int* row_of, int* perm,
                                 int* err, int pair, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_route_fused<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(4 * (2 * kMaxE + kMaxR * kMaxR + 32 * kMaxE +
                                                    kFusedSmemIdx)));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const unsigned blocks = (unsigned)((s.T + kFusedSelTokens - 1) / kFusedSelTokens);
  return launch_kernel(k_route_fused<VPL>, dim3(blocks), dim3(1024), smem, st, 1, logits, s.T,
                       s.E, s.k, R, chunk, idx, w, counts, offsets, tiles, send, rank_off, row_of,
                       perm, err, err + kRouteTicket, pair,
                       max_mtiles_of((long long)s.T * s.k, s.E));
}

cudaError_t launch_route_fused(const float* logits, const moe_shape& s, int* idx, float* w,
                               int* counts, int* offsets, int* tiles, int* send,
                               int* rank_off, int* row_of, int* perm, int* err,
                               cudaStream_t st, int pair) {
  if (pair < 0) pair = pair_tiles(s) ? 1 : 0;
  const int R = s.R > 1 ? s.R : 0;
  const int chunk = R ? (s.T + R - 1) / R : 1;
  const long long tk = (long long)s.T * s.k;
  const size_t smem = sizeof(int) * (2 * s.E + (R ? R * R : 0) + 32 * s.E +
                                     (tk <= kFusedSmemIdx ? tk : 0));
  const int vpl = (s.E + 31) / 32;
#define MOE_FUSED_CALL(V)                                                                 \
  return route_fused_t<V>(logits, s, R, chunk, smem, idx, w, counts, offsets, tiles, send, \
                          rank_off, row_of, perm, err, pair, st)
  MOE_VPL_DISPATCH(vpl, MOE_FUSED_CALL);
#undef MOE_FUSED_CALL
}

cudaError_t launch_route_tables(const int* idx, const moe_shape& s, const WsLayout& L,
                                char* ws, int* counts, int* offsets, int* row_of,
                                int* perm, int* send, int* rank_off, cudaStream_t st,
                                int pair) {
  if (pair < 0) pair = pair_tiles(s) ? 1 : 0;
  int* err = reinterpret_cast<int*>(ws + L.err);
  int* blockhist = reinterpret_cast<int*>(ws + L.blockhist);
  int* blockbase = reinterpret_cast<int*>(ws + L.blockbase);
  int* blocksend = reinterpret_cast<int*>(ws + L.blocksend);
  int* tiles = reinterpret_cast<int*>(ws + L.tiles);
  const int R = s.R > 1 ? s.R : 0;
  const int chunk = R ? (s.T + R - 1) / R : 1;
  const size_t hist_smem = sizeof(int) * (s.E + (R ? R * R : 0));
  cudaError_t e = launch_kernel(k_hist, dim3(L.nblocks), dim3(kTokensPerRouteBlock), hist_smem,
                                st, 1, idx, s.T, s.E, s.k, R, chunk, blockhist, blocksend, err);
  if (e != cudaSuccess) return e;
  e = launch_kernel(k_scan, dim3(1), dim3(1024), 0, st, 1, blockhist, L.nblocks, s.E, R,
                    blocksend, blockbase, counts, offsets, tiles, send, rank_off, pair,
                    L.max_mtiles);
  if (e != cudaSuccess) return e;
  const size_t scat_smem = sizeof(uint32_t) * (kTokensPerRouteBlock / 32) * s.E;
  return launch_kernel(k_scatter, dim3(L.nblocks), dim3(kTokensPerRouteBlock), scat_smem, st, 1,
                       idx, s.T, s.E, s.k, blockbase, row_of, perm);
}

cudaError_t launch_tiles_from_offsets(const int* offsets, const moe_shape& s,
                                      int* tiles, int* err, cudaStream_t st, int pair) {
  if (pair < 0) pair = pair_tiles(s) ? 1 : 0;
  return launch_kernel(k_tiles_from_offsets, dim3(1), dim3(1024), 0, st, 1, offsets, s.E,
                       (int)((long long)s.T * s.k), tiles, err, pair);
}

cudaError_t launch_gather(const __nv_bfloat16* x, const int* perm, long long P, int T,
                          int d, __nv_bfloat16* x_perm, int* err, cudaStream_t st) {
  if (P == 0) return cudaSuccess;
  const long long blocks = (P + 7) / 8;
  return launch_kernel(k_gather_rows, dim3((unsigned)blocks), dim3(256), 0, st, 1, x, perm, P, T,
                       d, x_perm, err);
}

cudaError_t launch_combine(const __nv_bfloat16* z, const int* row_of, const float* w,
                           const moe_shape& s, __nv_bfloat16* y, cudaStream_t st) {
  // Large batches: 512 columns per warp (1 KB of each row per request
  // stream); small ones keep 256 so more warps share the latency.
  const bool wide = (long long)s.T * s.d >= (1LL << 22) && s.d % 512 == 0;
  const int span = wide ? 512 : 256;
  const long long warps = (long long)s.T * ((s.d + span - 1) / span);
  const unsigned blocks = (unsigned)((warps + 7) / 8);
  if (wide)
    return launch_kernel(k_combine<2>, dim3(blocks), dim3(256), 0, st, 1, z, row_of, w, s.T,
                         s.d, s.k, y);
  return launch_kernel(k_combine<1>, dim3(blocks), dim3(256), 0, st, 1, z, row_of, w, s.T, s.d,
                       s.k, y);
}

}  // namespace moe
