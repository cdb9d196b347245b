// Receive side of the expert-parallel token exchange.
//
// "Serving MoE models with expert parallelism on 8xH200", section "Tensor
// parallel vs expert parallel": each device holds whole experts, tokens are
// sent to the devices holding their experts and the results come back through
// a second exchange; "Wide Expert Parallelism", section "All-to-all
// communication: the essential tradeoff".  A rank's dispatch buffer is
// expert-major, so the rows it sends to rank r are ordered by r's local
// expert; what rank r receives is therefore ordered by (source rank, local
// expert, token).  This kernel labels every received row with its local
// expert from the exchanged per-(source, expert) counts, so the receiver can
// regroup the rows expert-major with the ordinary dispatch (k = 1) and run
// the expert GEMMs once per expert over the rows of all sources.
#include "moe_kernels.cuh"

using namespace moe;

namespace {

constexpr int kSegThreads = 256;

// recv_counts: [R * E_loc] rows per (source, local expert), source-major.
// Every block scans the (at most kMaxE) counts in shared memory, then each
// thread finds its row's segment by binary search.  Rows at or beyond the
// counts' total (or any row, when a count is negative) get -1, which the
// dispatch that consumes the labels records as an invalid expert id.
__global__ void __launch_bounds__(kSegThreads) k_ep_recv_experts(
    const int* __restrict__ recv_counts, int nseg, int E_loc, int N, int* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ int off[kMaxE + 1];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  // sequential scan by one warp (nseg <= 1024): lane-strided partial sums
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (nseg + 31) / 32;
    const int a = min(lane * per, nseg), b = min(a + per, nseg);
    int s = 0;
    for (int i = a; i < b; ++i) {
      const int c = recv_counts[i];
      if (c < 0) bad = 1;
      s += c;
    }
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    int run = inc - s;
    for (int i = a; i < b; ++i) {
      off[i] = run;
      run += recv_counts[i];
    }
    if (lane == 31) off[nseg] = inc;
  }
  __syncthreads();
  const int r = blockIdx.x * kSegThreads + threadIdx.x;
  if (r >= N) return;
  if (bad || r >= off[nseg]) {
    out[r] = -1;
    return;
  }
  int lo = 0, hi = nseg - 1;  // last segment with off[seg] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  out[r] = lo % E_loc;
}

bool al4(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace

extern "C" int moe_ep_recv_experts(const int32_t* recv_counts, int32_t R, int32_t E_loc,
                                   int32_t N, int32_t* expert_of_row, void* stream) {
  if (R < 1 || R > kMaxR || E_loc < 1 || (long long)R * E_loc > kMaxE || N < 0 ||
      N > (1 << 25) || !al4(recv_counts) || (N > 0 && !al4(expert_of_row)))
    return MOE_ERR_INVALID_ARG;
  if (N == 0) return MOE_OK;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  const unsigned blocks = (unsigned)((N + kSegThreads - 1) / kSegThreads);
  cudaError_t e = launch_kernel(k_ep_recv_experts, dim3(blocks), dim3(kSegThreads), 0,
                                static_cast<cudaStream_t>(stream), 1, recv_counts, R * E_loc,
                                E_loc, N, expert_of_row);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
