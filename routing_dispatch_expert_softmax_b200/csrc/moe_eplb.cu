// Expert load balancing (EPLB-style): the replica plan on the host and the
// logical -> physical expert remap on the device.
//
// "Serving MoE models with expert parallelism on 8xH200", section "Routing
// imbalance": the load of each expert is measured, the busiest experts get
// extra copies hosted by the devices with spare capacity, and busy and idle
// experts are mixed on each device.  "vLLM Expert Parallel deployment" (EPLB
// section): the load comes from a window of recent steps and the count of
// extra copies is a setting.  The pages
// give no algorithm; the plan below is the plainest integer reading:
//   1. every expert starts with one copy; n_redundant times the expert with
//      the largest load per copy gets another (ties: lower id);
//   2. replica i of expert e is credited load_e / n_e, plus one if
//      i < load_e mod n_e;
//   3. replicas, by decreasing credit (ties: lower expert, lower replica), go
//      to the least-loaded rank that has a free slot (ties: lower rank); rank
//      r owns physical slots r*S .. r*S + S - 1 in the order they are filled;
//   4. slot j of token t with logical expert e uses replica t mod n_e.
#include <algorithm>
#include <vector>

#include "moe_kernels.cuh"

namespace moe {

__global__ void __launch_bounds__(256) k_eplb_remap(const int* __restrict__ idx, int T, int k,
                                                    int E, const int* __restrict__ rep_offsets,
                                                    const int* __restrict__ rep_phys, int P,
                                                    int* __restrict__ idx_phys, int* err) {
  pdl_trigger();
  pdl_wait();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * k) return;
  const int t = (int)(i / k);
  const int e = idx[i];
  int p = -1;
  if (e >= 0 && e < E) {
    const int a = rep_offsets[e], b = rep_offsets[e + 1];
    if (a >= 0 && b > a && b <= P) {
      const int q = rep_phys[a + t % (b - a)];
      if (q >= 0 && q < P) p = q;
    }
  }
  if (p < 0) record_error(err, MOE_ERR_DEVICE_CHECK, 30);  // never dereferenced downstream
  idx_phys[i] = p;
}

cudaError_t launch_eplb_remap(const int* idx, int T, int k, int E, const int* rep_offsets,
                              const int* rep_phys, int P, int* idx_phys, int* err,
                              cudaStream_t st) {
  const long long n = (long long)T * k;
  if (n == 0) return cudaSuccess;
  return launch_kernel(k_eplb_remap, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, 1,
                       idx, T, k, E, rep_offsets, rep_phys, P, idx_phys, err);
}

}  // namespace moe

using namespace moe;

extern "C" int moe_eplb_plan(const int64_t* load, int32_t E, int32_t R, int32_t n_redundant,
                             int32_t* phys_to_logical, int32_t* rep_offsets,
                             int32_t* rep_phys) {
  if (!load || !phys_to_logical || !rep_offsets || !rep_phys) return MOE_ERR_INVALID_ARG;
  if (E < 1 || R < 1 || R > kMaxR || n_redundant < 0) return MOE_ERR_INVALID_ARG;
  const int P = E + n_redundant;
  if (P > kMaxE || P % R) return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < E; ++e)
    if (load[e] < 0 || load[e] > (1LL << 50)) return MOE_ERR_INVALID_ARG;
  // 1. copies
  std::vector<long long> n(E, 1);
  for (int r = 0; r < n_redundant; ++r) {
    int best = 0;
    for (int e = 1; e < E; ++e)
      if (load[e] * n[best] > load[best] * n[e]) best = e;  // exact: both < 2^61
    ++n[best];
  }
  // 2. credits
  struct Rep {
    long long share;
    int e, i;
  };
  std::vector<Rep> reps;
  reps.reserve(P);
  for (int e = 0; e < E; ++e)
    for (int i = 0; i < n[e]; ++i)
      reps.push_back({load[e] / n[e] + (i < load[e] % n[e] ? 1 : 0), e, i});
  std::sort(reps.begin(), reps.end(), [](const Rep& a, const Rep& b) {
    if (a.share != b.share) return a.share > b.share;
    if (a.e != b.e) return a.e < b.e;
    return a.i < b.i;
  });
  // 3. placement
  const int S = P / R;
  rep_offsets[0] = 0;
  for (int e = 0; e < E; ++e) rep_offsets[e + 1] = rep_offsets[e] + (int32_t)n[e];
  std::vector<long long> rank_load(R, 0);
  std::vector<int> rank_fill(R, 0);
  for (const Rep& rp : reps) {
    int r = -1;
    for (int q = 0; q < R; ++q)
      if (rank_fill[q] < S && (r < 0 || rank_load[q] < rank_load[r])) r = q;
    const int slot = r * S + rank_fill[r]++;
    rank_load[r] += rp.share;
    rep_phys[rep_offsets[rp.e] + rp.i] = slot;
    phys_to_logical[slot] = rp.e;
  }
  return MOE_OK;
}
