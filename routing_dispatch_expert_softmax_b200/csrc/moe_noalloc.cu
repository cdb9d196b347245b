// moe_dispatch_noalloc: the dispatch step without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they dispatch
// tokens: code running under an allocator that is frozen after start-up, a
// host runtime that hands out only fixed, pre-registered buffers, or a plugin
// that is given its inputs and outputs and nothing else.  For them this entry
// point keeps the dispatch scratch (per-block expert histograms and bases,
// per-block send counts, the expert tile list, the device error word) in a
// file-scope device array instead of `ws`.  The array is MOE_NOALLOC_SCRATCH
// bytes; every GPU that loads the library holds it until the process exits.
#include <mutex>

#include "moe_kernels.cuh"

using namespace moe;

namespace {

constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH;

// The scratch itself.  In host code `g_dispatch_scratch` names a host-side
// stand-in, never device memory: kernels get the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_dispatch_scratch[kScratchBytes];

// Scratch carve for one shape: only the regions the dispatch kernels use.
bool scratch_layout(const moe_shape& s, WsLayout* L) {
  *L = WsLayout{};
  const long long E = s.E, k = s.k, T = s.T;
  const long long R = s.R > 1 ? s.R : 1;
  L->P = T * k;
  L->Ppad = L->P + kGemmBM;
  L->nblocks = (int)((T + kTokensPerRouteBlock - 1) / kTokensPerRouteBlock);
  L->max_mtiles = max_mtiles_of(L->P, (int)E);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L->err = take(64);
  L->blockhist = take(sizeof(int) * (size_t)L->nblocks * E);
  L->blockbase = take(sizeof(int) * (size_t)L->nblocks * E);
  L->blocksend = take(sizeof(int) * (size_t)L->nblocks * R * R);
  L->send = take(sizeof(int) * R * R);
  L->rank_off = take(sizeof(int) * (R + 1));
  L->tiles = take(sizeof(int) * tile_list_ints(L->max_mtiles, (int)E));
  L->total = o;
  return o <= kScratchBytes;
}

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_address(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  static std::mutex mu;
  static unsigned char* addr[128];
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = addr[dev];
  return MOE_OK;
}

bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" int moe_dispatch_noalloc(const int32_t* idx, const moe_bf16* x,
                                    const moe_shape* s, int32_t* counts, int32_t* offsets,
                                    int32_t* perm, int32_t* row_of, moe_bf16* x_perm,
                                    int32_t* send_counts, int32_t* rank_offsets,
                                    void* stream) {
  if (!shape_valid(s)) return MOE_ERR_INVALID_ARG;
  if (!counts || !offsets || !al(counts, 4) || !al(offsets, 4)) return MOE_ERR_INVALID_ARG;
  if ((send_counts || rank_offsets) && s->R <= 1) return MOE_ERR_INVALID_ARG;
  if ((send_counts && !al(send_counts, 4)) || (rank_offsets && !al(rank_offsets, 4)))
    return MOE_ERR_INVALID_ARG;
  if (s->T > 0 && (!idx || !x || !perm || !row_of || !x_perm || !al(idx, 4) || !al(x, 16) ||
                   !al(perm, 4) || !al(row_of, 4) || !al(x_perm, 16)))
    return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if (!scratch_layout(*s, &L)) return MOE_ERR_UNSUPPORTED;  // beyond the scratch
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  unsigned char* base = nullptr;
  int st = scratch_address(&base);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (s->T == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int) * s->E, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int) * (s->E + 1), cs);
    if (e == cudaSuccess && send_counts)
      e = cudaMemsetAsync(send_counts, 0, sizeof(int) * s->R * s->R, cs);
    if (e == cudaSuccess && rank_offsets)
      e = cudaMemsetAsync(rank_offsets, 0, sizeof(int) * (s->R + 1), cs);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  char* ws = reinterpret_cast<char*>(base);
  // The error word must start at zero; everything else is fully rewritten.
  cudaError_t e = cudaMemsetAsync(ws + L.err, 0, 64, cs);
  int* send = send_counts ? send_counts : reinterpret_cast<int*>(ws + L.send);
  int* roff = rank_offsets ? rank_offsets : reinterpret_cast<int*>(ws + L.rank_off);
  if (e == cudaSuccess)
    e = launch_route_tables(idx, *s, L, ws, counts, offsets, row_of, perm, send, roff, cs);
  if (e == cudaSuccess)
    e = launch_gather(reinterpret_cast<const __nv_bfloat16*>(x), perm, L.P, s->T, s->d,
                      reinterpret_cast<__nv_bfloat16*>(x_perm),
                      reinterpret_cast<int*>(ws + L.err), cs);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
