// C ABI of the B200 routed MoE layer: argument checks, workspace carving and
// the stream-ordered launch sequence.  No allocation, no host synchronisation
// (except moe_check), no CPU fallback.
#include <mutex>

#include "moe_kernels.cuh"

using namespace moe;

namespace {

constexpr int kVersion = 105;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool ok16(const void* p) { return p != nullptr && aligned(p, 16); }
bool ok4(const void* p) { return p != nullptr && aligned(p, 4); }

bool shape_ok(const moe_shape* s) { return shape_valid(s); }

// p can be read and written by the device as it is: device or managed
// memory, or page-locked host memory mapped at the same address.
bool device_addressable(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return true;
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

// Current device: its SM count, and whether it is an sm_100 part.
int device_check(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  static std::mutex mu;
  static int cc_major[128], sms[128];
  if (dev < 0 || dev >= 128) return MOE_ERR_CUDA;
  {
    std::lock_guard<std::mutex> g(mu);
    if (cc_major[dev] == 0) {
      int major = 0, n = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
              cudaSuccess ||
          cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      cc_major[dev] = major;
      sms[dev] = n;
    }
    *num_sms = sms[dev];
    return cc_major[dev] == 10 ? MOE_OK : MOE_ERR_UNSUPPORTED;
  }
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// Router logits: the cluster split-K kernel for small batches, the tensor
// cores (three bf16 planes of W_g) above kRouterTcMinT tokens.  moe_router
// and moe_forward both come here, so they give the same bits.
cudaError_t run_router(const __nv_bfloat16* x, const float* w_g, const float* bias,
                       const moe_shape& s, float* logits, const WsLayout& L, void* ws,
                       int sms, cudaStream_t st) {
  if (s.T >= kRouterTcMinT)
    return launch_router_tc(x, w_g, bias, s, logits, at<__nv_bfloat16>(ws, L.w3),
                            at<float>(ws, L.logit_part), at<int>(ws, L.err), sms, st);
  return launch_router(x, w_g, bias, s, logits, st);
}

}  // namespace

extern "C" {

const char* moe_error_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null or misaligned pointer, or shape out of range";
    case MOE_ERR_UNSUPPORTED:
      return "MOE_ERR_UNSUPPORTED: the current device is not an sm_100 GPU, or the shape is "
             "outside what this call runs (see the call's notes in moe.h)";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed or no CUDA device is usable";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait ran out";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a device-side consistency check failed";
    default: return "unknown moe_status";
  }
}

int moe_version(void) { return kVersion; }

size_t moe_workspace_size(const moe_shape* s) {
  if (!shape_ok(s)) return 0;
  return ws_layout(*s, 0).total;
}

int moe_router(const moe_bf16* x, const float* w_g, const float* bias, const moe_shape* s,
               float* logits, void* ws, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(x) || !ok4(w_g) || !ok4(logits) || (bias && !aligned(bias, 4)) || !ws ||
      !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  const WsLayout L = ws_layout(*s, sms);
  return cuda_status(run_router(reinterpret_cast<const __nv_bfloat16*>(x), w_g, bias, *s,
                                logits, L, ws, sms, static_cast<cudaStream_t>(stream)));
}

int moe_topk(const float* logits, const moe_shape* s, int32_t* idx, float* w, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok4(logits) || !ok4(idx) || !ok4(w)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(launch_topk(logits, *s, idx, w, static_cast<cudaStream_t>(stream)));
}

int moe_dispatch(const int32_t* idx, const moe_bf16* x, const moe_shape* s, int32_t* counts,
                 int32_t* offsets, int32_t* perm, int32_t* row_of, moe_bf16* x_perm,
                 int32_t* send_counts, int32_t* rank_offsets, void* ws, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (!ok4(counts) || !ok4(offsets) || !ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  if ((send_counts || rank_offsets) && s->R <= 1) return MOE_ERR_INVALID_ARG;
  if ((send_counts && !aligned(send_counts, 4)) || (rank_offsets && !aligned(rank_offsets, 4)))
    return MOE_ERR_INVALID_ARG;
  if (s->T > 0 && (!ok4(idx) || !ok16(x) || !ok4(perm) || !ok4(row_of) || !ok16(x_perm)))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*s, sms);
  if (s->T == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int) * s->E, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int) * (s->E + 1), cs);
    if (e == cudaSuccess && send_counts)
      e = cudaMemsetAsync(send_counts, 0, sizeof(int) * s->R * s->R, cs);
    if (e == cudaSuccess && rank_offsets)
      e = cudaMemsetAsync(rank_offsets, 0, sizeof(int) * (s->R + 1), cs);
    return cuda_status(e);
  }
  int* send = send_counts ? send_counts : at<int>(ws, L.send);
  int* roff = rank_offsets ? rank_offsets : at<int>(ws, L.rank_off);
  cudaError_t e = launch_route_tables(idx, *s, L, static_cast<char*>(ws), counts, offsets,
                                      row_of, perm, send, roff, cs);
  if (e == cudaSuccess)
    e = launch_gather(reinterpret_cast<const __nv_bfloat16*>(x), perm, L.P, s->T, s->d,
                      reinterpret_cast<__nv_bfloat16*>(x_perm), at<int>(ws, L.err), cs);
  return cuda_status(e);
}

int moe_ffn(const moe_bf16* x_perm, const int32_t* offsets, const moe_bf16* w13,
            const moe_bf16* w2, const moe_shape* s, moe_bf16* z, void* ws, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(x_perm) || !ok4(offsets) || !ok16(w13) || !ok16(w2) || !ok16(z) || !ws ||
      !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*s, sms);
  char* w = static_cast<char*>(ws);
  cudaError_t e = launch_tiles_from_offsets(offsets, *s, at<int>(ws, L.tiles),
                                            at<int>(ws, L.err), cs);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return launch_expert_ffn(reinterpret_cast<const __nv_bfloat16*>(x_perm), L.P,
                           reinterpret_cast<const __nv_bfloat16*>(w13),
                           reinterpret_cast<const __nv_bfloat16*>(w2), *s, L, w,
                           reinterpret_cast<__nv_bfloat16*>(z), sms, cs);
}

int moe_combine(const moe_bf16* z, const int32_t* row_of, const float* w, const moe_shape* s,
                moe_bf16* y, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(z) || !ok4(row_of) || !ok4(w) || !ok16(y)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(launch_combine(reinterpret_cast<const __nv_bfloat16*>(z), row_of, w, *s,
                                    reinterpret_cast<__nv_bfloat16*>(y),
                                    static_cast<cudaStream_t>(stream)));
}

// Expert weight / activation formats of the whole layer.
enum : int { kBf16 = 0, kFp8Weights = 1, kW8A8 = 2 };

// The whole layer: bf16 expert weights; E4M3 expert weights with one fp32
// scale per weight row (kFp8Weights, bf16 tokens); or those weights with the
// tokens and the SwiGLU output quantised to E4M3 too (kW8A8).
static int forward_impl(int mode, const moe_bf16* x, const float* w_g, const float* bias,
                        const void* w13, const float* w13_scale, const void* w2,
                        const float* w2_scale, const moe_shape* s, moe_bf16* y,
                        int32_t* idx_out, float* w_out, int32_t* counts_out, void* ws,
                        void* stream, void* const* events) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(x) || !ok4(w_g) || (bias && !aligned(bias, 4)) || !ok16(w13) || !ok16(w2) ||
      !ok16(y) || (idx_out && !aligned(idx_out, 4)) || (w_out && !aligned(w_out, 4)) ||
      (counts_out && !aligned(counts_out, 4)) ||
      (mode != kBf16 && (!ok4(w13_scale) || !ok4(w2_scale))))
    return MOE_ERR_INVALID_ARG;
  // The FP8-weight GEMMs run on the plain 128-row tile list; the bf16 and
  // W8A8 ones on the CTA-pair layout when pair_tiles(s).
  const int pair = mode == kFp8Weights ? 0 : -1;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  if (!device_addressable(y)) return MOE_ERR_INVALID_ARG;  // y may be page-locked host memory
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), cs,
                                    cudaEventRecordExternal);
  };
  const WsLayout L = ws_layout(*s, sms);
  char* wsb = static_cast<char*>(ws);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  float* logits = at<float>(ws, L.logits);
  int* idx = idx_out ? idx_out : at<int>(ws, L.idx);
  float* gw = w_out ? w_out : at<float>(ws, L.w);
  int* counts = counts_out ? counts_out : at<int>(ws, L.counts);
  int* offsets = at<int>(ws, L.offsets);
  int* perm = at<int>(ws, L.perm);
  int* row_of = at<int>(ws, L.row_of);
  __nv_bfloat16* x_perm = at<__nv_bfloat16>(ws, L.x_perm);
  __nv_bfloat16* z = at<__nv_bfloat16>(ws, L.z);

  cudaError_t e = mark(0);
  if (e == cudaSuccess) e = run_router(xb, w_g, bias, *s, logits, L, ws, sms, cs);
  if (e == cudaSuccess) e = mark(1);
  if (e == cudaSuccess) {
    if (s->T <= kFusedRouteMaxT) {
      e = launch_route_fused(logits, *s, idx, gw, counts, offsets, at<int>(ws, L.tiles),
                             at<int>(ws, L.send), at<int>(ws, L.rank_off), row_of, perm,
                             at<int>(ws, L.err), cs, pair);
    } else {
      e = launch_topk(logits, *s, idx, gw, cs);
      if (e == cudaSuccess)
        e = launch_route_tables(idx, *s, L, wsb, counts, offsets, row_of, perm,
                                at<int>(ws, L.send), at<int>(ws, L.rank_off), cs, pair);
    }
  }
  uint8_t* xq = at<uint8_t>(ws, L.x_perm);  // W8A8: token codes in the x_perm region
  float* xs = at<float>(ws, L.xs);
  // bf16 with at most 16 tokens: GEMM1 reads x itself (all tokens in one
  // 16-row tile, the bytes a gathered tile of up to 16 rows has); with more,
  // the whole token tile in every stage slows the weight stream (same-box A/B:
  // T = 64 116.5 -> 133.4 us, T = 8 66.2 -> 63.8, T = 1 44.9 -> 43.1)
  const bool direct = mode == kBf16 && s->T <= 16;
  if (e == cudaSuccess && !direct)
    e = mode == kW8A8
            ? launch_quant_rows(xb, perm, L.P, s->T, s->d, xq, xs, at<int>(ws, L.err), cs)
            : launch_gather(xb, perm, L.P, s->T, s->d, x_perm, at<int>(ws, L.err), cs);
  if (e == cudaSuccess) e = mark(2);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  void* const* ev = events ? events + 3 : nullptr;
  int r;
  if (mode == kW8A8)
    r = launch_expert_ffn_w8a8(xq, xs, L.Ppad, static_cast<const uint8_t*>(w13), w13_scale,
                               static_cast<const uint8_t*>(w2), w2_scale, *s, L, wsb, z, sms, cs,
                               ev, true);
  else if (mode == kFp8Weights)
    r = launch_expert_ffn_fp8(x_perm, L.Ppad, static_cast<const uint8_t*>(w13), w13_scale,
                              static_cast<const uint8_t*>(w2), w2_scale, *s, L, wsb, z, sms, cs,
                              ev);
  else
    r = direct ? launch_expert_ffn(xb, s->T, static_cast<const __nv_bfloat16*>(w13),
                                   static_cast<const __nv_bfloat16*>(w2), *s, L, wsb, z, sms, cs,
                                   ev, false, perm)
               : launch_expert_ffn(x_perm, L.Ppad, static_cast<const __nv_bfloat16*>(w13),
                                   static_cast<const __nv_bfloat16*>(w2), *s, L, wsb, z, sms, cs,
                                   ev, true);
  if (r != MOE_OK) return r;
  e = launch_combine(z, row_of, gw, *s, reinterpret_cast<__nv_bfloat16*>(y), cs);
  if (e == cudaSuccess) e = mark(5);
  return cuda_status(e);
}

int moe_forward(const moe_bf16* x, const float* w_g, const float* bias, const moe_bf16* w13,
                const moe_bf16* w2, const moe_shape* s, moe_bf16* y, int32_t* idx_out,
                float* w_out, int32_t* counts_out, void* ws, void* stream) {
  return forward_impl(kBf16, x, w_g, bias, w13, nullptr, w2, nullptr, s, y, idx_out, w_out,
                      counts_out, ws, stream, nullptr);
}

int moe_forward_staged(const moe_bf16* x, const float* w_g, const float* bias,
                       const moe_bf16* w13, const moe_bf16* w2, const moe_shape* s,
                       moe_bf16* y, void* ws, void* const* events, void* stream) {
  return forward_impl(kBf16, x, w_g, bias, w13, nullptr, w2, nullptr, s, y, nullptr, nullptr,
                      nullptr, ws, stream, events);
}

int moe_ffn_fp8(const moe_bf16* x_perm, const int32_t* offsets, const uint8_t* w13,
                const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                const moe_shape* s, moe_bf16* z, void* ws, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(x_perm) || !ok4(offsets) || !ok16(w13) || !ok4(w13_scale) || !ok16(w2) ||
      !ok4(w2_scale) || !ok16(z) || !ws || !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*s, sms);
  cudaError_t e = launch_tiles_from_offsets(offsets, *s, at<int>(ws, L.tiles),
                                            at<int>(ws, L.err), cs, 0);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return launch_expert_ffn_fp8(reinterpret_cast<const __nv_bfloat16*>(x_perm), L.P, w13,
                               w13_scale, w2, w2_scale, *s, L, static_cast<char*>(ws),
                               reinterpret_cast<__nv_bfloat16*>(z), sms, cs);
}

int moe_forward_fp8(const moe_bf16* x, const float* w_g, const float* bias, const uint8_t* w13,
                    const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                    const moe_shape* s, moe_bf16* y, int32_t* idx_out, float* w_out,
                    int32_t* counts_out, void* ws, void* stream) {
  return forward_impl(kFp8Weights, x, w_g, bias, w13, w13_scale, w2, w2_scale, s, y, idx_out,
                      w_out, counts_out, ws, stream, nullptr);
}

int moe_forward_fp8_staged(const moe_bf16* x, const float* w_g, const float* bias,
                           const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                           const float* w2_scale, const moe_shape* s, moe_bf16* y, void* ws,
                           void* const* events, void* stream) {
  return forward_impl(kFp8Weights, x, w_g, bias, w13, w13_scale, w2, w2_scale, s, y, nullptr,
                      nullptr, nullptr, ws, stream, events);
}

int moe_quantise_rows_e4m3(const moe_bf16* a, int64_t rows, int32_t cols, uint8_t* codes,
                           float* scales, void* stream) {
  if (rows < 0 || cols < 16 || cols % 16 || cols > (1 << 20)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!ok16(a) || !ok16(codes) || !ok4(scales)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(launch_quant_rows(reinterpret_cast<const __nv_bfloat16*>(a), nullptr, rows,
                                       0, cols, codes, scales, nullptr,
                                       static_cast<cudaStream_t>(stream)));
}

int moe_ffn_w8a8(const moe_bf16* x_perm, const int32_t* offsets, const uint8_t* w13,
                 const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                 const moe_shape* s, moe_bf16* z, void* ws, void* stream) {
  if (!shape_ok(s)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(x_perm) || !ok4(offsets) || !ok16(w13) || !ok4(w13_scale) || !ok16(w2) ||
      !ok4(w2_scale) || !ok16(z) || !ws || !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*s, sms);
  uint8_t* xq = at<uint8_t>(ws, L.x_perm);
  float* xs = at<float>(ws, L.xs);
  // the work list first, so GEMM1 may read it before the quantisation completes
  cudaError_t e = launch_tiles_from_offsets(offsets, *s, at<int>(ws, L.tiles),
                                            at<int>(ws, L.err), cs);
  if (e == cudaSuccess)
    e = launch_quant_rows(reinterpret_cast<const __nv_bfloat16*>(x_perm), nullptr, L.P, 0, s->d,
                          xq, xs, at<int>(ws, L.err), cs);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return launch_expert_ffn_w8a8(xq, xs, L.Ppad, w13, w13_scale, w2, w2_scale, *s, L,
                                static_cast<char*>(ws), reinterpret_cast<__nv_bfloat16*>(z), sms,
                                cs, nullptr, true);
}

int moe_forward_w8a8(const moe_bf16* x, const float* w_g, const float* bias, const uint8_t* w13,
                     const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                     const moe_shape* s, moe_bf16* y, int32_t* idx_out, float* w_out,
                     int32_t* counts_out, void* ws, void* stream) {
  return forward_impl(kW8A8, x, w_g, bias, w13, w13_scale, w2, w2_scale, s, y, idx_out, w_out,
                      counts_out, ws, stream, nullptr);
}

int moe_forward_w8a8_staged(const moe_bf16* x, const float* w_g, const float* bias,
                            const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                            const float* w2_scale, const moe_shape* s, moe_bf16* y, void* ws,
                            void* const* events, void* stream) {
  return forward_impl(kW8A8, x, w_g, bias, w13, w13_scale, w2, w2_scale, s, y, nullptr, nullptr,
                      nullptr, ws, stream, events);
}

size_t moe_workspace_size_eplb(const moe_shape* s, int32_t E_phys) {
  if (!shape_ok(s) || E_phys < s->E || E_phys > kMaxE || (s->R > 1 && E_phys % s->R))
    return 0;
  return ws_layout(*s, 0, E_phys).total;
}

int moe_eplb_remap(const int32_t* idx, const moe_shape* s, const int32_t* rep_offsets,
                   const int32_t* rep_phys, int32_t E_phys, int32_t* idx_phys, void* ws,
                   void* stream) {
  if (!shape_ok(s) || E_phys < s->E || E_phys > kMaxE) return MOE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok4(idx) || !ok4(rep_offsets) || !ok4(rep_phys) || !ok4(idx_phys))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(launch_eplb_remap(idx, s->T, s->k, s->E, rep_offsets, rep_phys, E_phys,
                                       idx_phys, static_cast<int*>(ws),
                                       static_cast<cudaStream_t>(stream)));
}

int moe_forward_eplb(const moe_bf16* x, const float* w_g, const float* bias,
                     const moe_bf16* w13_phys, const moe_bf16* w2_phys, const moe_shape* s,
                     const int32_t* rep_offsets, const int32_t* rep_phys, int32_t E_phys,
                     moe_bf16* y, int32_t* idx_out, float* w_out, int32_t* counts_out,
                     void* ws, void* stream) {
  if (!shape_ok(s) || E_phys < s->E || E_phys > kMaxE || (s->R > 1 && E_phys % s->R))
    return MOE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!ok16(x) || !ok4(w_g) || (bias && !aligned(bias, 4)) || !ok16(w13_phys) ||
      !ok16(w2_phys) || !ok16(y) || !ok4(rep_offsets) || !ok4(rep_phys) ||
      (idx_out && !aligned(idx_out, 4)) || (w_out && !aligned(w_out, 4)) ||
      (counts_out && !aligned(counts_out, 4)))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  moe_shape sp = *s;  // the physical experts: dispatch tables and expert GEMMs
  sp.E = E_phys;
  const WsLayout L = ws_layout(*s, sms, E_phys);
  char* wsb = static_cast<char*>(ws);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  float* logits = at<float>(ws, L.logits);
  int* idx = idx_out ? idx_out : at<int>(ws, L.idx);
  int* idx_p = at<int>(ws, L.idx_phys);
  float* gw = w_out ? w_out : at<float>(ws, L.w);
  int* counts = counts_out ? counts_out : at<int>(ws, L.counts);
  int* perm = at<int>(ws, L.perm);
  int* row_of = at<int>(ws, L.row_of);
  __nv_bfloat16* x_perm = at<__nv_bfloat16>(ws, L.x_perm);
  __nv_bfloat16* z = at<__nv_bfloat16>(ws, L.z);
  int* err = at<int>(ws, L.err);
  // router and selection over the logical experts, then each selection to
  // its replica, then the layer over the physical experts
  cudaError_t e = run_router(xb, w_g, bias, *s, logits, L, ws, sms, cs);
  if (e == cudaSuccess) e = launch_topk(logits, *s, idx, gw, cs);
  if (e == cudaSuccess)
    e = launch_eplb_remap(idx, s->T, s->k, s->E, rep_offsets, rep_phys, E_phys, idx_p, err, cs);
  if (e == cudaSuccess)
    e = launch_route_tables(idx_p, sp, L, wsb, counts, at<int>(ws, L.offsets), row_of, perm,
                            at<int>(ws, L.send), at<int>(ws, L.rank_off), cs);
  if (e == cudaSuccess) e = launch_gather(xb, perm, L.P, s->T, s->d, x_perm, err, cs);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  int r = launch_expert_ffn(x_perm, L.Ppad, reinterpret_cast<const __nv_bfloat16*>(w13_phys),
                            reinterpret_cast<const __nv_bfloat16*>(w2_phys), sp, L, wsb, z, sms,
                            cs, nullptr, true);
  if (r != MOE_OK) return r;
  return cuda_status(
      launch_combine(z, row_of, gw, *s, reinterpret_cast<__nv_bfloat16*>(y), cs));
}

int moe_selftest_bounded_wait(long long limit_ns, void* ws, void* stream) {
  if (limit_ns <= 0 || limit_ns > 1000000000LL || !ws || !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(launch_selftest_bounded_wait((unsigned long long)limit_ns,
                                                  static_cast<int*>(ws),
                                                  static_cast<cudaStream_t>(stream)));
}

int moe_copy(void* dst, const void* src, int64_t bytes, void* stream) {
  if (bytes < 0 || bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (bytes == 0) return MOE_OK;
  if (!ok16(dst) || !ok16(src)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  int st = device_check(&sms);
  if (st != MOE_OK) return st;
  if (!device_addressable(dst) || !device_addressable(src)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_copy(dst, src, bytes, sms, static_cast<cudaStream_t>(stream)));
}

int moe_check(void* ws, void* stream) {
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (h[0] != 0) {
    if (cudaMemsetAsync(ws, 0, 64, cs) != cudaSuccess || cudaStreamSynchronize(cs) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return h[0];
}

}  // extern "C"
