// Internal launchers shared by the C ABI (moe_abi.cu) and the kernel files.
#pragma once

#include <algorithm>
#include <climits>

#include "moe_common.cuh"

namespace moe {

cudaError_t launch_router(const __nv_bfloat16* x, const float* w_g, const float* bias,
                          const moe_shape& s, float* logits, cudaStream_t st);
cudaError_t launch_router_tc(const __nv_bfloat16* x, const float* w_g, const float* bias,
                             const moe_shape& s, float* logits, __nv_bfloat16* w3,
                             float* part, int* err, int num_sms, cudaStream_t st);
cudaError_t launch_topk(const float* logits, const moe_shape& s, int* idx, float* w,
                        cudaStream_t st);
// Selection + dispatch tables in one block; valid for T <= kFusedRouteMaxT.
constexpr int kFusedRouteMaxT = 1024;
// `pair`: 1 = the work lists of the CTA-pair expert GEMMs (tile pairs plus a
// leftover list), 0 = plain 128-row tiles, -1 = pair_tiles(s) (the bf16 GEMMs'
// choice; the FP8 GEMMs always take plain tiles).
cudaError_t launch_route_fused(const float* logits, const moe_shape& s, int* idx, float* w,
                               int* counts, int* offsets, int* tiles, int* send,
                               int* rank_off, int* row_of, int* perm, int* err,
                               cudaStream_t st, int pair = -1);
cudaError_t launch_route_tables(const int* idx, const moe_shape& s, const WsLayout& L,
                                char* ws, int* counts, int* offsets, int* row_of,
                                int* perm, int* send, int* rank_off, cudaStream_t st,
                                int pair = -1);
cudaError_t launch_tiles_from_offsets(const int* offsets, const moe_shape& s,
                                      int* tiles, int* err, cudaStream_t st, int pair = -1);
cudaError_t launch_gather(const __nv_bfloat16* x, const int* perm, long long P, int T,
                          int d, __nv_bfloat16* x_perm, int* err, cudaStream_t st);
cudaError_t launch_selftest_bounded_wait(unsigned long long limit_ns, int* err,
                                         cudaStream_t st);
// bytes (a multiple of 16) from src to dst, both 16-byte aligned and
// addressable by the device.
cudaError_t launch_copy(void* dst, const void* src, long long bytes, int num_sms,
                        cudaStream_t st);
cudaError_t launch_combine(const __nv_bfloat16* z, const int* row_of, const float* w,
                           const moe_shape& s, __nv_bfloat16* y, cudaStream_t st);
// early_gemm1: the kernel just before (the row gather) lets GEMM1 launch only
// after its own wait, and the work list comes from a kernel before it, so
// GEMM1 may start streaming weights before the gather completes.
// tok_row (T <= 64 only; else ignored): x_perm is the unpermuted x (x_rows =
// T) and tok_row[r] the token of dispatch row r; GEMM1 multiplies all T
// tokens per item and stores each entry's rows itself, so no gather runs
// (the forward uses it up to 16 tokens).
int launch_expert_ffn(const __nv_bfloat16* x_perm, long long x_rows,
                      const __nv_bfloat16* w13, const __nv_bfloat16* w2,
                      const moe_shape& s, const WsLayout& L, char* ws,
                      __nv_bfloat16* z, int num_sms, cudaStream_t st,
                      void* const* events = nullptr, bool early_gemm1 = false,
                      const int* tok_row = nullptr);

// The same two GEMMs with E4M3 expert weights and one fp32 scale per weight
// row (moe_gemm_fp8.cu): swap-AB form at every batch size, over the plain
// 128-row tile list above 64 tokens.
int launch_expert_ffn_fp8(const __nv_bfloat16* x_perm, long long x_rows, const uint8_t* w13,
                          const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                          const moe_shape& s, const WsLayout& L, char* ws, __nv_bfloat16* z,
                          int num_sms, cudaStream_t st, void* const* events = nullptr);

// Row quantisation to E4M3 with power-of-two row scales (moe_w8a8.cu):
// output row r from input row perm[r] (perm != nullptr; ids outside
// [0, n_src) are recorded in err) or row r.
cudaError_t launch_quant_rows(const __nv_bfloat16* a, const int* perm, long long rows, int n_src,
                              int cols, uint8_t* codes, float* scales, int* err,
                              cudaStream_t st);

// The small-batch W8A8 SwiGLU output quantised per work-list entry while
// GEMM1 runs (moe_w8a8.cu): one block per entry (max_entries blocks; the
// count is list_count[0]), waiting on ready1[i] >= target1 and setting
// ready2[i].
cudaError_t launch_quant_entries(const __nv_bfloat16* h, int cols, const int* list_count,
                                 const int* list, int row_tiles, int max_entries,
                                 const int* ready1, int target1, int* ready2, uint8_t* codes,
                                 float* scales, int* err, cudaStream_t st);

// Both expert GEMMs with E4M3 weights (one fp32 scale per weight row) and
// E4M3 tokens (xq, one scale per row in xs): GEMM1 with the SwiGLU epilogue
// into h (bf16), h quantised into the workspace, GEMM2 (moe_gemm_sm100.cu).
int launch_expert_ffn_w8a8(const uint8_t* xq, const float* xs, long long x_rows,
                           const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                           const float* w2_scale, const moe_shape& s, const WsLayout& L,
                           char* ws, __nv_bfloat16* z, int num_sms, cudaStream_t st,
                           void* const* events = nullptr, bool early_gemm1 = false);

// Logical -> physical expert ids of a replica plan (moe_eplb.cu).
cudaError_t launch_eplb_remap(const int* idx, int T, int k, int E, const int* rep_offsets,
                              const int* rep_phys, int P, int* idx_phys, int* err,
                              cudaStream_t st);

}  // namespace moe
