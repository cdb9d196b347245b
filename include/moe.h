/*
 * moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts layer forward.
 *
 * The operation is the routed MoE layer the expert-parallel serving pages
 * describe, on one GPU:
 *   - "Wide Expert Parallelism" (llm-d), section "What is an MoE layer?": a
 *     routing gate scores every token and sends it to a few experts (8 of 256
 *     in the DeepSeek example);
 *   - "Serving MoE models with expert parallelism on 8xH200", section "Tensor
 *     parallel vs expert parallel": tokens are dispatched to the holders of
 *     their experts, run through full-size expert GEMMs, and returned by a
 *     second exchange.  On one GPU both exchanges become local permutations;
 *   - same page, section "Routing imbalance": per-expert token counts;
 *   - "Expert Parallelism for MoE Models" (apxml), section "Mechanics of Token
 *     Routing and All-to-All Communication": token representations travel to
 *     the expert and the output travels back.
 * The pages leave the arithmetic open; this library computes softmax scoring
 * of linear router logits, top-k selection (ties to the lower expert index,
 * slots in descending logit order), gates renormalised over the k selected,
 * SwiGLU experts h = silu(x Wg) * (x Wu), z = h Wd, and the gate-weighted sum.
 *
 * Conventions for every entry point
 *   - Pointers named x, w_g, ... are DEVICE pointers, 16-byte aligned, owned by
 *     the caller.  The library never allocates, frees or synchronises (except
 *     moe_check) and writes only the outputs named in each call plus `ws`.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on it.
 *   - bf16 tensors are passed as raw 16-bit patterns (moe_bf16).  All matrices
 *     are row-major and densely packed.
 *   - The return value is a moe_status.  Argument errors are detected on the
 *     host before anything is launched.  Errors found on the device (an expert
 *     index out of range, inconsistent offsets, a bounded wait that ran out) are
 *     recorded in the workspace's error word and reported by moe_check.
 *   - There is no CPU fallback: a call that would launch work returns
 *     MOE_ERR_CUDA when no CUDA device is usable and MOE_ERR_UNSUPPORTED when
 *     the current device is not an sm_100 GPU.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16; /* raw bfloat16 bits */

/* Problem statement: T tokens of hidden size d routed to k of E experts, each
 * a SwiGLU FFN with intermediate size f; R virtual expert-parallel ranks. */
typedef struct moe_shape {
  int32_t T; /* tokens in the batch, 0 <= T <= 1<<20 (T = 0 is a no-op)      */
  int32_t d; /* hidden size, a multiple of 64, 64 <= d <= 16384               */
  int32_t E; /* routed experts, 1 <= E <= 1024                                */
  int32_t k; /* experts per token, 1 <= k <= min(E, 32)                       */
  int32_t f; /* expert intermediate size, a multiple of 64, 64 <= f <= 32768  */
  int32_t R; /* virtual EP ranks: 0 or 1 = none; otherwise R divides E, R<=64 */
} moe_shape;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, shape out of range  */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but unsupported (no sm_100 device, ...)  */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed           */
  MOE_ERR_TIMEOUT = 4,      /* a bounded device wait ran out (moe_check)      */
  MOE_ERR_DEVICE_CHECK = 5  /* a device-side consistency check failed         */
} moe_status;

/* Human-readable name of a moe_status. Never NULL. */
MOE_API const char* moe_error_string(int status);

/* Library ABI version (major * 100 + minor): 101 adds the EPLB calls and
 * moe_dispatch_dedup; 102 the FP8-weight calls; 103 moe_ep_recv_experts and
 * FP8 weights at every batch size; 104 the FP8-activation (W8A8) calls and
 * moe_quantise_rows_e4m3 (the workspace grows by their buffers); 105
 * moe_copy, and the layer calls' y may be pinned host memory. */
MOE_API int moe_version(void);

/* Bytes of scratch workspace `ws` that moe_dispatch / moe_ffn / moe_forward
 * need for shape *s (enough for all three).  Returns 0 if *s is invalid.
 * The workspace must be 256-byte aligned.  Its first 64 bytes hold the
 * device error word and a block counter of moe_forward's routing kernel:
 * zero them once before the first call (every call leaves the counter at
 * zero again; moe_check clears the error word after reporting an error); the
 * rest needs no initialisation.  Calls sharing one workspace must not run
 * concurrently. */
MOE_API size_t moe_workspace_size(const moe_shape* s);

/* Router gate ("What is an MoE layer?": the gate scores each token).
 *   x      [T, d] bf16          hidden states
 *   w_g    [d, E] fp32          router weight
 *   bias   [E] fp32 or NULL     per-expert additive bias
 *   logits [T, E] fp32 out      logits[t,e] = sum_i x[t,i] w_g[i,e] + bias[e]
 *   ws     workspace of moe_workspace_size(s) bytes
 * Up to 256 tokens: fp32 FMA in a fixed order (a thread-block cluster splits
 * K; its partial sums meet in distributed shared memory in rank order).
 * Above 256 tokens: the tcgen05 tensor cores, with w_g split into three bf16
 * planes (hi + mid + lo = w_g to 24 significant bits) and fp32 accumulation.
 * Both orders are fixed, and moe_forward uses the same path for the same T,
 * so its internal logits equal this call's bit for bit. */
MOE_API int moe_router(const moe_bf16* x, const float* w_g, const float* bias,
                       const moe_shape* s, float* logits, void* ws, void* stream);

/* Expert selection and gates ("What is an MoE layer?": 8 of 256 experts per
 * token; "Batching ...": top-8 over 256).
 *   logits [T, E] fp32 in (finite values; NaN/Inf behaviour unspecified)
 *   idx    [T, k] int32 out     idx[t,j] = expert in slot j; slots ordered by
 *                               descending logit, ties to the lower index
 *   w      [T, k] fp32 out      w[t,j] = exp(L[idx[t,j]] - L[idx[t,0]]) /
 *                               sum_j' exp(L[idx[t,j']] - L[idx[t,0]]), i.e. the
 *                               softmax over E renormalised over the k chosen. */
MOE_API int moe_topk(const float* logits, const moe_shape* s, int32_t* idx, float* w,
             void* stream);

/* Dispatch: the local form of the token exchange ("Tensor parallel vs expert
 * parallel"; "Mechanics of Token Routing ...").  Rows of the expert-major
 * buffer are ordered by (expert, token) ascending.
 *   idx          [T, k] int32 in   expert ids; each in [0, E), distinct per token
 *   x            [T, d] bf16 in
 *   counts       [E] int32 out     rows per expert ("Routing imbalance")
 *   offsets      [E+1] int32 out   exclusive prefix sum, offsets[E] = T*k
 *   perm         [T*k] int32 out   perm[row] = token
 *   row_of       [T, k] int32 out  row_of[t,j] = row of (t, j)
 *   x_perm       [T*k, d] bf16 out x_perm[row] = x[perm[row]]
 *   send_counts  [R, R] int32 out or NULL (needs R > 1): S[s][r] = rows that
 *                source rank s = t / ceil(T/R) sends to the rank r = e/(E/R)
 *                owning the expert ("Expert Parallelism: keep specialists
 *                whole": contiguous expert blocks per device)
 *   rank_offsets [R+1] int32 out or NULL: first row of each rank; rank r's
 *                buffer is x_perm[rank_offsets[r] : rank_offsets[r+1]]
 *   ws           workspace of moe_workspace_size(s) bytes
 * An out-of-range expert id is recorded as MOE_ERR_DEVICE_CHECK.           */
MOE_API int moe_dispatch(const int32_t* idx, const moe_bf16* x, const moe_shape* s,
                 int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* row_of, moe_bf16* x_perm, int32_t* send_counts,
                 int32_t* rank_offsets, void* ws, void* stream);

/* Expert FFNs over the expert-major rows ("full-size expert GEMMs"):
 * for the rows r in [offsets[e], offsets[e+1]) of expert e,
 *   h = silu(x_perm[r] Wg_e) * (x_perm[r] Wu_e)   (fp32 accumulate, h in bf16)
 *   z[r] = h Wd_e                                  (fp32 accumulate, bf16 out)
 *   x_perm [T*k, d] bf16 in
 *   offsets [E+1] int32 in      device-resident; monotone, offsets[E] = T*k
 *   w13    [E, 2f, d] bf16 in   rows 0..f-1 = Wg_e^T, rows f..2f-1 = Wu_e^T
 *   w2     [E, d, f] bf16 in    Wd_e^T
 *   z      [T*k, d] bf16 out
 *   ws     workspace of moe_workspace_size(s) bytes
 * Runs on the tcgen05 tensor cores with TMA-fed operands: up to 256 tokens
 * with the weights as the 128-row MMA operand and the expert's tokens as N;
 * larger batches with 128-row token tiles, on 2-CTA clusters (256 x 256
 * tiles) once experts average at least 128 rows.  Bad offsets are recorded
 * as MOE_ERR_DEVICE_CHECK.                                                 */
MOE_API int moe_ffn(const moe_bf16* x_perm, const int32_t* offsets,
            const moe_bf16* w13, const moe_bf16* w2, const moe_shape* s,
            moe_bf16* z, void* ws, void* stream);

/* Combine: the return exchange plus the gate-weighted sum ("Tensor parallel
 * vs expert parallel": results are sent back by a second exchange),
 *   y[t] = sum_{j<k} w[t,j] * z[row_of[t,j]], summed in fp32 in slot order.
 *   z [T*k, d] bf16 in; row_of [T, k] int32 in; w [T, k] fp32 in;
 *   y [T, d] bf16 out.  Row indices out of range make y undefined. */
MOE_API int moe_combine(const moe_bf16* z, const int32_t* row_of, const float* w,
                const moe_shape* s, moe_bf16* y, void* stream);

/* The whole layer: router, selection, dispatch, expert FFNs, combine, in one
 * stream-ordered sequence with no host synchronisation (capturable in a CUDA
 * graph).  Inputs as above; y [T, d] bf16 out.  idx_out [T,k], w_out [T,k]
 * and counts_out [E] receive the routing decisions when non-NULL.  With
 * s->R > 1 the send-count matrix and rank offsets are computed too (in the
 * workspace).  ws: moe_workspace_size(s) bytes.  y may be device memory or
 * host memory the device addresses directly (page-locked, e.g. from
 * cudaHostAlloc): the combine then writes the result across the bus itself,
 * so no separate device-to-host copy is needed; pageable host memory is
 * rejected with MOE_ERR_INVALID_ARG (this and moe_forward_fp8 / _w8a8). */
MOE_API int moe_forward(const moe_bf16* x, const float* w_g, const float* bias,
                const moe_bf16* w13, const moe_bf16* w2, const moe_shape* s,
                moe_bf16* y, int32_t* idx_out, float* w_out,
                int32_t* counts_out, void* ws, void* stream);

/* moe_forward with stage timing: the same launches on the same stream, plus
 * cudaEventRecord(events[i], stream) at the stage boundaries so a caller can
 * time each stage with CUDA events inside a timed region (or a graph):
 *   events[0] before the router        events[3] after expert GEMM1 (+SwiGLU)
 *   events[1] after the router         events[4] after expert GEMM2
 *   events[2] after top-k, dispatch    events[5] after the combine
 *             tables and row gather
 * `events` points to MOE_STAGE_EVENTS cudaEvent_t handles (any may be NULL,
 * then it is skipped).  The records use cudaEventRecordExternal, so under
 * stream capture they become event-record nodes that fire on every replay.
 * Routing outputs stay in the workspace. */
#define MOE_STAGE_EVENTS 6
MOE_API int moe_forward_staged(const moe_bf16* x, const float* w_g, const float* bias,
                               const moe_bf16* w13, const moe_bf16* w2,
                               const moe_shape* s, moe_bf16* y, void* ws,
                               void* const* events, void* stream);

/* Dispatch without a workspace.  No counterpart in the pages: this is a
 * library convenience for callers that cannot allocate device memory when
 * they dispatch -- code running after a fixed memory pool has been carved
 * out, runtimes that only hand a plugin its inputs and outputs, or hosts
 * whose allocator may not be called from the dispatching thread.
 * Same arguments, layout and results as moe_dispatch, minus `ws`: the
 * per-block histograms, bases, send counts, tile list and error word live in
 * one file-scope device array of MOE_NOALLOC_SCRATCH bytes, which every GPU
 * that loads the library holds until the process exits.  The call allocates
 * nothing (no cudaMalloc / cudaFree, no allocating library routine).
 *   - A shape whose scratch would exceed MOE_NOALLOC_SCRATCH is rejected with
 *     MOE_ERR_UNSUPPORTED before anything is launched (e.g. T = 16384,
 *     E = 256, R = 8 needs about 160 KB; T = 1<<20 with E = 256 does not fit).
 *   - The first call on a device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress) and caches it for the life
 *     of the process; make that first call before any stream capture.  A
 *     cudaDeviceReset (or anything else that destroys the device's primary
 *     context) invalidates the cached address: after one, unload and reload
 *     the library before calling this entry point again.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     the error word is cleared at the start of each call and the rest is
 *     rewritten.  Calls that overlap on the GPU (other streams, other threads)
 *     race on it and must be serialised by the caller.
 *   - There is no error word to read back: rejected expert ids (out of range
 *     or repeated within a token) are not counted, so they show as
 *     offsets[E] < T*k. */
#define MOE_NOALLOC_SCRATCH (2u << 20)
MOE_API int moe_dispatch_noalloc(const int32_t* idx, const moe_bf16* x, const moe_shape* s,
                                 int32_t* counts, int32_t* offsets, int32_t* perm,
                                 int32_t* row_of, moe_bf16* x_perm, int32_t* send_counts,
                                 int32_t* rank_offsets, void* stream);

/* Token-deduplicated per-rank dispatch ("Serving MoE models with expert
 * parallelism on 8xH200", section "Tensor parallel vs expert parallel";
 * "Expert Parallelism for MoE Models", section "Mechanics of Token Routing
 * and All-to-All Communication": a token's representation travels to the
 * devices holding its experts).  A token goes once to every virtual rank that
 * owns at least one of its k experts (owner(e) = e / (E/R), source rank
 * t / ceil(T/R)); the send buffer is rank-major with tokens ascending inside a
 * rank (the pages give no layout; this is the plainest reading).  Needs
 * s->R >= 2.  rows = T * min(k, R) bounds the buffer.
 *   idx          [T, k] int32 in    expert ids
 *   x            [T, d] bf16 in     (only read when x_dedup != NULL)
 *   send_counts  [R, R] int32 out   tokens source rank s sends to rank r
 *   rank_offsets [R+1] int32 out    first row of each destination rank;
 *                                   rank_offsets[R] = rows used
 *   token_of     [rows] int32 out   token of each row
 *   slot_mask    [rows] uint32 out  bit j: slot j's expert is on that rank
 *   rank_row_of  [T, R] int32 out or NULL: row of (t, r), -1 if none
 *   x_dedup      [rows, d] bf16 out or NULL: x[token_of[row]]
 *   ws           workspace of moe_workspace_size(s) bytes
 * Out-of-range ids are recorded as MOE_ERR_DEVICE_CHECK and skipped.      */
MOE_API int moe_dispatch_dedup(const int32_t* idx, const moe_bf16* x, const moe_shape* s,
                               int32_t* send_counts, int32_t* rank_offsets,
                               int32_t* token_of, uint32_t* slot_mask,
                               int32_t* rank_row_of, moe_bf16* x_dedup, void* ws,
                               void* stream);

/* Receive side of a real expert-parallel exchange ("Serving MoE models with
 * expert parallelism on 8xH200", section "Tensor parallel vs expert
 * parallel": tokens travel to the devices holding their experts and the
 * results travel back; "Wide Expert Parallelism", section "All-to-all
 * communication: the essential tradeoff").  With R ranks each owning E_loc =
 * E / R whole experts, every rank dispatches its own tokens with moe_dispatch
 * (s->R = R): its expert-major buffer is then rank-contiguous, and the slice
 * for rank r is ordered by r's local expert.  After an all-to-all-v of those
 * slices (and of the per-expert counts), rank r holds rows ordered by
 * (source rank, local expert, token).  This call labels each received row
 * with its local expert, so that moe_dispatch with k = 1 and these labels as
 * ids regroups the rows expert-major (rows of one expert across all sources
 * contiguous, source-ascending) for moe_ffn.
 *   recv_counts   [R, E_loc] int32 in (device): rows source s sent for local
 *                 expert e (the slices of each source's `counts`)
 *   N             rows received (host-known; the sum of recv_counts)
 *   expert_of_row [N] int32 out: local expert in [0, E_loc) of each row
 * R <= 64, R * E_loc <= 1024.  Rows beyond the counts' total, or every row
 * when a count is negative, get -1; moe_dispatch then reports them as
 * MOE_ERR_DEVICE_CHECK.  Allocates nothing; no workspace. */
MOE_API int moe_ep_recv_experts(const int32_t* recv_counts, int32_t R, int32_t E_loc,
                                int32_t N, int32_t* expert_of_row, void* stream);

/* ---------------------------------------------------------------------------
 * Expert load balancing with replicated experts ("Serving MoE models with
 * expert parallelism on 8xH200", section "Routing imbalance": the busiest
 * experts get extra copies on devices with spare capacity and busy and idle
 * experts share devices; "vLLM Expert Parallel deployment", EPLB section:
 * the load is taken over a window of steps, the number of extra copies is a
 * setting).
 * The pages give no algorithm; these calls implement the plainest integer
 * reading (the oracle's tests/golden/eplb_worked_examples.json cases are
 * worked by hand from it):
 *   1. each expert starts with one copy; n_redundant times the expert with
 *      the largest load per copy gets another (ties: lower id);
 *   2. replica i of expert e is credited load[e] / n_e, plus one if
 *      i < load[e] mod n_e;
 *   3. by decreasing credit (ties: lower expert, then lower replica) each
 *      replica goes to the least-loaded rank with a free slot (ties: lower
 *      rank); rank r owns physical experts r*S .. r*S+S-1, S = P / R, in the
 *      order they were filled;
 *   4. slot j of token t with logical expert e uses replica t mod n_e.
 * ------------------------------------------------------------------------- */

/* The replica plan, on the host (no device work, no allocation).
 *   load            [E] int64 host in   per-expert load, 0 .. 2^50 (e.g. the
 *                                       counts of moe_forward over a window)
 *   E, R            logical experts, ranks (1 .. 64)
 *   n_redundant     extra copies; P = E + n_redundant <= 1024, P % R == 0
 *   phys_to_logical [P] int32 host out  logical expert of each physical slot
 *   rep_offsets     [E+1] int32 host out  replicas of e are
 *   rep_phys        [P] int32 host out    rep_phys[rep_offsets[e] .. rep_offsets[e+1])
 * Returns MOE_ERR_INVALID_ARG for null pointers or out-of-range arguments. */
MOE_API int moe_eplb_plan(const int64_t* load, int32_t E, int32_t R, int32_t n_redundant,
                          int32_t* phys_to_logical, int32_t* rep_offsets,
                          int32_t* rep_phys);

/* Logical -> physical expert ids (rule 4), on the device:
 *   idx [T, k] int32 in (logical ids < s->E); rep_offsets [s->E + 1],
 *   rep_phys [E_phys] int32 in, device-resident (moe_eplb_plan's output);
 *   idx_phys [T, k] int32 out.  ws: only its error word is used.
 * An id or plan entry out of range gives -1 and MOE_ERR_DEVICE_CHECK. */
MOE_API int moe_eplb_remap(const int32_t* idx, const moe_shape* s, const int32_t* rep_offsets,
                           const int32_t* rep_phys, int32_t E_phys, int32_t* idx_phys,
                           void* ws, void* stream);

/* Workspace bytes for moe_forward_eplb (0 if the arguments are invalid). */
MOE_API size_t moe_workspace_size_eplb(const moe_shape* s, int32_t E_phys);

/* The layer with replicated experts: router and top-k over the s->E logical
 * experts (as moe_forward), every selection mapped to its replica (rule 4),
 * then dispatch, expert FFNs and combine over the E_phys physical experts.
 *   w13_phys [E_phys, 2f, d], w2_phys [E_phys, d, f]: the weights of
 *     physical expert p are those of logical expert phys_to_logical[p]
 *     (the caller lays them out when it adopts a plan).
 *   idx_out / w_out: logical ids and gates; counts_out [E_phys]: rows per
 *     physical expert.  With s->R > 1, rank r owns physical experts
 *     [r*E_phys/R, (r+1)*E_phys/R) in the virtual-EP layout.
 * Replicas hold the same weights and every output row depends only on its own
 * token, so y equals moe_forward's y; bit for bit whenever both pick the same
 * expert-GEMM kernels (always up to 256 tokens; above, the CTA-pair choice
 * depends on rows per expert, which replicas lower).
 * ws: moe_workspace_size_eplb(s, E_phys) bytes, first 64 bytes zeroed once. */
MOE_API int moe_forward_eplb(const moe_bf16* x, const float* w_g, const float* bias,
                             const moe_bf16* w13_phys, const moe_bf16* w2_phys,
                             const moe_shape* s, const int32_t* rep_offsets,
                             const int32_t* rep_phys, int32_t E_phys, moe_bf16* y,
                             int32_t* idx_out, float* w_out, int32_t* counts_out, void* ws,
                             void* stream);

/* FP8 expert weights ("Serving MoE models with expert parallelism on
 * 8xH200", sections "Memory math for 8xH200" and "Quantization choices":
 * native FP8 checkpoints store one byte per weight; the small-batch expert
 * GEMMs are bound by reading them).  The pages fix no encoding; this library
 * takes OCP FP8 E4M3 codes (bias 7, subnormals at exponent 0, S.1111.111 is
 * NaN, no infinities) with one fp32 scale per weight row:
 *   w13   [E, 2f, d] uint8 in   E4M3 codes, rows as moe_ffn's w13
 *   w13_scale [E, 2f] fp32 in   W13[e, r, c] = e4m3(w13[e, r, c]) * w13_scale[e, r]
 *   w2    [E, d, f] uint8 in    E4M3 codes, rows as moe_ffn's w2
 *   w2_scale  [E, d] fp32 in    W2[e, r, c] = e4m3(w2[e, r, c]) * w2_scale[e, r]
 * Activations, accumulation and rounding points are those of the bf16 calls:
 * the result is moe_ffn / moe_forward on the dequantised weights (each row
 * scale multiplies the fp32 accumulator before SwiGLU / the bf16 store).
 * Code pointers 16-byte aligned, scales 4-byte aligned.  Every batch size
 * runs the weights-as-M (swap-AB) form: a converter warpgroup widens each
 * streamed e4m3 weight tile to bf16 for the tensor cores; above 64 tokens the
 * work items are 128-row token tiles of an expert, each streaming the
 * expert's (one-byte) weights again, so large batches trade repeated weight
 * reads for the halved weight bytes. */
MOE_API int moe_ffn_fp8(const moe_bf16* x_perm, const int32_t* offsets, const uint8_t* w13,
                        const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                        const moe_shape* s, moe_bf16* z, void* ws, void* stream);

/* The whole layer (as moe_forward) with FP8 expert weights (as moe_ffn_fp8). */
MOE_API int moe_forward_fp8(const moe_bf16* x, const float* w_g, const float* bias,
                            const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                            const float* w2_scale, const moe_shape* s, moe_bf16* y,
                            int32_t* idx_out, float* w_out, int32_t* counts_out, void* ws,
                            void* stream);

/* moe_forward_fp8 with the stage events of moe_forward_staged. */
MOE_API int moe_forward_fp8_staged(const moe_bf16* x, const float* w_g, const float* bias,
                                   const uint8_t* w13, const float* w13_scale,
                                   const uint8_t* w2, const float* w2_scale,
                                   const moe_shape* s, moe_bf16* y, void* ws,
                                   void* const* events, void* stream);

/* FP8 activations too (the W8A8 layer): both operands of both expert GEMMs
 * are E4M3, so the tensor cores multiply one-byte codes (tcgen05 kind::f8f6f4)
 * and the bytes streamed per weight are those of the codes alone.  The pages
 * fix no activation format; this library's reading: each activation row gets
 * one power-of-two scale and round-to-nearest-even codes, as
 * moe_quantise_rows_e4m3 defines.  The token rows are quantised as they are
 * gathered; GEMM1's SwiGLU output is rounded to bf16 (as in moe_ffn), then
 * quantised row by row; each fp32 accumulator is multiplied by its weight
 * row's scale and its token row's scale before SwiGLU / the bf16 store.
 * Weights, scales, alignment and outputs as moe_ffn_fp8 / moe_forward_fp8;
 * d and f multiples of 64 as everywhere (a K block of 128 codes past the
 * end reads zeros).  Every batch size runs the swap-AB form (touched-expert
 * items up to 64 tokens, 128-row token tiles above).
 * moe_ffn_w8a8 quantises x_perm's P = T*k rows itself. */
MOE_API int moe_ffn_w8a8(const moe_bf16* x_perm, const int32_t* offsets, const uint8_t* w13,
                         const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                         const moe_shape* s, moe_bf16* z, void* ws, void* stream);

MOE_API int moe_forward_w8a8(const moe_bf16* x, const float* w_g, const float* bias,
                             const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                             const float* w2_scale, const moe_shape* s, moe_bf16* y,
                             int32_t* idx_out, float* w_out, int32_t* counts_out, void* ws,
                             void* stream);

/* moe_forward_w8a8 with the stage events of moe_forward_staged (the SwiGLU
 * output's quantisation falls in the GEMM2 stage). */
MOE_API int moe_forward_w8a8_staged(const moe_bf16* x, const float* w_g, const float* bias,
                                    const uint8_t* w13, const float* w13_scale,
                                    const uint8_t* w2, const float* w2_scale,
                                    const moe_shape* s, moe_bf16* y, void* ws,
                                    void* const* events, void* stream);

/* Row quantisation of bf16 activations to E4M3 with power-of-two scales:
 *   a      [rows, cols] bf16 in (finite values; non-finite rows unspecified)
 *   codes  [rows, cols] uint8 out   E4M3 codes
 *   scales [rows] fp32 out          2^e_r
 * e_r is the smallest integer with max_c |a[r,c]| <= 448 * 2^e_r (0 for a
 * row of zeros), and codes[r,c] the E4M3 value nearest to a[r,c] * 2^-e_r,
 * ties to the even code; the sign bit is a's, also for values that round to
 * zero.  a * 2^-e_r is exact, so the codes depend on a alone.  cols a
 * multiple of 16 (16 to 2^20); a and codes 16-byte aligned, scales 4-byte.
 * One warp per row; asynchronous on `stream`. */
MOE_API int moe_quantise_rows_e4m3(const moe_bf16* a, int64_t rows, int32_t cols,
                                   uint8_t* codes, float* scales, void* stream);

/* Copy of `bytes` bytes from src to dst by a kernel on `stream`, in the
 * library's launch chain: the next library kernel may launch while it runs
 * and waits for it (so a captured graph goes from the copy into the layer
 * without a copy-engine node between them).  Either pointer may be device
 * memory or host memory the device addresses directly (page-locked); both
 * 16-byte aligned, bytes a multiple of 16.  Pageable host memory, a NULL or
 * misaligned pointer or a size that is not a multiple of 16 give
 * MOE_ERR_INVALID_ARG; overlapping ranges are undefined.  bytes == 0 does
 * nothing. */
MOE_API int moe_copy(void* dst, const void* src, int64_t bytes, void* stream);

/* Self-test of the failure path every device-side wait uses: launches one
 * kernel that waits on a barrier nothing will ever complete, through the same
 * bounded wait as the expert-GEMM pipeline, with a limit of limit_ns
 * (1 .. 1e9 ns).  The wait gives up, the kernel records MOE_ERR_TIMEOUT in
 * the error word of `ws` (at least 64 bytes, 256-byte aligned) and returns;
 * moe_check then reports it.  Nothing hangs or traps. */
MOE_API int moe_selftest_bounded_wait(long long limit_ns, void* ws, void* stream);

/* Synchronises `stream`, returns the device error word recorded in `ws`
 * (MOE_OK if none) and clears it. */
MOE_API int moe_check(void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
