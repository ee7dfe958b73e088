/*
 * colibri.h -- C ABI of the B200 (sm_100a) MoE layer forward.
 *
 * One call runs the four stages of a sparse Mixture-of-Experts FFN layer:
 *   Gate     router logits x . Wr^T (+ b), softmax, top-k with lowest-index tie-break
 *   Scatter  per-expert histogram, prefix sum, stable permutation of token rows
 *   Expert   grouped SwiGLU FFN per expert: W2_e (silu(W1_e x) * (W3_e x))
 *   Gather   y[t] = sum_j w[t][j] * FFN_{idx[t][j]}(x_t)  (+ shared expert FFN(x_t))
 *
 * The method is the one the "Colibri" MoE engine pages describe:
 *   www.0539edu.com/news/4774449  §2.2 (Gate -> Scatter -> Expert Compute -> Gather, one custom
 *                                 kernel per stage; expert weights stored contiguously per expert)
 *   www.hotelren.com/news/4731937 §2.1 (router logits, top-k, dispatch, k GEMMs, weighted sum),
 *                                 §2.3 (init / infer / free C API over plain structs)
 *   www.mhpq.cn/news/563172       §2.1 (fixed stride per expert), §3.2 (top-k scan, ties keep
 *                                 the lower index), §4.3 (colibri_get_error)
 *   www.pptc.cn/news/100465       §3.3 (expert_offsets over one weight buffer), §3.4 ([batch][k]
 *                                 routing layout), §4.1 (colibri_moe_forward over device pointers)
 *   www.trdm.cn/news/555962       §6.2 (group tokens by the expert they activate)
 *
 * Conventions for every entry point
 *   - Return a colibri_status; nothing is printed unless COLIBRI_DEBUG=1 is set in the
 *     environment.  colibri_last_error() returns a one-line reason for the last failure.
 *   - Arguments are validated on the host before anything is launched.
 *   - Work is enqueued on the caller's CUDA stream (passed as void*; NULL = legacy default
 *     stream) and the call returns without synchronising, except where stated.
 *   - The caller owns every tensor it passes.  The context owns only the workspace it
 *     allocates in colibri_init and frees in colibri_free.
 *   - One context serves one forward at a time: calls that overlap on the GPU (for example on
 *     two streams) share the workspace and race.
 *   - Not re-entrant from several host threads on one context.
 */
#ifndef COLIBRI_H_
#define COLIBRI_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  COLIBRI_OK = 0,
  COLIBRI_ERR_INVALID_ARG = -1, /* NULL pointer, size out of range, bad dtype combination    */
  COLIBRI_ERR_ALIGNMENT = -2,   /* a tensor is not 16-byte aligned                           */
  COLIBRI_ERR_UNSUPPORTED = -3, /* valid request the library does not implement              */
  COLIBRI_ERR_OOM = -4,         /* workspace allocation failed in colibri_init               */
  COLIBRI_ERR_CUDA = -5,        /* a CUDA runtime/driver call or a launch failed             */
  COLIBRI_ERR_TIMEOUT = -6      /* a device-side wait gave up (reported by colibri_sync_status) */
} colibri_status;

typedef enum { COLIBRI_F32 = 0, COLIBRI_BF16 = 1, COLIBRI_I8 = 2, COLIBRI_I4 = 3 } colibri_dtype;

/* Layout of the int8 weight scales (colibri_desc.weight_scale_mode). */
typedef enum {
  COLIBRI_SCALE_PER_CHANNEL = 0,  /* per expert e at e * (2f + d): s1[f] | s3[f] | s2[d] (one fp32
                                     per output channel of W1, W3, W2)                          */
  COLIBRI_SCALE_PER_MATRIX = 1    /* per expert e at 3 * e: s1 | s3 | s2, one fp32 per weight
                                     matrix (www.0539edu.com/news/4774449 §3.1: a scale computed
                                     for each expert weight matrix, symmetric int8)            */
} colibri_scale_mode;

/* Router variants, OR-ed into colibri_desc.router_flags (0 = the default router). */
typedef enum {
  COLIBRI_ROUTER_CLAMP = 1,       /* clamp every logit to [-50, 50] before selection and
                                     weighting (www.0539edu.com/news/4774449 §5.2, the
                                     gate-softmax clip option against overflow)              */
  COLIBRI_ROUTER_RAW_WEIGHTS = 2  /* combine weights = the k chosen logits themselves, no
                                     softmax (www.hotelren.com/news/4731937 §3.2)             */
} colibri_router_flag;

/*
 * Layer description, fixed for the life of a context.
 *   d_model, d_ff   hidden size d and routed-expert FFN size f; both multiples of 64.
 *   num_experts     E, 1..256.
 *   top_k           k, 1..min(E, 8).
 *   shared_d_ff     f_s of one always-on shared SwiGLU expert added with weight 1, or 0 for
 *                   none; a multiple of 64 (www.0539edu.com/news/4774449 §2.2 names the
 *                   shared-expert-augmented variant).
 *   act_dtype       dtype of x, router weights and y: COLIBRI_F32 or COLIBRI_BF16.
 *   weight_dtype    dtype of the expert weights.  Supported pairs (act, weight):
 *                   (F32, F32)   fp32 throughout (SIMT FMA; no TF32);
 *                   (BF16, BF16) bf16 operands, fp32 accumulation on tcgen05 tensor cores;
 *                   (BF16, I8)   int8 weights with per-output-channel fp32 scales,
 *                                dequantised inside the kernel (weight-streaming path).
 *                   (BF16, I4)   int4 weights, two per byte along the input dimension, with
 *                                one fp32 scale per output channel and group of 128 inputs
 *                                (www.mhpq.cn/news/563172 §4.2: INT4 packed in INT32, group
 *                                size 128; www.trdm.cn/news/555962 §6.1: two 4-bit weights per
 *                                byte); d_model and d_ff multiples of 128.
 *                   The shared expert is available for (F32, F32) and (BF16, BF16).
 *   max_tokens      largest T a forward may be called with (sizes the workspace).
 *   device_id       CUDA device the context lives on.
 *   router_flags    0, or COLIBRI_ROUTER_* bits.  Default: weights are the softmax over all E
 *                   logits renormalised over the k chosen.  Selection (logit descending, lower
 *                   expert index on ties) is the same for every variant, applied to the clamped
 *                   logits when COLIBRI_ROUTER_CLAMP is set (logits above 50 then tie and go to
 *                   the lower index).  Unknown bits: COLIBRI_ERR_INVALID_ARG.
 *   weight_scale_mode  COLIBRI_I8 weights: COLIBRI_SCALE_PER_CHANNEL (0) or
 *                   COLIBRI_SCALE_PER_MATRIX; must be 0 for other weight types (INVALID_ARG).
 *                   W[o][i] = s * q[o][i] with s the channel's or the matrix's scale.
 */
typedef struct {
  int32_t d_model;
  int32_t d_ff;
  int32_t num_experts;
  int32_t top_k;
  int32_t shared_d_ff;
  int32_t act_dtype;
  int32_t weight_dtype;
  int32_t max_tokens;
  int32_t device_id;
  int32_t router_flags;
  int32_t weight_scale_mode;
} colibri_desc;

typedef struct colibri_ctx colibri_ctx; /* opaque */

/*
 * colibri_init -- validate *desc, allocate the device workspace for max_tokens tokens on
 * desc->device_id and return a context in *out.  (www.hotelren.com/news/4731937 §2.3, §4.3:
 * init / infer / free.)  Blocking.  On failure *out is set to NULL and nothing is leaked.
 * Errors: INVALID_ARG (NULL pointers, sizes out of range), UNSUPPORTED (dtype pair,
 * shared expert with int8 weights, device not sm_100), OOM, CUDA.
 */
colibri_status colibri_init(const colibri_desc* desc, colibri_ctx** out);

/*
 * colibri_expert_stride -- elements between the starts of consecutive experts in the expert
 * weight buffer: 3 * d_model * d_ff rounded up to a multiple of 128 (of 256 for int4, whose
 * elements are half a byte), so every expert starts at least 128-byte aligned.  (www.mhpq.cn/news/563172 §2.1: each expert occupies a fixed
 * stride, address = id * EXPERT_SIZE.)  Returns -1 for a NULL context.
 */
int64_t colibri_expert_stride(const colibri_ctx* ctx);

/*
 * colibri_moe_forward -- y = MoE(x) for T tokens.  (www.pptc.cn/news/100465 §4.1.)
 *
 *   x            [T, d_model] row-major, act_dtype.  Device memory, or host memory (pinned or
 *                pageable): host x is copied into one of two workspace staging buffers, on a
 *                copy stream of the context, which `stream` then waits for.  That copy may start
 *                before work enqueued earlier on `stream` has finished (it overlaps the previous
 *                call's compute), so host x must hold its data when the call is made.
 *   T            0 <= T <= max_tokens.  T == 0 returns COLIBRI_OK and launches nothing.
 *   router_w     [E, d_model] row-major, act_dtype, device.
 *   router_b     [E] fp32 device, or NULL for no bias.
 *   expert_w     device; expert e starts at element e * colibri_expert_stride(ctx) and holds
 *                W1[f][d] | W3[f][d] | W2[d][f], each row-major with rows = output channels
 *                ([out, in]).  W1 is the gate, W3 the up and W2 the down projection.
 *   expert_scales  COLIBRI_I8: device fp32, per expert e at e * (2f + d): s1[f] | s3[f] |
 *                s2[d]; weight W[o][i] = s[o] * q[o][i] (with COLIBRI_SCALE_PER_MATRIX: at 3 * e,
 *                s1 | s3 | s2, W[o][i] = s * q[o][i]).
 *                COLIBRI_I4: device fp32, per expert e at e * 3 * d * f / 128: s1[d/128][f] |
 *                s3[d/128][f] | s2[f/128][d] (group-major); W[o][i] = s[i / 128][o] * q[o][i],
 *                where q[o][i] is the two's-complement nibble of element o * cols + i of the
 *                matrix (element 2j of the buffer in the low nibble of byte j, 2j + 1 in the high
 *                nibble; expert e starts at byte e * stride / 2).  Must be NULL for F32 / BF16.
 *   shared_w     device, W1s[f_s][d] | W3s[f_s][d] | W2s[d][f_s] in weight_dtype, when
 *                shared_d_ff > 0; must be NULL otherwise.
 *   y            [T, d_model] act_dtype, device or host; fully overwritten.  Host y is written
 *                by a device-to-host copy on a copy stream of the context that `stream` waits
 *                for; it is valid once `stream` has been synchronised.  (With
 *                COLIBRI_STAGED=0, or while `stream` is being captured into a graph, both copies
 *                run on `stream` itself, through one staging pair.)
 *   stream       cudaStream_t.
 * Every device pointer must be 16-byte aligned.  Errors: INVALID_ARG, ALIGNMENT, CUDA.
 * A device-side wait that gives up is reported later by colibri_sync_status().
 * When x and y are device memory, `stream` is not the legacy default stream, COLIBRI_PROFILE
 * printing is off and the stream is not itself being captured, the launch sequence is captured into a
 * CUDA graph the first time a given argument set is seen and replayed on later calls with the
 * same arguments (up to 8 argument sets per context; COLIBRI_GRAPHS=0 disables this).
 * With COLIBRI_PROFILE=1 in the environment the call records CUDA events per stage,
 * synchronises the stream and prints one line "Gate | Scatter | ExpertCompute | Gather |
 * Total" in milliseconds to stderr (the stage profile of www.0539edu.com/news/4774449 §3.3).
 */
colibri_status colibri_moe_forward(colibri_ctx* ctx, const void* x, int32_t T,
                                   const void* router_w, const float* router_b,
                                   const void* expert_w, const float* expert_scales,
                                   const void* shared_w, void* y, void* stream);

/*
 * colibri_moe_forward_routed -- the same layer with routing supplied by the caller: stages
 * Scatter, Expert and Gather only.  (www.pptc.cn/news/100465 §2.3 pluggable routing function,
 * §4.1 forward over precomputed d_routing, §3.4 [batch][k] layout.)
 *   topk_idx     [T, k] int32 device, expert ids in [0, E), k distinct per token.
 *   topk_w       [T, k] fp32 device, the weight of each slot.
 * Other arguments as colibri_moe_forward.  Ids are not checked on the device beyond being
 * clamped into [0, E) for addressing; out-of-range or repeated ids give unspecified y but no
 * out-of-bounds access.
 */
colibri_status colibri_moe_forward_routed(colibri_ctx* ctx, const void* x, int32_t T,
                                          const int32_t* topk_idx, const float* topk_w,
                                          const void* expert_w, const float* expert_scales,
                                          const void* shared_w, void* y, void* stream);

/*
 * colibri_get_routing -- enqueue device-to-device copies of the routing state of the last
 * forward on this context into caller buffers (any pointer may be NULL to skip it).  The pages
 * have no counterpart of this call: it exposes the Gate and Scatter results (whose layouts follow
 * www.pptc.cn/news/100465 §3.3-§3.4 and www.trdm.cn/news/555962 §6.2) for parity checks.
 *   topk_idx [T, k] int32   chosen experts, slot 0 = largest logit
 *   topk_w   [T, k] fp32    renormalised softmax weights
 *   counts   [E]    int32   rows per expert
 *   offsets  [E+1]  int32   exclusive prefix sum of counts
 *   src_row  [T*k]  int32   token of each grouped row (ascending token within an expert)
 *   dst_row  [T, k] int32   grouped row of each (token, slot)
 * T is the last forward's T.  Errors: INVALID_ARG (no forward yet), CUDA.
 */
colibri_status colibri_get_routing(colibri_ctx* ctx, int32_t* topk_idx, float* topk_w,
                                   int32_t* counts, int32_t* offsets, int32_t* src_row,
                                   int32_t* dst_row, void* stream);

/*
 * colibri_combine -- the Gather stage alone (www.pptc.cn/news/100465 §2.1 k-way aggregation;
 * www.hotelren.com/news/4731937 §2.3 combine_kernel): y[t] = sum_{j<k} topk_w[t][j] *
 * Yp[dst_row[t][j]], summed in slot order in fp32 and rounded once to act_dtype.  For callers
 * whose expert outputs come from elsewhere, e.g. the expert-parallel layer, where the grouped
 * rows were computed on the GPUs that own the experts and sent back.
 *   Yp       [rows, d_model] act_dtype, the expert outputs of the grouped rows.
 *   dst_row  [T, k] int32, grouped row of each (token, slot); topk_w [T, k] fp32.
 *   y        [T, d_model] act_dtype, fully overwritten.
 * All buffers caller-owned device memory of the current device, 16-byte aligned; d_model a
 * multiple of 8; 1 <= k <= 8.  No context, no allocation; enqueued on `stream`.  T == 0 launches
 * nothing.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA (reason via colibri_last_error(NULL)).
 */
colibri_status colibri_combine(const void* Yp, int32_t act_dtype, const int32_t* dst_row,
                               const float* topk_w, int32_t T, int32_t top_k, int32_t d_model,
                               void* y, void* stream);

/*
 * colibri_sync_status -- synchronise `stream`, then read and clear the context's device
 * error word.  Returns COLIBRI_ERR_TIMEOUT if a kernel's bounded wait gave up since the last
 * check (its output is then undefined), COLIBRI_ERR_CUDA if the stream reports an error,
 * else COLIBRI_OK.  Blocking.
 */
colibri_status colibri_sync_status(colibri_ctx* ctx, void* stream);

/*
 * Per-stage timing (www.0539edu.com/news/4774449 §3.3: enable_profiling reports the time of
 * each stage).  Between colibri_profile_begin and colibri_profile_end every forward on this
 * context records CUDA events on its own stream at the stage boundaries, without
 * synchronising.  A forward that would replay a CUDA graph still does: a second graph of the
 * same call carries event-record nodes at the stage boundaries (no programmatic dependent
 * launch across them), so what is timed is the replayed launch sequence.  colibri_profile_end synchronises those events and writes, per stage, the
 * total milliseconds over the recorded calls:
 *   stage_ms[0] Gate (router logits, softmax, top-k)
 *   stage_ms[1] Scatter (histogram, prefix sum, permutation)
 *   stage_ms[2] Expert gate/up projection (+ SiLU * up)
 *   stage_ms[3] Expert down projection
 *   stage_ms[4] Gather (weighted combine)
 * and the number of calls recorded in *ncalls.  At most max_calls (1..65536) calls are
 * recorded; later calls are not timed.  Errors: INVALID_ARG, OOM (event creation), CUDA.
 */
#define COLIBRI_NUM_STAGES 5
colibri_status colibri_profile_begin(colibri_ctx* ctx, int32_t max_calls);
colibri_status colibri_profile_end(colibri_ctx* ctx, float* stage_ms, int32_t* ncalls);

/*
 * colibri_profile_calls -- after colibri_profile_end, the per-call stage times of the recorded
 * calls (same stage order, same passage as above): call_stage_ms [n][COLIBRI_NUM_STAGES] host
 * fp32 milliseconds, caller-owned, for the first n = min(max_calls, recorded calls) calls.
 * The events stay valid until the next colibri_profile_begin.  Blocking (synchronises those
 * events).  Errors: INVALID_ARG (NULL ctx or buffer, profiling still active), CUDA.
 */
colibri_status colibri_profile_calls(colibri_ctx* ctx, float* call_stage_ms, int32_t max_calls);

/*
 * colibri_route_noalloc -- the Gate and Scatter stages alone (router logits, fp32 softmax,
 * top-k, per-expert histogram, prefix sum and the stable grouping of token rows), with no
 * context and no device allocation of any kind.  The pages have no counterpart of this call;
 * it exists for callers that cannot call cudaMalloc, such as an engine whose device memory is
 * reserved up front by its own allocator (an extra allocation would fail or fragment it) or a
 * latency-critical loop that must not pay cudaMalloc's implicit synchronisation.  It runs the
 * default router (router_flags = 0).
 *   x [T, d_model] act_dtype (COLIBRI_F32 or COLIBRI_BF16), router_w [E, d_model] act_dtype,
 *   router_b [E] fp32 or NULL; outputs topk_idx/topk_w/dst_row [T, k], counts [E],
 *   offsets [E+1], src_row [T*k] and Xp [T*k, d_model] (x's rows grouped by expert, act_dtype),
 *   with the meanings of colibri_get_routing.  All buffers are caller-owned device memory of the
 *   current device, 16-byte aligned.  Work is enqueued on `stream`.
 * Limits: d_model a multiple of 64, 1 <= E <= 256, 1 <= k <= min(E, 8), and
 * ceil(T / 256) * E <= 32768 (the size of the built-in scratch array); larger sizes are
 * rejected with COLIBRI_ERR_INVALID_ARG before anything is launched.  T == 0 launches nothing.
 * The scratch is one file-scope device array (about 257 KB, held by every GPU that loads the
 * library until exit).  Each call looks up its device address on the current device and sets the
 * router kernels' shared-memory limit there; the first call on each device loads the kernels and
 * should come before any stream capture.  All calls share the array: calls that overlap on the GPU race.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA; reason via colibri_last_error(NULL).  A
 * device-side wait that gives up is reported by colibri_route_noalloc_check.
 */
colibri_status colibri_route_noalloc(const void* x, int32_t act_dtype, int32_t T, int32_t d_model,
                                     const void* router_w, const float* router_b,
                                     int32_t num_experts, int32_t top_k, int32_t* topk_idx,
                                     float* topk_w, int32_t* counts, int32_t* offsets,
                                     int32_t* src_row, int32_t* dst_row, void* Xp, void* stream);

/*
 * colibri_route_noalloc_check -- synchronise `stream` and report whether a bounded device wait
 * of the last colibri_route_noalloc call on the current device gave up (COLIBRI_ERR_TIMEOUT; its
 * outputs are then undefined).  No counterpart on the pages (see colibri_route_noalloc).  The
 * word lives in the same scratch array and is cleared by the next colibri_route_noalloc call.
 * Blocking; allocates nothing.  Errors: TIMEOUT, CUDA.
 */
colibri_status colibri_route_noalloc_check(void* stream);

/*
 * Failure-detection self test (no counterpart on the pages; it exercises the error reporting of
 * www.mhpq.cn/news/563172 §4.3).  Enqueues on `stream` one kernel whose single thread waits on a
 * device barrier that nothing ever completes, giving up after `timeout_us` microseconds
 * (1..1000000) exactly as a stalled pipeline wait of the forward kernels gives up after 4 s: it
 * sets the context's device error word and returns.  Nothing faults or hangs; the next
 * colibri_sync_status() on that stream returns COLIBRI_ERR_TIMEOUT and clears the word, and the
 * context stays usable.  Errors: INVALID_ARG (NULL ctx, timeout out of range), CUDA.
 */
colibri_status colibri_selftest_wait_timeout(colibri_ctx* ctx, int32_t timeout_us, void* stream);

/* One-line description of a status code (static storage).  No counterpart on the pages; the
 * codes are those of colibri_status above. */
const char* colibri_status_string(colibri_status status);

/* One-line reason for the last failure on this context, or on any context if ctx is NULL
 * (www.mhpq.cn/news/563172 §4.3 colibri_get_error).  Valid until the next call. */
const char* colibri_last_error(const colibri_ctx* ctx);

/* colibri_free -- release the workspace and the context (www.hotelren.com/news/4731937 §2.3,
 * §4.3: the free step of init / infer / free).  Blocking (synchronises the device's work that
 * uses the workspace).  NULL is ignored. */
void colibri_free(colibri_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* COLIBRI_H_ */
