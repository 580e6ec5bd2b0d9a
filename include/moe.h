/*
 * moe.h -- C ABI of libmoe.so, a B200 (sm_100a) implementation of the sparse
 * Mixture-of-Experts block of the Qwen3.x hybrid models.
 *
 * The block (one per layer; "Vue d'ensemble" page of the Qwen3.8-Max report,
 * section "Le motif": every layer ends in a MoE block), per token x of width d:
 *   1. a linear router scores the E experts            (Qwen3.6 explainer page,
 *   2. softmax over the E scores, keep the k largest    router paragraphs)
 *   3. renormalise the k kept probabilities to sum to 1
 *   4. each kept expert is a SwiGLU MLP                 ("Architecture" page,
 *        E_e(x) = W_down[e] (SiLU(W_gate[e] x) * (W_up[e] x))   config.json keys
 *      with intermediate width I                        hidden_act = silu,
 *                                                       moe_intermediate_size)
 *   5. one shared SwiGLU expert of width I_s is always  (Qwen3.6 explainer: one
 *      added with weight 1                              "shared" expert always on;
 *                                                       shared_expert_intermediate_size)
 *   y = sum_{e kept} w_e E_e(x) + S(x).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers into contiguous row-major
 *     buffers that the caller allocates and owns.  The library never
 *     allocates or frees device memory and never synchronises the stream.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  A return of MOE_OK means the work was enqueued.
 *   - Errors the host can see (bad sizes, NULL or misaligned pointers, a
 *     workspace that is too small) are returned before anything is launched;
 *     MOE_ERR_CUDA reports a launch error.  Faults the device sees (an expert
 *     id out of range in moe_permute's input, a pipeline wait that timed out)
 *     are recorded in a device status word that moe_device_status() reads.
 *   - moe_last_error_string() describes the last non-OK status returned on
 *     the calling thread.
 *   - Weight layout is the linear-layer convention (out x in, row-major):
 *       w_router [E, d] (activation type), w_gate [E, I, d], w_up [E, I, d],
 *       w_down [E, d, I]; shared: ws_gate [I_s, d], ws_up [I_s, d],
 *       ws_down [d, I_s].  I_s == 0 means no shared expert (ws_* ignored).
 *   - Types: activations (x, x_perm, y_perm, y) are MOE_F32 or MOE_BF16;
 *     weights are MOE_F32 (with F32 activations), MOE_BF16, or
 *     MOE_FP8_E4M3_B128 (bf16 activations; E4M3 codes with one fp32 scale per
 *     128 x 128 block: value = decode(q) * scale[row/128][col/128]).
 *   - FP8 `scales` packs, in this order: gate [E][I/128][d/128], up (same),
 *     down [E][d/128][I/128], shared gate [I_s/128][d/128], shared up (same),
 *     shared down [d/128][I_s/128].  NULL for non-FP8 weights.
 *   - Limits: 1 <= k <= min(E, 16); E <= 512; d, I, I_s multiples of 8
 *     (multiples of 128 for FP8 weights); T >= 0 with T * (k + 1) < 2^31;
 *     every pointer 16-byte aligned.
 */
#ifndef MOE_H
#define MOE_H

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

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,          /* a size, pointer or type is not allowed */
  MOE_ERR_UNSUPPORTED = 2,          /* a valid combination the library does not implement */
  MOE_ERR_ALIGNMENT = 3,            /* a pointer or a row stride is not 16-byte aligned */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes below the *_workspace_size() figure */
  MOE_ERR_CUDA = 5,                 /* a CUDA runtime call or a launch failed */
  MOE_ERR_DEVICE_CHECK = 6,         /* device status: a kernel rejected its input */
  MOE_ERR_TIMEOUT = 7               /* device status: a pipeline wait gave up */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_FP8_E4M3_B128 = 2 } moe_dtype;

/* Shapes of one block invocation.  R = T*k routed rows; R' = R + T (I_s > 0)
 * or R (I_s == 0) dispatched rows. */
typedef struct {
  int64_t T;         /* tokens */
  int32_t d;         /* hidden width */
  int32_t E;         /* routed experts */
  int32_t k;         /* experts kept per token */
  int32_t I;         /* routed expert intermediate width */
  int32_t I_s;       /* shared expert intermediate width, 0 = none */
  int32_t act_dtype; /* moe_dtype of activations and of w_router */
  int32_t w_dtype;   /* moe_dtype of expert weights */
} moe_problem;

/* Validate a problem on the host (no CUDA call).  MOE_OK or the reason. */
MOE_API moe_status moe_check_problem(const moe_problem* p);

/* Bytes of device workspace the calls below need (0 for an invalid problem).
 * moe_workspace_size covers moe_layer_forward and moe_block_forward; moe_stage_workspace_size
 * covers moe_permute and moe_expert_ffn.  Pure host functions. */
MOE_API size_t moe_workspace_size(const moe_problem* p);
MOE_API size_t moe_stage_workspace_size(const moe_problem* p);

/* Router stage (steps 1-3).  x [T, d]; w_router [E, d]; router_bias [E] fp32
 * or NULL (added to the logits before the softmax).  Writes topk_ids
 * int32 [T, k] (descending probability, equal values -> lower index) and
 * topk_w fp32 [T, k] (renormalised, each row sums to 1).  ws:
 * moe_stage_workspace_size() bytes (holds the logits; may be NULL for F32
 * problems). */
MOE_API moe_status moe_router_topk(const moe_problem* p, const void* x, const void* w_router,
                           const float* router_bias, int32_t* topk_ids, float* topk_w,
                           void* ws, size_t ws_bytes, void* stream);

/* Dispatch stage (the token is "sent to" its experts, Qwen3.6 explainer,
 * router paragraph): a stable sort of the T*k (token, slot) pairs by expert.
 * Outputs: offs int32 [E+2] (group e = rows offs[e]..offs[e+1]-1, ordered by
 * (token, slot); group E = the shared expert, every token in order);
 * row_tok int32 [R'] (source token of each row); row_w fp32 [R'] (routing
 * weight; 1 for shared rows); pos int32 [T, k] (row of pair (t, j));
 * x_perm [R', d] = x[row_tok].  ws: moe_stage_workspace_size() bytes.
 * An expert id outside [0, E) sets MOE_ERR_DEVICE_CHECK in the device status
 * and the affected pairs are dropped. */
MOE_API moe_status moe_permute(const moe_problem* p, const void* x, const int32_t* topk_ids,
                       const float* topk_w, void* x_perm, int32_t* row_tok, float* row_w,
                       int32_t* pos, int32_t* offs, void* ws, size_t ws_bytes, void* stream);

/* Expert stage (step 4 and the shared expert of step 5, unweighted):
 * y_perm[r] = E_g(x_perm[r]) for every row r of group g (g == E: shared).
 * x_perm, y_perm [R', d] in the activation type; offs as moe_permute writes
 * it.  ws: moe_stage_workspace_size() bytes. */
MOE_API moe_status moe_expert_ffn(const moe_problem* p, const void* x_perm, const int32_t* offs,
                          const void* w_gate, const void* w_up, const void* w_down,
                          const void* ws_gate, const void* ws_up, const void* ws_down,
                          const float* scales, void* y_perm, void* ws, size_t ws_bytes,
                          void* stream);

/* Combine stage (steps 3 and 5: the token's output is the kept experts'
 * outputs weighted by their renormalised router probabilities -- Qwen3.6
 * explainer, router paragraphs -- plus the always-on shared expert's output
 * with weight 1 -- Qwen3.6 explainer, shared-expert paragraph; Qwen3-Next
 * story, the shared expert that treats every input):
 *   y[t] = sum_j topk_w[t, j] * y_perm[pos[t, j]] + y_perm[offs[E] + t]
 * (the last term when I_s > 0); pairs with pos < 0 (dropped by moe_permute)
 * add nothing.  Sums in fp32 in slot order, rounded once.  y [T, d] in the
 * activation type. */
MOE_API moe_status moe_combine(const moe_problem* p, const void* y_perm, const int32_t* pos,
                       const float* topk_w, const int32_t* offs, void* y, void* stream);

/* The whole block, fused (steps 1-5 above: the router and softmax top-k of the
 * Qwen3.6 explainer's router paragraphs, the SwiGLU experts of the
 * Architecture page's config.json, the shared expert of the explainer's
 * shared-expert paragraph, summed as y = sum_{e kept} w_e E_e(x) + S(x)):
 * router + top-k, dispatch, gate/up GEMM with SwiGLU,
 * down GEMM whose epilogue applies the routing weight and stores each row in
 * (token, slot) order, then one ordered fp32 sum per token of its k slot rows
 * and its shared-expert row (reproducible: no atomics).  y [T, d] in the activation type.  topk_ids_out and
 * topk_w_out ([T, k]) may be NULL.  ws: moe_workspace_size() bytes.
 * On the row-tiled bf16 form (see moe_set_path) with T * d * 2 <= 256 MiB the
 * gate/up GEMM reads each dispatched row straight from x, and the dispatch
 * writes no copy of them. */
MOE_API moe_status moe_layer_forward(const moe_problem* p, const void* x, const void* w_router,
                             const float* router_bias, const void* w_gate, const void* w_up,
                             const void* w_down, const void* ws_gate, const void* ws_up,
                             const void* ws_down, const float* scales, void* y,
                             int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                             void* stream);

/* The block's neighbours on its input (Qwen3-Next story page: the models use
 * a "zero-centred" RMSNorm whose parameters start at zero, so the applied
 * scale is 1 + gamma; Architecture page, config.json: rms_norm_eps = 1e-6).
 *   norm_weight  gamma [d] in the activation type, 16-byte aligned, or NULL:
 *                x_n = x / sqrt(mean_j x_j^2 + norm_eps) * (1 + gamma), stored
 *                in the activation type, is the input of the router and the
 *                experts (sums in fp32);
 *   norm_eps     >= 0 and finite (1e-6 for the Qwen3.x configs);
 *   shared_gate  w [d] in the activation type, 16-byte aligned, or NULL: the
 *                shared expert's output is weighted by sigmoid(x_n . w)
 *                instead of 1.  The pages do not describe such a gate; some
 *                implementations of this block carry one.  Ignored when
 *                I_s == 0. */
typedef struct {
  const void* norm_weight;
  float norm_eps;
  const void* shared_gate;
} moe_block_options;

/* moe_layer_forward with the options above (opt NULL: exactly
 * moe_layer_forward).  Same arguments and workspace otherwise; x is the
 * block's input before the norm. */
MOE_API moe_status moe_block_forward(const moe_problem* p, const moe_block_options* opt, const void* x,
                             const void* w_router, const float* router_bias, const void* w_gate,
                             const void* w_up, const void* w_down, const void* ws_gate,
                             const void* ws_up, const void* ws_down, const float* scales, void* y,
                             int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                             void* stream);

/* The zero-centred RMSNorm of moe_block_options as a stage: x_out [T, d] =
 * x / sqrt(mean_j x_j^2 + eps) * (1 + norm_weight), in the activation type
 * (sums in fp32).  norm_weight [d] in the activation type; x, norm_weight and
 * x_out 16-byte aligned; eps >= 0 and finite. */
MOE_API moe_status moe_rmsnorm(const moe_problem* p, const void* x, const void* norm_weight, float eps,
                       void* x_out, void* stream);

/* Expert parallelism, receive side.  The block split over G ranks, rank g
 * holding experts [g * E_local, (g + 1) * E_local) (the path's experts are
 * independent, so they partition; the pages raise "how many GPUs for how many
 * parameters" only as a chapter title, Fondations page, chapter 06).  A rank's
 * dispatch leaves the rows bound for each rank contiguous and grouped by
 * expert, so the rows a rank receives are blocks (source s, local expert e) in
 * that order.  counts int32
 * [G * E_local] (device): counts[s * E_local + e] = rows from source s for
 * local expert e.  Writes ids int32 [R] (device): the local expert of each
 * received row; R = the sum of the counts, known to the caller from the count
 * exchange.  A k = 1 moe_permute on (received rows, ids) then groups the rows
 * by expert for moe_expert_ffn.
 * Errors: G or E_local < 1, G * E_local > 4096, R < 0 or > INT32_MAX ->
 * MOE_ERR_INVALID_ARG; NULL or not 16-byte aligned pointers (R > 0) ->
 * MOE_ERR_INVALID_ARG / MOE_ERR_ALIGNMENT, all before any launch.  A negative
 * count, or fewer counted rows than R (those ids are written -1), sets
 * MOE_ERR_DEVICE_CHECK in the device status. */
MOE_API moe_status moe_ep_expand_ids(const int32_t* counts, int32_t G, int32_t E_local, int64_t R,
                             int32_t* ids, void* stream);

/* moe_router_topk for callers that cannot allocate device memory: code that
 * runs where cudaMalloc is off limits (inside a host framework that owns every
 * device allocation, or on a latency-critical thread that must not enter an
 * allocator) and so cannot hand the router a workspace.  The block's pages
 * have no counterpart of this entry point; it is a property of the library.
 * Same arguments and results as moe_router_topk minus the workspace: the
 * router's logit partials go to a file-scope __device__ array of
 * MOE_ROUTER_STATIC_SCRATCH_BYTES that every device that loads the library
 * keeps until the process exits.  Nothing is allocated or freed.
 *   - Problems whose scratch needs more than that are rejected with
 *     MOE_ERR_UNSUPPORTED before anything is launched: about
 *     splits * T * roundup(E, 32) * 4 bytes of split-K partials (e.g. T = 8192
 *     with E = 512).  The router that selects in its GEMM epilogue (E <= 256,
 *     T >= 1921) uses no scratch, so it takes any T.
 *   - The first call on a device looks up that device's copy of the array
 *     (a one-time set-up); make it before any stream capture.
 *   - Every call uses the same array and leaves its contents behind; calls
 *     that overlap on the GPU (other streams, other threads) race on it and
 *     must be serialised by the caller. */
#define MOE_ROUTER_STATIC_SCRATCH_BYTES (32u << 20)
MOE_API moe_status moe_router_topk_static(const moe_problem* p, const void* x, const void* w_router,
                                  const float* router_bias, int32_t* topk_ids, float* topk_w,
                                  void* stream);

/* What moe_layer_forward / moe_block_forward launch for problem p under the
 * current moe_set_path, decided on the host (no CUDA call, no device needed):
 * expert_form: 0 SIMT kernels, 1 row-tiled tensor-core GEMMs, 2 weight-row
 * (swap-AB) GEMMs, 3 row-tiled GEMMs on CTA pairs, 4 split (CTA pairs for the
 * groups of 256 rows or more, weight-row GEMMs for the others), 5 GEMMs on CTA
 * pairs with the tokens as the MMA's N; router_selects: 1 when the
 * router's GEMM selects the top k in its epilogue (bf16, E <= 256, at least
 * 16 tiles of 128 tokens), 0 for the split-K GEMM + top-k kernel or the SIMT
 * router; gathered: 1 when the gate/up GEMM reads its rows straight from x.
 * Any output pointer may be NULL.  Errors: those of moe_check_problem, and
 * MOE_ERR_UNSUPPORTED where moe_set_path asks for a form the types do not
 * allow. */
MOE_API moe_status moe_forward_plan(const moe_problem* p, int32_t* expert_form, int32_t* router_selects,
                            int32_t* gathered);

/* Kernel-path selection for the calls above on the calling process:
 * 0 = automatic (tensor-core kernels where the types allow; for the expert
 *     GEMMs the weight-row form when T*k <= 64*E, i.e. when an expert sees at
 *     most one 64-token chunk on average, the form of 4 when bf16 experts
 *     average 2048 rows or more (T*k >= 2048*E), else the row-tiled form);
 * 1 = SIMT CUDA kernels only (fp32 FMA; the path of fp32 problems);
 * 2 = tensor-core kernels required, row-tiled expert GEMMs;
 * 3 = tensor-core kernels required, weight-row expert GEMMs;
 * 4 = tensor-core kernels required, row-tiled expert GEMMs on 2-CTA clusters
 *     (256-row tiles, tcgen05 pair MMAs; E4M3 weights take the form of 2);
 * 5 = tensor-core kernels required, split expert GEMMs: the groups of 256
 *     rows or more as in 4, the others as in 3, one launch each per
 *     projection (E4M3 weights take the form of 2).  Never chosen
 *     automatically: on skewed prefill batches the row-tiled form of 2 was
 *     faster, since it runs the small groups' tiles among the large ones;
 * 6 = tensor-core kernels required, expert GEMMs on 2-CTA clusters with the
 *     weights as the pair MMA's M = 256 operand and a tile's tokens (up to
 *     256, the count rounded up to 16) as its N (E4M3 weights take the form
 *     of 2).  Never chosen automatically: it measured no faster than 2 on
 *     the skewed prefill batch and than 4 on long groups.
 * 2 to 6 return MOE_ERR_UNSUPPORTED when the types do not allow them. */
MOE_API moe_status moe_set_path(int path);

/* Synchronously read and clear the device status word of the current device
 * (MOE_OK, MOE_ERR_DEVICE_CHECK or MOE_ERR_TIMEOUT); *detail receives the
 * raw code (which kernel and which wait), or 0.  Synchronises the device. */
MOE_API moe_status moe_device_status(int32_t* detail);

/* The bound, in SM clock cycles, of every pipeline wait in the library's
 * kernels on the current device (cycles <= 0: the default, 4e9 cycles, about
 * 2 s at B200 clocks).  A wait that passes it gives up: the kernel records
 * MOE_ERR_TIMEOUT with the kernel and the wait in the device status word,
 * drains the copies it issued (always with the default bound), releases its
 * tensor memory and returns, leaving its outputs incomplete.  A short bound
 * lets a test make waits give up on purpose and check that the kernels come
 * back and the device stays usable.  Takes effect for kernels that start
 * after the call returns; call it with no library work in flight on the
 * device (the write is a synchronous copy to device memory).  MOE_ERR_CUDA if
 * that copy fails. */
MOE_API moe_status moe_set_wait_limit(int64_t cycles);

/* 1 in the bounds-checking build of the library (libmoe_checks.so, compiled
 * with -DMOE_CHECKS), 0 otherwise.  That build checks, on the device, the
 * indices the kernels compute or read before they address memory with them:
 * the row a (token, slot) pair is dispatched to and the rows the dispatch
 * copies into, the token row a gathering GEMM reads, the (token, slot) row a
 * down GEMM's epilogue stores, and the dispatched rows moe_combine reads for
 * the caller's pos (and the shared row offs[E] + t).  An index out of range
 * skips that access and records MOE_ERR_DEVICE_CHECK with code
 * 0x08000000 | site (1 dispatched row, 2 copied row, 3 gathered token row,
 * 4 slot row, 5 combined row) in the device status word.  The normal build
 * compiles these checks away. */
MOE_API int moe_bounds_checked(void);

/* Number of kernels the last successful call on this thread launched. */
MOE_API int moe_last_launch_count(void);

/* Per-launch timing for profiling.  on = 1: every kernel the calling thread
 * launches through this library is bracketed by two CUDA events recorded on
 * its stream; on = 2: only the tensor-core GEMM launches; on = 0: off.
 * Events are created once and reused; at most 4096 launches are recorded
 * until the next read.  Every call clears the record.  A thread starts in the
 * mode the environment variable MOE_PROFILE gives (1 or 2), else off.
 * Independently of this, every entry point and every stage of the fused
 * forward (moe.router, moe.dispatch, moe.expert_gemms, moe.slot_sum) is an
 * NVTX range on the host, for nsys and for ncu's NVTX filters. */
MOE_API moe_status moe_profile_enable(int on);

/* Copy up to `max` recorded launches, in launch order, into ms[] (device
 * milliseconds, -1 if unavailable) and names[] (static strings owned by the
 * library; either array may be NULL), waiting for each launch's end event.
 * Returns the number copied and clears the record. */
MOE_API int moe_profile_read(int max, float* ms, const char** names);

MOE_API const char* moe_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
