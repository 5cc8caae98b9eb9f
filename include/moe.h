/*
 * moe.h -- C ABI of libmoe.so: the forward pass of an expert-parallel MoE layer
 * on one NVIDIA B200 (sm_100a).
 *
 * The layer follows the four-stage pipeline of "Expert Parallel (EP)" (twinkle-kit
 * docs), section Communication Pattern: router -> preprocess -> token pre-all-to-all
 * (permute) -> local experts -> token post-all-to-all (unpermute + routing weights).
 * On one GPU the all-to-all exchange becomes the permutation itself: the dispatch
 * buffer is laid out rank-major (ep_size virtual ranks, contiguous expert ranges
 * per rank) and rank_splits are exactly the exchange's per-destination split sizes.
 *
 * Conventions for every call
 *  - Memory: the caller owns all memory.  Pointers named "device" must point to
 *    device memory of the current CUDA device; the library allocates nothing in
 *    these calls and keeps no state between them.
 *  - Streams: every call only enqueues work on `stream` (0 = legacy default) and
 *    returns without synchronising.  Outputs are valid once the stream reaches
 *    that point.
 *  - Layouts: all tensors are dense row-major (C order) with the shapes given.
 *  - Errors: invalid arguments are detected on the host before anything is
 *    enqueued and returned synchronously (MOE_ERR_INVALID_ARG / _UNSUPPORTED);
 *    a failed launch returns MOE_ERR_CUDA.  Errors found on the device (an
 *    expert index out of range, a bounded wait that expired) are written to the
 *    caller's int32 `status` word (device memory, caller sets it to 0), never
 *    by trapping; outputs of that call are then unspecified.
 *  - Thread safety: calls are reentrant; concurrent calls on different streams
 *    must not share output or workspace buffers.
 *
 * Shorthand: T tokens, D model dim, E routed experts, ep = ep_size, El = E/ep,
 * k = top_k, F expert intermediate dim, R = T*k routed rows, S shared experts of
 * intermediate Fs.  "bf16" = bfloat16 storage; accumulation is always fp32.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, E % ep != 0, k out of range */
  MOE_ERR_UNSUPPORTED = 2,  /* valid MoE but outside what the kernels implement   */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed                */
  MOE_ERR_INDEX_OOB = 4,    /* device status: an expert index was outside [0, E)   */
  MOE_ERR_TIMEOUT = 5,      /* device status: a bounded wait in a kernel expired   */
  MOE_ERR_SCRATCH_LIMIT = 6 /* moe_preprocess_noalloc: config exceeds its fixed scratch */
} moe_status;

typedef enum { MOE_DT_F32 = 0, MOE_DT_BF16 = 1 } moe_dtype;
typedef enum { MOE_ACT_GELU = 0, MOE_ACT_SWIGLU = 1 } moe_act;

/* Layer configuration ("Expert Parallel (EP)", section Configuration:
 * router_dtype, ignore_shared_experts, ep_size; section Requirements). */
typedef struct {
  int32_t T;            /* tokens, >= 0                                               */
  int32_t D;            /* model dim, multiple of 64                                  */
  int32_t E;            /* routed experts, 1..1024                                    */
  int32_t ep_size;      /* virtual EP ranks; E % ep_size == 0 (section Requirements)  */
  int32_t top_k;        /* 1..min(E, 32)                                              */
  int32_t F;            /* expert intermediate dim: multiple of 128 (SwiGLU) or 64 (GELU) */
  int32_t act;          /* moe_act                                                     */
  int32_t renormalize;  /* 1: weights renormalised over the top-k (sum to 1); 0: plain softmax over E */
  int32_t x_dtype;      /* moe_dtype of x, residual and out                           */
  int32_t router_dtype; /* must be MOE_DT_F32 (the fp32 router)                        */
  int32_t n_shared;     /* S always-on shared SwiGLU experts; 0 = none (ignore_shared_experts) */
  int32_t F_shared;     /* Fs, multiple of 128 when n_shared > 0                      */
} moe_config;

/* Returns MOE_OK if `cfg` is a configuration the kernels implement, else the
 * reason.  Pure host check, needs no GPU. */
MOE_API moe_status moe_validate_config(const moe_config* cfg);

/* Bytes of scratch a caller must pass as `workspace` to moe_route,
 * moe_preprocess, moe_expert_ffn and moe_forward (one buffer serves all of them,
 * 256-byte aligned).  Holds the fp32 logits when the caller keeps none, the
 * preprocess block histograms, the per-expert GEMM tile prefix and the shared
 * experts' activations.  0 for an invalid config. */
MOE_API size_t moe_workspace_size(const moe_config* cfg);

/* Bytes of the prepacked weight buffer written by moe_prepare_weights. */
MOE_API size_t moe_packed_weights_size(const moe_config* cfg);

/* Repack expert weights once into the layout the grouped GEMMs read (K-major
 * tiles; for SwiGLU, gate and up columns interleaved in groups of 64 so every
 * 128-wide half of a 256-wide output tile holds matching gate/up columns).  Not
 * part of the forward.
 *   w_gate_up  device bf16 [E, D, 2F] (SwiGLU: columns [0,F) gate, [F,2F) up)
 *              or [E, D, F] (GELU: W1)  -- "Expert Parallel (EP)", Requirements:
 *              tensor-style gate_up_proj / down_proj experts
 *   w_down     device bf16 [E, F, D]
 *   ws_gate_up device bf16 [S, D, 2Fs] or NULL when S == 0
 *   ws_down    device bf16 [S, Fs, D]  or NULL when S == 0
 *   packed     device, moe_packed_weights_size(cfg) bytes, 256-byte aligned;
 *              written.  Inputs are only read. */
MOE_API moe_status moe_prepare_weights(const moe_config* cfg, const void* w_gate_up, const void* w_down,
                               const void* ws_gate_up, const void* ws_down, void* packed,
                               void* stream);

/* Stage 0, router + top-k.  "Worked Example: Tracing a Token Through Expert
 * Parallelism", Step 1; "Expert Parallel (EP)", Configuration (router_dtype
 * 'fp32', keep_router_logits).
 *   logits[t,e] = fp32( sum_d x[t,d]*w_router[e,d] ) (+ expert_bias[e] in fp32)
 *   topk_idx[t,:] = the k largest logits, descending, ties to the lower index
 *   topk_w[t,j] = exp(l_j - l_max) / sum over the top-k (renormalize) or over all E
 *   x           device [T, D], x_dtype
 *   w_router    device fp32 [E, D]
 *   expert_bias device fp32 [E] or NULL
 *   logits_out  device fp32 [T, E] or NULL (keep_router_logits)
 *   topk_idx    device int32 [T, k], written
 *   topk_w      device fp32 [T, k], written
 *   workspace   device, moe_workspace_size(cfg) bytes */
MOE_API moe_status moe_route(const moe_config* cfg, const void* x, const float* w_router,
                     const float* expert_bias, float* logits_out, int32_t* topk_idx,
                     float* topk_w, void* workspace, void* stream);

/* Stage 1, preprocess.  "Expert Parallel (EP)", Communication Pattern, step 1
 * (per-expert token counts and split sizes) and the order of step 2; "Worked
 * Example ...", Steps 2-3 (expert e on rank e / El, local index e mod El).
 *   counts[e]         device int32 [E]: pairs (t, j) with topk_idx[t,j] == e
 *   expert_offsets    device int32 [E+1]: exclusive prefix sum of counts
 *   rank_splits[r]    device int32 [ep]: sum of counts over experts r*El..r*El+El-1
 *   rank_offsets      device int32 [ep+1]: exclusive prefix sum of rank_splits
 *   pos[t*k+j]        device int32 [R]: permuted row of pair (t, j)
 *   src[row]          device int32 [R]: flat pair index t*k+j held by `row`
 * Rows are ordered rank-major, then local expert, then token ascending (the
 * same as global expert order).  Bit-exact and deterministic.  An index outside
 * [0, E) sets *status = MOE_ERR_INDEX_OOB and that pair is skipped.
 * Also writes the GEMM tile prefix into `workspace` for moe_expert_ffn. */
MOE_API moe_status moe_preprocess(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                          int32_t* expert_offsets, int32_t* rank_splits, int32_t* rank_offsets,
                          int32_t* pos, int32_t* src, void* workspace, int32_t* status,
                          void* stream);

/* Stage 2a, dispatch (token pre-all-to-all).  "Expert Parallel (EP)",
 * Communication Pattern, step 2; "Worked Example ...", Step 2 (each chosen expert
 * receives its own copy of the token).
 *   x_perm[pos[t*k+j], :] = bf16( x[t, :] )  for every token t and slot j
 *   (equivalently x_perm[row] = bf16(x[src[row] / k]); fp32 x rounds to nearest even)
 *   x      device [T, D] x_dtype;  pos device int32 [R] from moe_preprocess;
 *   x_perm device bf16 [R, D], written.  Rows whose pos is outside [0, R) are skipped. */
MOE_API moe_status moe_dispatch_permute(const moe_config* cfg, const void* x, const int32_t* pos,
                                void* x_perm, void* stream);

/* Stage 2b, local experts.  "Expert Parallel (EP)", Communication Pattern, step 3;
 * "Worked Example ...", Step 3 (two-layer FFN per expert).  Grouped GEMMs on the
 * tensor cores over each expert's row range [expert_offsets[e], expert_offsets[e+1]):
 *   SwiGLU: act = silu(x_perm W_gate) * (x_perm W_up);  y_perm = act W_down
 *   GELU:   act = gelu(x_perm W1);                       y_perm = act W2
 * Shared experts ("Expert Parallel (EP)", Requirements; torchtitan issue 5554):
 *   shared_out[t] = sum_i SwiGLU_i(x[t]), unit weight.
 *   x_perm         device bf16 [R, D]
 *   x              device bf16 [T, D] (read only when S > 0)
 *   expert_offsets device int32 [E+1] from moe_preprocess
 *   packed         device, from moe_prepare_weights
 *   act            device bf16 [R, F], written (intermediate)
 *   y_perm         device bf16 [R, D], written
 *   shared_out     device bf16 [T, D], written when S > 0; NULL skips the shared
 *                  experts (moe_shared_ffn runs them alone)
 *   workspace      the buffer moe_preprocess (or moe_route_dispatch) wrote its tile
 *                  prefix into, for this same routing: moe_preprocess_noalloc writes no
 *                  prefix, so its outputs need a moe_preprocess of the same topk_idx
 *                  before this call, or the tiles follow an earlier routing
 *   status         device int32, MOE_ERR_TIMEOUT if a bounded wait expired */
MOE_API moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const void* x,
                          const int32_t* expert_offsets, const void* packed, void* act,
                          void* y_perm, void* shared_out, void* workspace, int32_t* status,
                          void* stream);

/* The shared experts alone (S > 0): shared_out[t] = sum_i SwiGLU_i(x[t]) for the T
 * tokens of cfg, from the shared part of `packed` (moe_prepare_weights of any config
 * with the same E, D, F, act, S and Fs).  Used by the multi-rank forward, where a
 * rank runs the routed experts on rows received from other ranks but the shared
 * experts on its own tokens.  Arguments as moe_expert_ffn. */
MOE_API moe_status moe_shared_ffn(const moe_config* cfg, const void* x, const void* packed,
                                  void* shared_out, void* workspace, int32_t* status, void* stream);

/* Stage 3, combine (token post-all-to-all, unpermute, routing weights, residual).
 * "Expert Parallel (EP)", Communication Pattern, step 4; "Worked Example ...",
 * Step 4 (weighted sum) and Step 5 (residual):
 *   out[t] = x[t] + shared_out[t] + sum_j topk_w[t,j] * y_perm[pos[t*k+j]]
 * accumulated in fp32, stored once in x_dtype.
 *   y_perm device bf16 [R, D]; pos device int32 [R]; topk_w device fp32 [T, k]
 *   x device [T, D] x_dtype; shared_out device bf16 [T, D] or NULL
 *   out device [T, D] x_dtype, written (must not alias x) */
MOE_API moe_status moe_combine_unpermute(const moe_config* cfg, const void* y_perm, const int32_t* pos,
                                 const float* topk_w, const void* x, const void* shared_out,
                                 void* out, void* stream);

/* Router, preprocess and dispatch together ("Expert Parallel (EP)", Communication
 * Pattern steps 1-2; "Worked Example: Tracing a Token Through Expert Parallelism",
 * Steps 1-2): the outputs of moe_route, moe_preprocess and moe_dispatch_permute,
 * bit for bit, with the same arguments as those calls.  With at most 32 experts and
 * W_r plus one SM's share of the x rows fitting in 200 KB of shared memory this is
 * ONE cooperative launch that reads x once (each block routes its tokens, publishes
 * its expert histogram, passes one grid barrier, writes its pairs' rows and copies
 * its x rows into x_perm); otherwise (or with MOE_ROUTE_FUSED=0 in the environment)
 * it enqueues the three calls, as it also does when the cooperative launch is refused
 * for want of SMs.  Errors: those of the three calls; a grid barrier that does not
 * complete within about a second sets MOE_ERR_TIMEOUT in *status. */
MOE_API moe_status moe_route_dispatch(const moe_config* cfg, const void* x, const float* w_router,
                              const float* expert_bias, float* logits_out, int32_t* topk_idx,
                              float* topk_w, int32_t* counts, int32_t* expert_offsets,
                              int32_t* rank_splits, int32_t* rank_offsets, int32_t* pos,
                              int32_t* src, void* x_perm, void* workspace, int32_t* status,
                              void* stream);

/* 1 if moe_route_dispatch runs as one launch for this configuration (on the current
 * device, with the current environment), else 0 (also for an invalid configuration). */
MOE_API int32_t moe_route_dispatch_is_fused(const moe_config* cfg);

/* The whole layer: moe_route_dispatch (moe_route, moe_preprocess and
 * moe_dispatch_permute), moe_expert_ffn and moe_combine_unpermute enqueued in that
 * order on `stream`, with the same arguments as above.  logits_out and expert_bias
 * may be NULL. */
MOE_API moe_status moe_forward(const moe_config* cfg, const void* x, const float* w_router,
                       const float* expert_bias, const void* packed, float* logits_out,
                       int32_t* topk_idx, float* topk_w, int32_t* counts,
                       int32_t* expert_offsets, int32_t* rank_splits, int32_t* rank_offsets,
                       int32_t* pos, int32_t* src, void* x_perm, void* act, void* y_perm,
                       void* shared_out, void* out, void* workspace, int32_t* status,
                       void* stream);

/* Preprocess without a workspace -- for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for deployment.
 * moe_preprocess needs a caller-allocated `workspace` for its per-block expert
 * histograms.  Some callers have no way to provide one: a plugin inside a host
 * framework that owns every device allocation and only lends out the tensors it
 * already has, or a latency-critical loop in which cudaMalloc (which may
 * synchronise the whole device) is not acceptable.  This call takes no workspace
 * and allocates nothing: its scratch is one file-scope device array of
 * MOE_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds until
 * the process exits.
 *
 * Outputs, layouts, ordering and the device status word are exactly those of
 * moe_preprocess (bit-identical results); it does not write the GEMM tile prefix
 * that moe_expert_ffn reads from a workspace, so it is a drop-in for the
 * bookkeeping outputs only.
 *   Limit: max(1, min(160, ceil(T*k / 256))) * E + 2*(E + 1) + 2 int32 values must
 *   fit in the scratch (the check uses this count; the launch may then use fewer
 *   blocks on a GPU with fewer SMs); larger configurations return
 *   MOE_ERR_SCRATCH_LIMIT before anything is enqueued.
 *   First call on each device: finds the scratch array's device address with
 *   cudaGetSymbolAddress (once per device, with that device current), so make that
 *   first call before any stream capture.  The address is looked up again when the
 *   device's context is not the one it was found in (after cudaDeviceReset, the
 *   library's device array is loaded anew); that lookup, too, must not fall inside a
 *   stream capture.
 *   Concurrency: every call shares the one array and leaves its contents behind
 *   (each call rewrites all it reads); calls that may overlap on the GPU, e.g. on
 *   two streams without ordering between them, race and must not be issued. */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 18)
MOE_API moe_status moe_preprocess_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                          int32_t* counts, int32_t* expert_offsets,
                                          int32_t* rank_splits, int32_t* rank_offsets,
                                          int32_t* pos, int32_t* src, int32_t* status,
                                          void* stream);

/* Multi-rank expert parallelism ("Expert Parallel (EP)", Communication Pattern
 * steps 2-4): with ep_size = number of ranks, rank r owns experts
 * [r*El, (r+1)*El).  Each rank routes, preprocesses and dispatches its own tokens;
 * x_perm is then rank-major, and rows [rank_offsets[r], rank_offsets[r+1]) go to
 * rank r in the token pre-all-to-all (performed by the caller's communication
 * library).  These two calls do the row bookkeeping around the exchanges.
 *
 * ids[row] = local expert, on its destination rank, of dispatch row `row`:
 *   topk_idx[src[row]] % El  (-1 where src is outside [0, T*k)).
 *   topk_idx, src device int32 [T*k] (from moe_route / moe_preprocess of cfg);
 *   ids device int32 [T*k], written.  Sent along with the rows so the receiver can
 *   group its rows by local expert (moe_preprocess with k = 1 over them). */
MOE_API moe_status moe_ep_local_ids(const moe_config* cfg, const int32_t* topk_idx, const int32_t* src,
                                    int32_t* ids, void* stream);

/* dst[i, :] = src[index[i], :] for i in [0, n): bf16 rows of D elements (D % 8 == 0).
 * Rows whose index is outside [0, n_src) are left unwritten.  Used on the
 * receiving rank to put the local experts' output rows back in received order
 * (index = the pos of its k = 1 preprocess) for the token post-all-to-all.
 *   src device bf16 [n_src, D]; index device int32 [n]; dst device bf16 [n, D]. */
MOE_API moe_status moe_gather_rows(const void* src, const int32_t* index, void* dst, int32_t n,
                                   int32_t n_src, int32_t D, void* stream);

/* Self-check of device-side failure detection.  The cooperative kernels (moe_preprocess,
 * moe_route_dispatch) synchronise their blocks at a grid barrier whose wait is bounded
 * (~1 s of SM cycles); a block that gives up writes MOE_ERR_TIMEOUT to the status word
 * and the kernel returns, so the CUDA context stays usable and the caller reads the
 * status when convenient (the error convention of every call above).  This call runs
 * that barrier with one block where two are expected, so nothing completes it and the
 * wait runs out: after the stream reaches it, *status holds MOE_ERR_TIMEOUT (if it was
 * MOE_OK before).  Takes ~1 s of device time.
 *   barrier: two device uint32 words of scratch (zeroed by the call);
 *   status: device int32, not reset by the call. */
MOE_API moe_status moe_check_wait_timeout(uint32_t* barrier, int32_t* status, void* stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* MOE_ABI_VERSION of the loaded library. */
MOE_API int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
