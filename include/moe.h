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

/* 2: the MXFP8 routed-expert calls, moe_dispatch_mxfp8, the router filter view and the
 * peer-memory exchange calls.  3: the moe_ipc_* calls that map another process's
 * exchange buffers, moe_ep_expert_ffn_return and moe_instr_read. */
#define MOE_ABI_VERSION 3

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
 * preprocess block histograms, the tensor-core router's intermediates, the shared
 * experts' activations and the expert-FFN launch's tile and band counters.  0 for an
 * invalid config. */
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
 * `workspace` holds the per-block histograms (scratch). */
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
 *   workspace      moe_workspace_size(cfg) bytes of scratch; the tile schedule comes
 *                  from expert_offsets alone (each CTA derives the per-expert M tiles)
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
 * moe_preprocess (bit-identical results), and they are all moe_dispatch_permute,
 * moe_expert_ffn and moe_combine_unpermute read.
 *   Limit: max(1, min(160, ceil(T*k / 256))) * E + 2 int32 values must fit in the
 *   scratch (the check uses this count; the launch may then use fewer
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

/* Expert-parallel exchange over peer memory ("Expert Parallel (EP)", Communication
 * Pattern steps 2-4; "Worked Example ...", Steps 2 and 4): the token pre- and
 * post-all-to-all as stores into the other ranks' buffers, with no host round trip.
 * P = cfg->ep_size ranks; rank r owns experts [r*El, (r+1)*El), El = E / P, and holds
 * cfg->T tokens.  Every rank's exchange buffers are reachable from every rank through
 * the tables below: device arrays of P device pointers, entry p = rank p's buffer
 * (peer mappings of other GPUs' memory on a multi-GPU node; with several ranks on one
 * GPU, buffers of that GPU).  Each call covers ranks [rank0, rank0 + nlocal), the
 * ranks whose own data is on the calling device; their per-rank inputs are stacked
 * (rank rank0 + i at slice i of each argument; an int32 argument of n values per rank
 * has rows of (n + 3) / 4 * 4 values, so each rank's row is 16-byte aligned).  `epoch` numbers the exchange: every
 * call of one forward passes the same value, the next forward a different one (flags
 * are compared for equality, never reset).  Waits are bounded (~1 s of SM cycles) and
 * report MOE_ERR_TIMEOUT in *status; after an error the caller zeroes `done` and the
 * flag arrays before the next exchange.  Received rows of local expert l are ordered
 * by sending rank, then token, which the grouped FFN takes as is.
 * Order of one forward, on every rank: moe_route + moe_preprocess of its tokens,
 * moe_ep_send_counts, moe_ep_send_rows, moe_ep_recv_layout, moe_expert_ffn on the
 * received rows (a config with E = El, top_k = 1, T = cap, shared_out = NULL),
 * moe_ep_return_rows (or the last two as one: moe_ep_expert_ffn_return),
 * moe_ep_wait_returned, then moe_shared_ffn and moe_combine_unpermute with y_back in
 * place of y_perm (same rows, same order). */
typedef struct {
  int32_t P;                   /* ranks in the exchange (== cfg->ep_size) */
  int32_t cap;                 /* rows each rank's receive buffers hold */
  int32_t* const* cnt;         /* int32 [P, E]: row s = counts sent by rank s */
  uint32_t* const* flags;      /* uint32 [3, P], zero before the first exchange: epochs
                                  of counts / rows / returned rows from each rank */
  void* const* recv_x;         /* bf16 [cap, D]: rows received for the local experts */
  int32_t* const* recv_src;    /* int32 [cap]: the sender's dispatch row of each */
  int32_t* const* recv_rank;   /* int32 [cap]: the sender's rank of each */
  void* const* y_back;         /* bf16 [T*k, D]: output rows returned to this rank, at
                                  its own dispatch rows (pos) */
} moe_ep_peers;

/* Each covered rank's counts [E] (from moe_preprocess) into row `rank` of every rank's
 * count matrix, then its count flag there.  counts: device int32 [nlocal, E]. */
MOE_API moe_status moe_ep_send_counts(const moe_config* cfg, const moe_ep_peers* peers,
                                      int32_t rank0, int32_t nlocal, const int32_t* counts,
                                      uint32_t epoch, void* stream);

/* The token pre-all-to-all: waits for every rank's counts, then stores each covered
 * rank's k rows per token (bf16; an fp32 x is rounded to nearest even, as the dispatch
 * does) into the owning ranks' recv_x, with recv_src / recv_rank beside them, and
 * raises its row flag on every rank.  x [nlocal, T, D] (x_dtype), topk_idx and pos
 * [nlocal, T*k], expert_offsets [nlocal, E+1] (moe_route / moe_preprocess outputs);
 * done: device int32 [nlocal], zero (left zero).  A row beyond cap sets
 * MOE_ERR_INVALID_ARG in *status and is dropped. */
MOE_API moe_status moe_ep_send_rows(const moe_config* cfg, const moe_ep_peers* peers,
                                    int32_t rank0, int32_t nlocal, const void* x,
                                    const int32_t* topk_idx, const int32_t* pos,
                                    const int32_t* expert_offsets, uint32_t epoch, int32_t* done,
                                    int32_t* status, void* stream);

/* Waits until every rank's rows have arrived, then writes each covered rank's local
 * expert offsets [nlocal, El+1] over its received rows (the expert_offsets argument of
 * the local moe_expert_ffn). */
MOE_API moe_status moe_ep_recv_layout(const moe_config* cfg, const moe_ep_peers* peers,
                                      int32_t rank0, int32_t nlocal, int32_t* local_offsets,
                                      uint32_t epoch, int32_t* status, void* stream);

/* The token post-all-to-all: each covered rank's output rows y_recv [nlocal, cap, D]
 * (bf16, the local experts' y over the received rows, local_offsets as written by
 * moe_ep_recv_layout) go back to their senders' y_back at the senders' rows; then the
 * rank raises its return flag on every rank.  done: device int32 [nlocal], zero. */
MOE_API moe_status moe_ep_return_rows(const moe_config* cfg, const moe_ep_peers* peers,
                                      int32_t rank0, int32_t nlocal, const void* y_recv,
                                      const int32_t* local_offsets, uint32_t epoch,
                                      int32_t* done, int32_t* status, void* stream);

/* The local experts and the token post-all-to-all as one step, for rank `rank` (one
 * rank per call): moe_expert_ffn on the received rows (local_cfg: E = El, top_k = 1,
 * T = peers->cap, the tokens config's D, F, act and shared-expert sizes; the shared
 * experts are not run) whose down-projection epilogue stores each output row straight
 * into its sender's y_back at the sender's dispatch row (recv_rank / recv_src, this
 * rank's own buffers), over NVLink / NVSwitch peer memory as each tile finishes, so the
 * return overlaps the GEMM tile by tile and the rows never pass through a y_recv
 * buffer; then the rank's return flag on every rank.  Equivalent to moe_expert_ffn into
 * y_recv followed by moe_ep_return_rows, which is what runs where the down GEMM is not
 * a CTA-pair launch (D not a multiple of 256) or MOE_EP_FUSED_RETURN=0 is set: y_recv
 * (bf16 [cap, D]) is needed then and may be NULL otherwise.  recv_x: bf16 [cap, D];
 * recv_src, recv_rank: int32 [cap] (4-byte aligned); local_offsets: [El+1] from
 * moe_ep_recv_layout; act: bf16 [cap, F] scratch; workspace:
 * moe_workspace_size(local_cfg) bytes; done: one device int32 (4-byte aligned), zero. */
MOE_API moe_status moe_ep_expert_ffn_return(const moe_config* cfg, const moe_config* local_cfg,
                                            const moe_ep_peers* peers, int32_t rank, const void* recv_x,
                                            const int32_t* recv_src, const int32_t* recv_rank,
                                            const int32_t* local_offsets, const void* packed, void* act,
                                            void* y_recv, void* workspace, uint32_t epoch, int32_t* done,
                                            int32_t* status, void* stream);

/* Waits until every rank has returned the covered ranks' rows (y_back complete). */
MOE_API moe_status moe_ep_wait_returned(const moe_config* cfg, const moe_ep_peers* peers,
                                        int32_t rank0, int32_t nlocal, uint32_t epoch,
                                        int32_t* status, void* stream);

/* One process per GPU: the moe_ep_peers tables of a rank hold pointers into the other
 * ranks' processes, mapped once before the first exchange ("Expert Parallel (EP)",
 * Communication Pattern, steps 2 and 4: rows are stored straight into the owning
 * rank's buffers).  Each rank exports its exchange buffers, sends the handle bytes and
 * offsets to the others over its process group (host memory), and imports theirs.
 * Setup-time calls (synchronous, no stream); the buffers must come from cudaMalloc
 * (a caching allocator's blocks are fine; memory from cuMemCreate is not exportable
 * and gives MOE_ERR_CUDA).  A rank never imports its own handle: its own table entry
 * is its own pointer.
 *
 * Size in bytes of an exported handle (the bytes the caller sends to the other ranks). */
MOE_API int32_t moe_ipc_handle_bytes(void);
/* ptr: a device pointer inside a cudaMalloc allocation of the calling process.
 * handle: host buffer of moe_ipc_handle_bytes() bytes, written: the allocation's
 * handle.  offset: host, written: ptr's byte offset from the allocation's start.
 * MOE_ERR_INVALID_ARG for a null argument or a pointer the driver does not know. */
MOE_API moe_status moe_ipc_export(const void* ptr, void* handle, uint64_t* offset);
/* Maps another process's allocation (handle and offset from its moe_ipc_export, on
 * another device of this node) into this process, with peer access enabled on first
 * use; *ptr (host, written) = the mapped buffer's device address.  The mapping stays
 * until moe_ipc_close; the exporting process must keep the buffer alive until every
 * importer has closed it.  MOE_ERR_CUDA if the driver refuses the handle (for
 * instance a handle of this same process). */
MOE_API moe_status moe_ipc_import(const void* handle, uint64_t offset, void** ptr);
/* Unmaps a buffer mapped by moe_ipc_import (the same ptr and offset). */
MOE_API moe_status moe_ipc_close(void* ptr, uint64_t offset);

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

/* Where moe_route's tensor-core router leaves its intermediate values, so that a
 * caller (the parity tests) can measure how close the filter runs to its error bound.
 * "Expert Parallel (EP)", Configuration: the router is computed in fp32
 * (router_dtype='fp32'); for bf16 x with more experts than the shared-memory router
 * holds, moe_route without returned logits finds each token's top-k in two steps:
 * approx[t,e] = x_t . (hi_e + mid_e) on the tensor cores (W_r = hi + mid + lo, hi and
 * mid bf16), and an exact fp32 logit for every expert whose approx + bias is at least
 * the k-th largest minus 2 eps_t, eps_t = coef * sum_d |x_t,d| wmax_d.  That is sound
 * when |approx - exact| <= eps_t, which this view lets a test check.
 * After moe_route with this cfg and workspace (no logits returned), the workspace
 * holds, until the next call that uses it:
 *   approx [T, approx_ld] fp32 at byte *approx_offset (bias not added; columns >= E
 *          are padding), wmax [D] fp32 at byte *wmax_offset; *coef is the coefficient.
 * Returns MOE_ERR_UNSUPPORTED when moe_route takes another path for cfg (fp32 x, few
 * experts, few tokens, no renormalisation, or MOE_ROUTER_TC=0 in the environment).
 * Host-only: enqueues nothing. */
MOE_API moe_status moe_router_filter_view(const moe_config* cfg, size_t* approx_offset,
                                          int32_t* approx_ld, size_t* wmax_offset, float* coef);

/* MXFP8 quantisation of bf16 rows (OCP Microscaling v1.0 "MXFP8 (E4M3)"; the MXFP8
 * routed-expert option of torchtitan issue 5554): every 32 consecutive elements of a row
 * share one power-of-two scale 2^s, s = floor(log2 max|v|) - 8 clamped to [-127, 127]
 * (-127 for an all-zero block), and each element becomes v / 2^s rounded to the nearest
 * E4M3 value, ties to even, magnitudes above 448 clamped to 448.
 *   x      device bf16 [rows, K], K % 32 == 0, 16-byte aligned
 *   q      device uint8 [rows, K], written: E4M3 bit patterns
 *   scales device uint8 [rows, K/32], written: s + 127 (E8M0)
 * Errors: MOE_ERR_INVALID_ARG for a bad pointer, a negative size or K % 32 != 0. */
MOE_API moe_status moe_mxfp8_quantize(const void* x, int64_t rows, int32_t K, void* q, void* scales,
                                      void* stream);

/* MXFP8 routed experts (opt-in; the layer's default path is bf16).  torchtitan issue 5554
 * names MXFP8 routed experts as an option; the expert FFN is the same two-layer network
 * ("Expert Parallel (EP)", Communication Pattern step 3), with every operand of both
 * GEMMs quantised to MXFP8 as moe_mxfp8_quantize does along its K axis: x_perm and the
 * weights of gate_up along D, the activation and the down weights along F.  The tensor
 * cores form the scaled products exactly and accumulate in fp32 (tcgen05 kind::mxf8f6f4
 * with block scales); the activation (SiLU(gate) * up, or GELU) is formed in fp32 and
 * quantised from fp32, never rounded to bf16.  Needs D % 256 == 0, F % 128 == 0 and a
 * gate_up width (2F for SwiGLU, F for GELU) that is a multiple of 256, else
 * MOE_ERR_UNSUPPORTED.
 *
 * Bytes of the MXFP8 weight buffer: */
MOE_API size_t moe_packed_weights_mxfp8_size(const moe_config* cfg);
/* Bytes of workspace for moe_expert_ffn_mxfp8 (includes moe_workspace_size's). */
MOE_API size_t moe_workspace_mxfp8_size(const moe_config* cfg);
/* Quantises the routed experts of `packed` (moe_prepare_weights' output for cfg) into
 * packed_mx (caller-allocated, moe_packed_weights_mxfp8_size bytes); one time. */
MOE_API moe_status moe_prepare_weights_mxfp8(const moe_config* cfg, const void* packed, void* packed_mx,
                                             void* stream);
/* Dispatch straight into MXFP8 (bf16 x only): each routed row r, in the expert-grouped
 * order of moe_preprocess, is quantised from x[src[r] / k] ("Expert Parallel (EP)",
 * Communication Pattern step 2) into the MXFP8 workspace, E4M3 elements with their
 * scales ordered for the expert GEMM's tiles; moe_expert_ffn_mxfp8 with x_perm = NULL
 * then uses them.  Equal, bit for bit, to moe_dispatch_permute followed by the
 * quantisation inside moe_expert_ffn_mxfp8, without writing the bf16 x_perm.
 *   x              device bf16 [T, D];  src, expert_offsets from moe_preprocess
 *   workspace      the MXFP8 workspace later passed to moe_expert_ffn_mxfp8
 * Errors: MOE_ERR_UNSUPPORTED for fp32 x or a shape moe_expert_ffn_mxfp8 refuses;
 * MOE_ERR_INVALID_ARG for a bad pointer. */
MOE_API moe_status moe_dispatch_mxfp8(const moe_config* cfg, const void* x, const int32_t* src,
                                      const int32_t* expert_offsets, void* workspace, void* stream);
/* moe_expert_ffn with MXFP8 routed experts: quantises x_perm (E4M3 rows and their
 * scales, ordered for the GEMM's tiles; x_perm NULL: the rows moe_dispatch_mxfp8 left in
 * the workspace), runs gate_up with the activation and its
 * quantisation in the epilogue (the quantised activation stays in the workspace; no
 * bf16 act is written), then down into y_perm (bf16 [T*k, D]).  The shared experts (if
 * shared_out is not NULL) run in bf16 from `packed` as in moe_expert_ffn.  Other
 * arguments as moe_expert_ffn; workspace: moe_workspace_mxfp8_size bytes, nothing in it
 * needs clearing.  Errors as moe_expert_ffn. */
MOE_API moe_status moe_expert_ffn_mxfp8(const moe_config* cfg, const void* x_perm, const void* x,
                                        const int32_t* expert_offsets, const void* packed,
                                        const void* packed_mx, void* y_perm, void* shared_out,
                                        void* workspace, int32_t* status, void* stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* MOE_ABI_VERSION of the loaded library. */
MOE_API int32_t moe_abi_version(void);

/* Cycle counters of an instrumented build of the library (compiled with
 * -DMOE_INSTRUMENT: `python -m expert_dispatch_fp32_b200.instrument`).  kernel 0: the bf16
 * grouped-GEMM kernels, 1: the MXFP8 kernel.  counters: host uint64 [n], written with up
 * to 160 CTAs x 24 slots of summed SM cycles and counts (slot order: MMA issuer total, its
 * waits for the accumulator, its waits for a filled stage, then tiles and issuer cycles of
 * full, M = 128, folded and skinny tiles, K steps, the producer's waits for a free stage
 * and its total, the first epilogue warp's waits for a full accumulator and its total,
 * then the K steps of full, M = 128, folded and skinny tiles); the device counters are
 * zeroed.  Synchronous.  MOE_ERR_UNSUPPORTED in an ordinary build. */
MOE_API moe_status moe_instr_read(int32_t kernel, uint64_t* counters, int32_t n);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
