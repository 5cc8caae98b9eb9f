// Internal declarations shared by the libmoe.so translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// Sizes fixed by the kernels
// ---------------------------------------------------------------------------
constexpr int kMaxExperts = 1024;   // preprocess keeps one counter per expert in smem
constexpr int kMaxTopK = 32;        // top-k kernel keeps selection j in lane j
constexpr int kPreThreads = 256;    // preprocess block size
constexpr int kPreMaxBlocks = 160;  // preprocess grid cap (>= one block per SM on B200)
constexpr int kTileM = 128;         // GEMM tile rows (one tcgen05 M=128 accumulator)
constexpr int kTileK = 64;          // GEMM K step: 64 bf16 = one 128-byte swizzle row

// ---------------------------------------------------------------------------
// Workspace and packed-weight layouts (byte offsets, each 256-aligned)
// ---------------------------------------------------------------------------
struct WsLayout {
  size_t logits;        // fp32 [T, E]
  size_t block_counts;  // int32 [nblk, E]: preprocess per-block histograms
  size_t barrier;       // uint32 [2]: preprocess grid barrier (zeroed per call)
  size_t act_shared;    // bf16 [T, S*Fs]
  size_t r_split;       // bf16 [2*Epad, D]: tensor-core router weights
  size_t r_wmax;        // fp32 [D]
  size_t r_approx;      // fp32 [T, Epad]
  size_t counters;      // int32 [8]: GEMM tile counters (router, routed up/down, shared up/down,
                        // the fused FFN launch), followed directly by the fused FFN launch's
                        // band counts int32 [done_slots]
  size_t done_slots;
  size_t total;
  int nblk;
};
WsLayout ws_layout(const moe_config& c);

struct PackLayout {
  size_t w_up;          // bf16 [E, Nup, D]   (Nup = 2F SwiGLU interleaved, or F)
  size_t w_down;        // bf16 [E, D, F]
  size_t ws_up;         // bf16 [1, 2*S*Fs, D] interleaved
  size_t ws_down;       // bf16 [1, D, S*Fs]
  size_t total;
};
PackLayout pack_layout(const moe_config& c);

// MXFP8 routed-expert weights: E4M3 gate_up [E, Nup, D] and down [E, D, F] (the bf16
// packing's row order), their scales in block order, and a row-major scale scratch.
struct MxPackLayout {
  size_t w_up, w_down, sf_up, sf_down, sf_scratch, total;
};
MxPackLayout mx_pack_layout(const moe_config& c);
// Workspace of the MXFP8 FFN: the bf16 workspace, then the quantised x_perm and
// activation with their scale blocks, and two tile counters.
struct MxWsLayout {
  size_t xq, xsf, aq, asf, counters, total;
};
MxWsLayout mx_ws_layout(const moe_config& c);

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// GEMM tile widths chosen from the shapes
int up_tile_n(const moe_config& c);
int down_tile_n(const moe_config& c);

// ---------------------------------------------------------------------------
// Launchers (each returns cudaGetLastError() of its launches)
// ---------------------------------------------------------------------------
// Workspace buffers of the tensor-core router (bf16 x).
struct RouterScratch {
  bf16* bsplit;     // [2 * Epad, D]: W_r hi / mid rows in 64-expert groups
  float* wmax;      // [D]: max_e |W_r[e, d]|
  float* approx;    // [T, Epad]: tensor-core logits (hi + mid)
  int pair;         // GEMM on CTA pairs
  int32_t* status;
  int32_t* counter; // GEMM tile counter (zeroed by the router before its launch)
  double* part;     // fp64 slice totals of a split logits launch (aliases bsplit), or null
  size_t part_bytes;
};
// Whether moe_route (bf16 x) takes the tensor-core filter + exact refine for this
// configuration, and the filter's per-unit error coefficient (eps_t = coef * S_t).
bool route_takes_filter(const moe_config& c, size_t part_bytes, bool keep_logits);
float route_filter_coef(int D);
// logits: where the tiled path stores fp32 logits (caller's buffer or workspace);
// keep_logits: the caller asked for them (the fused few-expert path then writes them).
cudaError_t launch_route(const moe_config& c, const void* x, const float* w_router,
                         const float* bias, float* logits, bool keep_logits, int32_t* topk_idx,
                         float* topk_w, const RouterScratch& rs, cudaStream_t s);
// Preprocess grid size for R pairs (<= kPreMaxBlocks); block_counts needs
// preprocess_blocks(R) * E entries.
int preprocess_blocks(int64_t R);
cudaError_t launch_preprocess(const moe_config& c, const int32_t* topk_idx, int32_t* counts,
                              int32_t* expert_offsets, int32_t* rank_splits,
                              int32_t* rank_offsets, int32_t* pos, int32_t* src,
                              int32_t* block_counts, int max_blocks,
                              unsigned* barrier, int32_t* status, cudaStream_t s);
// Self-check of the bounded grid-barrier wait (preprocess.cu): one block, barrier for two.
cudaError_t launch_barrier_timeout_check(unsigned* barrier, int32_t* status, cudaStream_t s);
// Multi-rank helpers (ep.cu).
cudaError_t launch_local_ids(const int32_t* topk_idx, const int32_t* src, int32_t* ids, int R, int El,
                             cudaStream_t s);
// MXFP8 quantisation of bf16 rows (mxfp8.cu).
cudaError_t launch_mx_quant_rows(const bf16* x, int64_t rows, int K, uint8_t* q, uint8_t* scales,
                                 cudaStream_t s);
// MXFP8 grouped GEMM (grouped_gemm_mx.cu): E4M3 A [a_rows, K] with row-major scales
// sa [a_rows, K/32]; E4M3 B [G, N, K] with scales in the tensor cores' block order sb
// (launch_mx_block_scales); 128 x 128 tiles; `counter` zero at launch.
struct MxProblem {
  const uint8_t* A; int64_t a_rows;       // E4M3 [a_rows, K]
  const uint8_t* sa;                      // A's scale blocks (launch_mx_quant_a or an EPI_SWIGLU/GELU run)
  const uint8_t* B; int G;                // E4M3 [G, N, K]
  const uint8_t* sb;                      // B's scale blocks (launch_mx_block_scales)
  int N, K;                               // N % 256 == 0, K % 128 == 0
  const int32_t* group_offsets;
  bf16* out; int ldo;                     // EPI_STORE: bf16 [a_rows, ldo]
  uint8_t* q_out; uint8_t* q_sf;          // EPI_SWIGLU / EPI_GELU: E4M3 [a_rows, ldo] + scale blocks
  int epi;
  int half_tiles;                         // a group's last <= 128 rows as an M = 128 tile
  int fold;                               // > 0: a group of 257..256 + fold rows as one folded tile
  int32_t* status;
  int32_t* counter;
};
cudaError_t launch_grouped_mx(const MxProblem& p, cudaStream_t s);
// Bytes of the scale blocks of `tiles` 256-row tiles over K: a B operand (two 128-row
// blocks per tile and K step) and an A operand (a third block for a folded remainder).
size_t mx_sf_bytes(int64_t tiles, int K);
size_t mx_sfa_bytes(int64_t tiles, int K);
// Row-major scales [rows, K/32] -> the scale blocks of a B operand (rows % 256 == 0,
// K % 128 == 0).
cudaError_t launch_mx_block_scales(const uint8_t* rowmajor, uint8_t* blocked, int64_t rows, int K,
                                   cudaStream_t s);
// bf16 rows grouped by group_offsets -> E4M3 rows and the scale blocks of an A operand.
// half_tiles, fold: the tiling of the GEMM that reads the blocks (MxProblem).  Row r
// comes from x[r], or with src from x[src[r] / k] (dispatch and quantisation in one pass).
cudaError_t launch_mx_quant_a(const bf16* x, const int32_t* src, int k, int64_t rows,
                              const int32_t* group_offsets, int G, int K, int half_tiles, int fold, uint8_t* q,
                              uint8_t* sf, cudaStream_t s);
// Peer-memory exchange (ep_peer.cu).
cudaError_t launch_ep_send_counts(const moe_ep_peers& p, int rank0, int nlocal, const int32_t* counts,
                                  int E, uint32_t epoch, cudaStream_t s);
cudaError_t launch_ep_send_rows(const moe_config& c, const moe_ep_peers& p, int rank0, int nlocal,
                                const void* x, const int32_t* topk_idx, const int32_t* pos,
                                const int32_t* expert_offsets, int32_t* done, int32_t* status,
                                uint32_t epoch, cudaStream_t s);
cudaError_t launch_ep_recv_layout(const moe_config& c, const moe_ep_peers& p, int rank0, int nlocal,
                                  int32_t* local_offsets, int32_t* status, uint32_t epoch,
                                  cudaStream_t s);
cudaError_t launch_ep_return_rows(const moe_config& c, const moe_ep_peers& p, int rank0, int nlocal,
                                  const void* y_recv, const int32_t* local_offsets, int32_t* done,
                                  uint32_t epoch, cudaStream_t s);
// Rank r's return flag on every rank (after a system-scope fence): its output rows
// were stored into the senders' y_back by the expert FFN itself.
cudaError_t launch_ep_signal_returned(const moe_ep_peers& p, int r, uint32_t epoch, cudaStream_t s);
cudaError_t launch_ep_wait_returned(const moe_ep_peers& p, int rank0, int nlocal, int32_t* status,
                                    uint32_t epoch, cudaStream_t s);
cudaError_t launch_gather_rows(const bf16* src, const int32_t* index, bf16* dst, int n, int n_src,
                               int D, cudaStream_t s);
// Router + preprocess + dispatch in one cooperative launch (few experts; see
// route_dispatch.cu).  route_pre_dispatch_applies: whether the configuration fits it.
bool route_pre_dispatch_applies(const moe_config& c, int max_blocks);
cudaError_t launch_route_pre_dispatch(const moe_config& c, const void* x, const float* w,
                                      const float* bias, float* logits_out, int32_t* topk_idx,
                                      float* topk_w, int32_t* counts, int32_t* expert_offsets,
                                      int32_t* rank_splits, int32_t* rank_offsets, int32_t* pos,
                                      int32_t* src, int32_t* block_counts, int max_blocks,
                                      unsigned* barrier, bool barrier_zeroed,
                                      bf16* x_perm, int32_t* status, cudaStream_t s);
cudaError_t launch_dispatch(const moe_config& c, const void* x, const int32_t* pos,
                            bf16* x_perm, cudaStream_t s);
cudaError_t launch_combine(const moe_config& c, const bf16* y_perm, const int32_t* pos,
                           const float* topk_w, const void* x, const bf16* shared_out, void* out,
                           cudaStream_t s);
cudaError_t launch_pack(const moe_config& c, const bf16* w_up, const bf16* w_down,
                        const bf16* ws_up, const bf16* ws_down, uint8_t* packed, cudaStream_t s);

// Grouped GEMM on the tensor cores.  out[row, :] = epilogue(A[row, :] @ B[g]^T)
// for rows of group g; B is K-major [G, N, K].
// EPI_PAIRSUM_F32: out_f32[row, n*BN/2 + c] = acc[c] + acc[BN/2 + c] (256-wide tiles)
enum Epilogue { EPI_STORE = 0, EPI_GELU = 1, EPI_SWIGLU = 2, EPI_PAIRSUM_F32 = 3 };
struct GemmProblem {
  const bf16* A; int64_t a_rows;          // A [a_rows, K]
  const bf16* B; int G;                   // B [G, N, K]
  int N, K;
  const int32_t* group_offsets;           // [G+1] device, or nullptr: one dense group
  int dense_rows;                         // rows of the dense group
  int64_t max_tiles;                      // host upper bound on tiles (grid size)
  bf16* out; int ldo;                     // output row stride in elements
  float* outf;                            // fp32 output (EPI_PAIRSUM_F32)
  int epi; int tile_n;
  int pair;                               // 1: 256-row tiles on CTA pairs
  int32_t* status;
  int32_t* counter;                       // device tile counter, zero when the launch starts
  int dep;                                // launch_grouped_pair: index of the phase whose output
                                          // rows this phase reads as A, or -1
  // launch_grouped_pair, EPI_STORE: output row i goes to sc_base[sc_rank[i]] at row
  // sc_row[i] (another rank's buffer, through a table of sc_P device pointers, each
  // buffer of sc_rows rows) instead of out; null: out.  No skinny or folded tiles then.
  bf16* const* sc_base;
  const int32_t* sc_rank;
  const int32_t* sc_row;
  int sc_P, sc_rows;
};
// Up to 4 GEMMs (all 256-wide tiles) in one persistent CTA-pair launch, tiles taken
// phase after phase; probs[i].dep = j (j < i) makes phase i read phase j's output
// rows only after each 256-row band of them is stored.  `counter` (one int) and
// `done` (pair_done_slots ints) must be zero when the launch starts.
cudaError_t launch_grouped_pair(const GemmProblem* probs, int n, int32_t* counter, int32_t* done,
                                cudaStream_t s);
int64_t pair_done_slots(const GemmProblem* probs, int n);
cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t s);

int sm_count();
// Cycle counters of an instrumented build (-DMOE_INSTRUMENT): copied to host and zeroed;
// cudaErrorNotSupported in an ordinary build.
cudaError_t instr_read_pair(unsigned long long* host, int n);
cudaError_t instr_read_mx(unsigned long long* host, int n);

}  // namespace moe
