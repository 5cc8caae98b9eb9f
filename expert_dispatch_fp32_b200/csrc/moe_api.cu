// C ABI of libmoe.so: argument validation, buffer layouts and the stage calls.
// Each call checks its arguments on the host, then only enqueues kernels on the
// caller's stream.  Nothing here allocates device memory.
#include <stdlib.h>
#include <string.h>

#include "moe_internal.cuh"

namespace moe {

// Counter word of the fused FFN launch (words 0..4: the router GEMM and the separate GEMMs).
constexpr int kFfnCounter = 5;

WsLayout ws_layout(const moe_config& c) {
  WsLayout L;
  const size_t T = (size_t)c.T, E = (size_t)c.E;
  const size_t R = T * (size_t)c.top_k;
  // one histogram row per preprocess block (at most kPreMaxBlocks; the fused router +
  // preprocess + dispatch launch uses one block per SM)
  L.nblk = kPreMaxBlocks;
  (void)R;
  size_t o = 0;
  L.logits = o;       o = align256(o + T * E * sizeof(float));
  L.block_counts = o; o = align256(o + (size_t)L.nblk * E * sizeof(int32_t));
  L.barrier = o;      o = align256(o + 2 * sizeof(uint32_t));
  L.act_shared = o;   o = align256(o + T * (size_t)c.n_shared * c.F_shared * sizeof(bf16));
  const size_t Epad = (E + 127) / 128 * 128;
  L.r_split = o;      o = align256(o + 2 * Epad * (size_t)c.D * sizeof(bf16));
  L.r_wmax = o;       o = align256(o + (size_t)c.D * sizeof(float));
  L.r_approx = o;     o = align256(o + T * Epad * sizeof(float));
  // band counts of the fused FFN launch: routed gate_up bands (<= R/256 + E) and the
  // shared gate_up bands (ceil(T/256))
  const size_t done_slots = (size_t)(T * c.top_k) / 256 + E + (T + 255) / 256 + 2;
  L.counters = o;     o = align256(o + (8 + done_slots) * sizeof(int32_t));
  L.done_slots = done_slots;
  L.total = o;
  return L;
}

PackLayout pack_layout(const moe_config& c) {
  PackLayout L;
  const size_t E = c.E, D = c.D, F = c.F;
  const size_t nup = c.act == MOE_ACT_SWIGLU ? 2 * F : F;
  const size_t Fc = (size_t)c.n_shared * c.F_shared;
  size_t o = 0;
  L.w_up = o;    o = align256(o + E * nup * D * sizeof(bf16));
  L.w_down = o;  o = align256(o + E * D * F * sizeof(bf16));
  L.ws_up = o;   o = align256(o + 2 * Fc * D * sizeof(bf16));
  L.ws_down = o; o = align256(o + D * Fc * sizeof(bf16));
  L.total = o;
  return L;
}

MxPackLayout mx_pack_layout(const moe_config& c) {
  MxPackLayout L;
  const size_t E = c.E, D = c.D, F = c.F;
  const size_t nup = c.act == MOE_ACT_SWIGLU ? 2 * F : F;
  size_t o = 0;
  L.w_up = o;       o = align256(o + E * nup * D);
  L.w_down = o;     o = align256(o + E * D * F);
  L.sf_up = o;      o = align256(o + E * nup * (D / 32));
  L.sf_down = o;    o = align256(o + E * D * (F / 32));
  L.sf_scratch = o; o = align256(o + (E * nup * (D / 32) > E * D * (F / 32) ? E * nup * (D / 32) : E * D * (F / 32)));
  L.total = o;
  return L;
}

MxWsLayout mx_ws_layout(const moe_config& c) {
  MxWsLayout L;
  const size_t R = (size_t)c.T * c.top_k, D = c.D, F = c.F;
  const int64_t tiles = (int64_t)(R / 256) + c.E;     // bounds the 256-row tiles of all experts
  size_t o = ws_layout(c).total;
  L.xq = o;       o = align256(o + R * D);
  L.xsf = o;      o = align256(o + mx_sfa_bytes(tiles, c.D));
  L.aq = o;       o = align256(o + R * F);
  L.asf = o;      o = align256(o + mx_sfa_bytes(tiles, c.F));
  L.counters = o; o = align256(o + 2 * sizeof(int32_t));
  L.total = o;
  return L;
}

int up_tile_n(const moe_config& c) {
  if (c.act == MOE_ACT_SWIGLU) return 256;
  return c.F % 256 == 0 ? 256 : c.F % 128 == 0 ? 128 : 64;
}
int down_tile_n(const moe_config& c) { return c.D % 256 == 0 ? 256 : c.D % 128 == 0 ? 128 : 64; }

}  // namespace moe

using namespace moe;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_CHECK_PTR(p) \
  do {                                                 \
    if ((p) == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG; \
  } while (0)

// moe_route_dispatch; barrier_zeroed: grid-barrier words the caller zeroed on the stream
// already (moe_forward's one memset), else the workspace's words, zeroed here.
moe_status route_dispatch_run(const moe_config* cfg, const void* x, const float* w_router,
                              const float* expert_bias, float* logits_out, int32_t* topk_idx,
                              float* topk_w, int32_t* counts, int32_t* expert_offsets,
                              int32_t* rank_splits, int32_t* rank_offsets, int32_t* pos,
                              int32_t* src, void* x_perm, void* workspace, int32_t* status,
                              void* stream, unsigned* barrier_zeroed) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  const WsLayout L = ws_layout(c);
  // MOE_ROUTE_FUSED=0 runs the three stage calls (read at each call; for comparison)
  const bool fused = moe_route_dispatch_is_fused(cfg) != 0;
  if (!fused) {
    st = moe_route(cfg, x, w_router, expert_bias, logits_out, topk_idx, topk_w, workspace, stream);
    if (st != MOE_OK) return st;
    st = moe_preprocess(cfg, topk_idx, counts, expert_offsets, rank_splits, rank_offsets, pos, src,
                        workspace, status, stream);
    if (st != MOE_OK) return st;
    return moe_dispatch_permute(cfg, x, pos, x_perm, stream);
  }
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(w_router);
  MOE_CHECK_PTR(topk_idx);
  MOE_CHECK_PTR(topk_w);
  MOE_CHECK_PTR(counts);
  MOE_CHECK_PTR(expert_offsets);
  MOE_CHECK_PTR(rank_splits);
  MOE_CHECK_PTR(rank_offsets);
  MOE_CHECK_PTR(pos);
  MOE_CHECK_PTR(src);
  MOE_CHECK_PTR(x_perm);
  MOE_CHECK_PTR(workspace);
  MOE_CHECK_PTR(status);
  if (logits_out != nullptr && !aligned16(logits_out)) return MOE_ERR_INVALID_ARG;
  uint8_t* ws = (uint8_t*)workspace;
  const cudaError_t err = launch_route_pre_dispatch(
      c, x, w_router, expert_bias, logits_out, topk_idx, topk_w, counts, expert_offsets, rank_splits,
      rank_offsets, pos, src, (int32_t*)(ws + L.block_counts), L.nblk,
      barrier_zeroed != nullptr ? barrier_zeroed : (unsigned*)(ws + L.barrier), barrier_zeroed != nullptr,
      (bf16*)x_perm, status, as_stream(stream));
  if (err == cudaErrorCooperativeLaunchTooLarge) {
    // fewer SMs available than the one-block-per-SM grid needs (a partitioned GPU):
    // the stage calls compute the same outputs
    (void)cudaGetLastError();
    st = moe_route(cfg, x, w_router, expert_bias, logits_out, topk_idx, topk_w, workspace, stream);
    if (st != MOE_OK) return st;
    st = moe_preprocess(cfg, topk_idx, counts, expert_offsets, rank_splits, rank_offsets, pos, src,
                        workspace, status, stream);
    if (st != MOE_OK) return st;
    return moe_dispatch_permute(cfg, x, pos, x_perm, stream);
  }
  return cuda_status(err);
}

}  // namespace

extern "C" {

moe_status moe_validate_config(const moe_config* cfg) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  if (c.T < 0 || c.D <= 0 || c.E <= 0 || c.ep_size <= 0 || c.top_k <= 0 || c.F <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c.E % c.ep_size != 0) return MOE_ERR_INVALID_ARG;        // num_experts % ep_size
  if (c.top_k > c.E) return MOE_ERR_INVALID_ARG;
  if (c.act != MOE_ACT_GELU && c.act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (c.renormalize != 0 && c.renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (c.x_dtype != MOE_DT_F32 && c.x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
  if (c.router_dtype != MOE_DT_F32) return MOE_ERR_UNSUPPORTED;   // the fp32 router only
  if (c.n_shared < 0 || (c.n_shared > 0 && c.F_shared <= 0)) return MOE_ERR_INVALID_ARG;
  if (c.E > kMaxExperts || c.top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (c.D % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (c.act == MOE_ACT_SWIGLU ? (c.F % 128 != 0) : (c.F % 64 != 0)) return MOE_ERR_UNSUPPORTED;
  if (c.n_shared > 0 && (c.F_shared % 128 != 0 || c.x_dtype != MOE_DT_BF16)) return MOE_ERR_UNSUPPORTED;
  const int64_t R = (int64_t)c.T * c.top_k;
  if (R * (c.D / 8) >= (int64_t)1 << 31 || (int64_t)c.T * c.E >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

size_t moe_workspace_size(const moe_config* cfg) {
  if (moe_validate_config(cfg) != MOE_OK) return 0;
  return ws_layout(*cfg).total;
}

size_t moe_packed_weights_size(const moe_config* cfg) {
  if (moe_validate_config(cfg) != MOE_OK) return 0;
  return pack_layout(*cfg).total;
}

moe_status moe_prepare_weights(const moe_config* cfg, const void* w_gate_up, const void* w_down,
                               const void* ws_gate_up, const void* ws_down, void* packed,
                               void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  MOE_CHECK_PTR(w_gate_up);
  MOE_CHECK_PTR(w_down);
  MOE_CHECK_PTR(packed);
  if (c.n_shared > 0) {
    MOE_CHECK_PTR(ws_gate_up);
    MOE_CHECK_PTR(ws_down);
  }
  return cuda_status(launch_pack(c, (const bf16*)w_gate_up, (const bf16*)w_down,
                                 (const bf16*)ws_gate_up, (const bf16*)ws_down, (uint8_t*)packed,
                                 as_stream(stream)));
}

moe_status moe_route(const moe_config* cfg, const void* x, const float* w_router,
                     const float* expert_bias, float* logits_out, int32_t* topk_idx,
                     float* topk_w, void* workspace, void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.T == 0) return MOE_OK;
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(w_router);
  MOE_CHECK_PTR(topk_idx);
  MOE_CHECK_PTR(topk_w);
  MOE_CHECK_PTR(workspace);
  const WsLayout L = ws_layout(c);
  uint8_t* ws = (uint8_t*)workspace;
  float* logits = logits_out;
  if (logits == nullptr) logits = (float*)(ws + L.logits);
  else if (!aligned16(logits)) return MOE_ERR_INVALID_ARG;
  const char* pair_env = getenv("MOE_GEMM_CTA_PAIR");
  RouterScratch rs;
  rs.bsplit = (bf16*)(ws + L.r_split);
  rs.wmax = (float*)(ws + L.r_wmax);
  rs.approx = (float*)(ws + L.r_approx);
  rs.pair = !(pair_env && pair_env[0] == '0');
  rs.status = nullptr;
  rs.counter = (int32_t*)(ws + L.counters);
  // the split logits path and the tensor-core path never run in one call: the split
  // path's fp64 slice totals reuse the W_r split region
  rs.part = (double*)(ws + L.r_split);
  rs.part_bytes = L.r_wmax - L.r_split;
  return cuda_status(launch_route(c, x, w_router, expert_bias, logits, logits_out != nullptr,
                                  topk_idx, topk_w, rs, as_stream(stream)));
}

moe_status moe_preprocess(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                          int32_t* expert_offsets, int32_t* rank_splits, int32_t* rank_offsets,
                          int32_t* pos, int32_t* src, void* workspace, int32_t* status,
                          void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  MOE_CHECK_PTR(counts);
  MOE_CHECK_PTR(expert_offsets);
  MOE_CHECK_PTR(rank_splits);
  MOE_CHECK_PTR(rank_offsets);
  MOE_CHECK_PTR(workspace);
  MOE_CHECK_PTR(status);
  if (c.T > 0) {
    MOE_CHECK_PTR(topk_idx);
    MOE_CHECK_PTR(pos);
    MOE_CHECK_PTR(src);
  }
  const WsLayout L = ws_layout(c);
  uint8_t* ws = (uint8_t*)workspace;
  return cuda_status(launch_preprocess(c, topk_idx, counts, expert_offsets, rank_splits,
                                       rank_offsets, pos, src, (int32_t*)(ws + L.block_counts),
                                       L.nblk,
                                       (unsigned*)(ws + L.barrier), status, as_stream(stream)));
}

moe_status moe_dispatch_permute(const moe_config* cfg, const void* x, const int32_t* pos,
                                void* x_perm, void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.T == 0) return MOE_OK;
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(pos);
  MOE_CHECK_PTR(x_perm);
  return cuda_status(launch_dispatch(c, x, pos, (bf16*)x_perm, as_stream(stream)));
}

}  // extern "C"

namespace {

// The expert-FFN stage: the routed experts over x_perm (`routed`) and/or the shared
// experts over x (`shared`), one persistent launch when all tiles are 256 wide.
// Where the routed down projection's rows go when they are stored straight into other
// ranks' buffers (moe_ep_expert_ffn_return): row i to base[rank[i]] at row[i].
struct FfnScatter {
  bf16* const* base;
  const int32_t* rank;
  const int32_t* row;
  int P, rows;
};

moe_status ffn_run(const moe_config* cfg, const void* x_perm, const void* x,
                   const int32_t* expert_offsets, const void* packed, void* act, void* y_perm,
                   void* shared_out, void* workspace, int32_t* status, void* stream, bool routed,
                   bool shared, bool counters_zeroed = false, const FfnScatter* scatter = nullptr) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (shared && c.n_shared == 0) return MOE_ERR_INVALID_ARG;
  if (c.T == 0 || (!routed && !shared)) return MOE_OK;
  if (routed) {
    MOE_CHECK_PTR(x_perm);
    MOE_CHECK_PTR(expert_offsets);
    MOE_CHECK_PTR(act);
    if (scatter == nullptr) MOE_CHECK_PTR(y_perm);
  }
  if (scatter != nullptr && (!routed || shared)) return MOE_ERR_INVALID_ARG;
  MOE_CHECK_PTR(packed);
  MOE_CHECK_PTR(workspace);
  MOE_CHECK_PTR(status);
  if (shared) {
    MOE_CHECK_PTR(x);
    MOE_CHECK_PTR(shared_out);
  }
  cudaStream_t s = as_stream(stream);
  const WsLayout W = ws_layout(c);
  // 256-wide tiles run on CTA pairs (256 x 256 per pair) unless MOE_GEMM_CTA_PAIR=0
  // selects the one-CTA 128 x 256 kernel (kept for comparison and for narrow N).
  const char* pair_env = getenv("MOE_GEMM_CTA_PAIR");
  const bool use_pair = !(pair_env && pair_env[0] == '0');
  const PackLayout P = pack_layout(c);
  const uint8_t* pk = (const uint8_t*)packed;
  uint8_t* ws = (uint8_t*)workspace;
  const int64_t R = (int64_t)c.T * c.top_k;
  const int nup = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  int32_t* ctr = (int32_t*)(ws + W.counters);

  // Routed experts, gate_up (+ activation) then down, over the rank-major rows.
  GemmProblem up;
  memset(&up, 0, sizeof(up));
  up.A = (const bf16*)x_perm; up.a_rows = R;
  up.B = (const bf16*)(pk + P.w_up); up.G = c.E;
  up.N = nup; up.K = c.D;
  up.group_offsets = expert_offsets;
  up.tile_n = up_tile_n(c);
  up.pair = use_pair && up.tile_n == 256;
  up.max_tiles = (R / (up.pair ? 2 * kTileM : kTileM) + c.E) * (int64_t)(nup / up.tile_n);
  up.out = (bf16*)act; up.ldo = c.F;
  up.epi = c.act == MOE_ACT_SWIGLU ? EPI_SWIGLU : EPI_GELU;
  up.status = status;
  up.counter = ctr + 1;
  up.dep = -1;

  GemmProblem dn = up;
  dn.A = (const bf16*)act; dn.a_rows = R;
  dn.B = (const bf16*)(pk + P.w_down);
  dn.N = c.D; dn.K = c.F;
  dn.tile_n = down_tile_n(c);
  dn.pair = use_pair && dn.tile_n == 256;
  dn.max_tiles = (R / (dn.pair ? 2 * kTileM : kTileM) + c.E) * (int64_t)(c.D / dn.tile_n);
  dn.out = (bf16*)y_perm; dn.ldo = c.D;
  dn.epi = EPI_STORE;
  dn.counter = ctr + 2;
  if (scatter != nullptr) {
    dn.sc_base = scatter->base;
    dn.sc_rank = scatter->rank;
    dn.sc_row = scatter->row;
    dn.sc_P = scatter->P;
    dn.sc_rows = scatter->rows;
  }

  // Shared experts: one dense SwiGLU expert of intermediate S*Fs over all tokens.
  const int Fc = c.n_shared * c.F_shared;
  bf16* act_s = (bf16*)(ws + W.act_shared);
  GemmProblem su, sd;
  memset(&su, 0, sizeof(su));
  memset(&sd, 0, sizeof(sd));
  if (shared) {
    su.A = (const bf16*)x; su.a_rows = c.T;
    su.B = (const bf16*)(pk + P.ws_up); su.G = 1;
    su.N = 2 * Fc; su.K = c.D;
    su.group_offsets = nullptr; su.dense_rows = c.T;
    su.tile_n = 256;
    su.pair = use_pair;
    const int tm_s = su.pair ? 2 * kTileM : kTileM;
    su.max_tiles = ((int64_t)(c.T + tm_s - 1) / tm_s) * (2 * Fc / 256);
    su.out = act_s; su.ldo = Fc;
    su.epi = EPI_SWIGLU;
    su.status = status;
    su.counter = ctr + 3;
    su.dep = -1;

    sd = su;
    sd.A = act_s; sd.a_rows = c.T;
    sd.B = (const bf16*)(pk + P.ws_down);
    sd.N = c.D; sd.K = Fc;
    sd.tile_n = down_tile_n(c);
    sd.pair = use_pair && sd.tile_n == 256;
    const int tm_sd = sd.pair ? 2 * kTileM : kTileM;
    sd.max_tiles = ((int64_t)(c.T + tm_sd - 1) / tm_sd) * (c.D / sd.tile_n);
    sd.out = (bf16*)shared_out; sd.ldo = c.D;
    sd.epi = EPI_STORE;
    sd.counter = ctr + 4;
  }

  // MOE_GEMM_FUSED=0 selects one launch per GEMM (read at each call; for comparison)
  const char* fused_env = getenv("MOE_GEMM_FUSED");
  const bool fused = !(fused_env && fused_env[0] == '0');
  if (fused && (!routed || (up.pair && dn.pair)) && (!shared || (su.pair && sd.pair))) {
    // One persistent launch: routed gate_up, shared gate_up, routed down, shared down.
    // Each down tile waits only for the gate_up band it reads, so the down phase
    // starts while the last gate_up tiles finish (no launch gap, one tail).
    GemmProblem ph[4];
    int n = 0;
    if (routed) ph[n++] = up;
    if (shared) ph[n++] = su;
    if (routed) { ph[n] = dn; ph[n].dep = 0; ++n; }
    if (shared) { ph[n] = sd; ph[n].dep = routed ? 1 : 0; ++n; }
    // tile counter: word kFfnCounter; band counts from word 8.  Zeroed here unless the
    // caller (moe_forward) zeroed them earlier on the stream, so that the launch directly
    // follows the previous kernel (programmatic dependent launch needs no memset between)
    const int64_t slots = pair_done_slots(ph, n);
    if (!counters_zeroed &&
        cudaMemsetAsync(ctr + kFfnCounter, 0, (size_t)(8 - kFfnCounter + slots) * sizeof(int32_t), s) !=
            cudaSuccess)
      return MOE_ERR_CUDA;
    return cuda_status(launch_grouped_pair(ph, n, ctr + kFfnCounter, ctr + 8, s));
  }

  // the scattering store exists in the persistent pair launch only
  if (scatter != nullptr) return MOE_ERR_UNSUPPORTED;
  // Otherwise one launch per GEMM, each with its own tile counter.
  if (cudaMemsetAsync(ctr + 1, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  dn.dep = -1;
  sd.dep = -1;
  if (routed) {
    if (launch_grouped_gemm(up, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_grouped_gemm(dn, s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (shared) {
    if (launch_grouped_gemm(su, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_grouped_gemm(sd, s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const void* x,
                          const int32_t* expert_offsets, const void* packed, void* act,
                          void* y_perm, void* shared_out, void* workspace, int32_t* status,
                          void* stream) {
  const bool shared = cfg != nullptr && cfg->n_shared > 0 && shared_out != nullptr;
  return ffn_run(cfg, x_perm, x, expert_offsets, packed, act, y_perm, shared_out, workspace, status,
                 stream, true, shared);
}

moe_status moe_shared_ffn(const moe_config* cfg, const void* x, const void* packed, void* shared_out,
                          void* workspace, int32_t* status, void* stream) {
  return ffn_run(cfg, nullptr, x, nullptr, packed, nullptr, nullptr, shared_out, workspace, status,
                 stream, false, true);
}

moe_status moe_combine_unpermute(const moe_config* cfg, const void* y_perm, const int32_t* pos,
                                 const float* topk_w, const void* x, const void* shared_out,
                                 void* out, void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.T == 0) return MOE_OK;
  MOE_CHECK_PTR(y_perm);
  MOE_CHECK_PTR(pos);
  MOE_CHECK_PTR(topk_w);
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(out);
  if (out == x) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0) MOE_CHECK_PTR(shared_out);
  return cuda_status(launch_combine(c, (const bf16*)y_perm, pos, topk_w, x,
                                    c.n_shared > 0 ? (const bf16*)shared_out : nullptr, out,
                                    as_stream(stream)));
}

int32_t moe_route_dispatch_is_fused(const moe_config* cfg) {
  if (moe_validate_config(cfg) != MOE_OK) return 0;
  const char* env = getenv("MOE_ROUTE_FUSED");
  if (env && env[0] == '0') return 0;
  return route_pre_dispatch_applies(*cfg, ws_layout(*cfg).nblk) ? 1 : 0;
}

moe_status moe_route_dispatch(const moe_config* cfg, const void* x, const float* w_router,
                              const float* expert_bias, float* logits_out, int32_t* topk_idx,
                              float* topk_w, int32_t* counts, int32_t* expert_offsets,
                              int32_t* rank_splits, int32_t* rank_offsets, int32_t* pos,
                              int32_t* src, void* x_perm, void* workspace, int32_t* status,
                              void* stream) {
  return route_dispatch_run(cfg, x, w_router, expert_bias, logits_out, topk_idx, topk_w, counts,
                            expert_offsets, rank_splits, rank_offsets, pos, src, x_perm, workspace,
                            status, stream, nullptr);
}

moe_status moe_forward(const moe_config* cfg, const void* x, const float* w_router,
                       const float* expert_bias, const void* packed, float* logits_out,
                       int32_t* topk_idx, float* topk_w, int32_t* counts,
                       int32_t* expert_offsets, int32_t* rank_splits, int32_t* rank_offsets,
                       int32_t* pos, int32_t* src, void* x_perm, void* act, void* y_perm,
                       void* shared_out, void* out, void* workspace, int32_t* status,
                       void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(workspace);
  {
    // the expert FFN's tile counter and band counts (and, in words 6-7, the fused router's
    // grid barrier), zeroed before the router so that the FFN launch follows the dispatch
    // directly
    const WsLayout L = ws_layout(*cfg);
    int32_t* ctr = (int32_t*)((uint8_t*)workspace + L.counters);
    if (cfg->T > 0 && cudaMemsetAsync(ctr + kFfnCounter, 0,
                                      (8 - kFfnCounter + L.done_slots) * sizeof(int32_t),
                                      as_stream(stream)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  {
    // the fused router's grid-barrier words: two words of the block zeroed above
    const WsLayout L = ws_layout(*cfg);
    int32_t* ctr = (int32_t*)((uint8_t*)workspace + L.counters);
    st = route_dispatch_run(cfg, x, w_router, expert_bias, logits_out, topk_idx, topk_w, counts,
                            expert_offsets, rank_splits, rank_offsets, pos, src, x_perm, workspace,
                            status, stream, reinterpret_cast<unsigned*>(ctr + kFfnCounter + 1));
  }
  if (st != MOE_OK) return st;
  st = ffn_run(cfg, x_perm, x, expert_offsets, packed, act, y_perm, shared_out, workspace, status,
               stream, true, cfg->n_shared > 0 && shared_out != nullptr, true);
  if (st != MOE_OK) return st;
  return moe_combine_unpermute(cfg, y_perm, pos, topk_w, x, shared_out, out, stream);
}

moe_status moe_ep_local_ids(const moe_config* cfg, const int32_t* topk_idx, const int32_t* src,
                            int32_t* ids, void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.T == 0) return MOE_OK;
  MOE_CHECK_PTR(topk_idx);
  MOE_CHECK_PTR(src);
  MOE_CHECK_PTR(ids);
  return cuda_status(launch_local_ids(topk_idx, src, ids, c.T * c.top_k, c.E / c.ep_size,
                                      as_stream(stream)));
}

moe_status moe_gather_rows(const void* src, const int32_t* index, void* dst, int32_t n,
                           int32_t n_src, int32_t D, void* stream) {
  if (n < 0 || n_src < 0 || D <= 0 || D % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  MOE_CHECK_PTR(index);
  MOE_CHECK_PTR(dst);
  if (n_src > 0) MOE_CHECK_PTR(src);
  return cuda_status(launch_gather_rows((const bf16*)src, index, (bf16*)dst, n, n_src, D,
                                        as_stream(stream)));
}

// Host checks shared by the peer-exchange calls: a valid config, a peers table whose
// P is the config's ep_size, and a covered rank range inside [0, P).
static moe_status ep_check(const moe_config* cfg, const moe_ep_peers* peers, int32_t rank0,
                           int32_t nlocal) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  if (peers == nullptr || peers->P != cfg->ep_size || peers->P < 1 || peers->cap < 0) return MOE_ERR_INVALID_ARG;
  if (peers->cnt == nullptr || peers->flags == nullptr || peers->recv_x == nullptr ||
      peers->recv_src == nullptr || peers->recv_rank == nullptr || peers->y_back == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (nlocal < 1 || rank0 < 0 || rank0 + nlocal > peers->P) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status moe_ep_send_counts(const moe_config* cfg, const moe_ep_peers* peers, int32_t rank0,
                              int32_t nlocal, const int32_t* counts, uint32_t epoch, void* stream) {
  moe_status st = ep_check(cfg, peers, rank0, nlocal);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(counts);
  return cuda_status(launch_ep_send_counts(*peers, rank0, nlocal, counts, cfg->E, epoch, as_stream(stream)));
}

moe_status moe_ep_send_rows(const moe_config* cfg, const moe_ep_peers* peers, int32_t rank0,
                            int32_t nlocal, const void* x, const int32_t* topk_idx, const int32_t* pos,
                            const int32_t* expert_offsets, uint32_t epoch, int32_t* done,
                            int32_t* status, void* stream) {
  moe_status st = ep_check(cfg, peers, rank0, nlocal);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(expert_offsets);
  MOE_CHECK_PTR(done);
  MOE_CHECK_PTR(status);
  if (cfg->T > 0) {
    MOE_CHECK_PTR(x);
    MOE_CHECK_PTR(topk_idx);
    MOE_CHECK_PTR(pos);
  }
  return cuda_status(launch_ep_send_rows(*cfg, *peers, rank0, nlocal, x, topk_idx, pos, expert_offsets,
                                         done, status, epoch, as_stream(stream)));
}

moe_status moe_ep_recv_layout(const moe_config* cfg, const moe_ep_peers* peers, int32_t rank0,
                              int32_t nlocal, int32_t* local_offsets, uint32_t epoch, int32_t* status,
                              void* stream) {
  moe_status st = ep_check(cfg, peers, rank0, nlocal);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(local_offsets);
  MOE_CHECK_PTR(status);
  return cuda_status(launch_ep_recv_layout(*cfg, *peers, rank0, nlocal, local_offsets, status, epoch,
                                           as_stream(stream)));
}

moe_status moe_ep_return_rows(const moe_config* cfg, const moe_ep_peers* peers, int32_t rank0,
                              int32_t nlocal, const void* y_recv, const int32_t* local_offsets,
                              uint32_t epoch, int32_t* done, int32_t* status, void* stream) {
  moe_status st = ep_check(cfg, peers, rank0, nlocal);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(local_offsets);
  MOE_CHECK_PTR(done);
  MOE_CHECK_PTR(status);
  if (peers->cap > 0) MOE_CHECK_PTR(y_recv);
  return cuda_status(launch_ep_return_rows(*cfg, *peers, rank0, nlocal, y_recv, local_offsets, done,
                                           epoch, as_stream(stream)));
}

moe_status moe_ep_expert_ffn_return(const moe_config* cfg, const moe_config* local_cfg,
                                    const moe_ep_peers* peers, int32_t rank, const void* recv_x,
                                    const int32_t* recv_src, const int32_t* recv_rank,
                                    const int32_t* local_offsets, const void* packed, void* act,
                                    void* y_recv, void* workspace, uint32_t epoch, int32_t* done,
                                    int32_t* status, void* stream) {
  moe_status st = ep_check(cfg, peers, rank, 1);
  if (st != MOE_OK) return st;
  st = moe_validate_config(local_cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  const moe_config& l = *local_cfg;
  if (l.E * c.ep_size != c.E || l.D != c.D || l.F != c.F || l.act != c.act || l.top_k != 1 ||
      l.T != peers->cap || l.n_shared != c.n_shared || l.F_shared != c.F_shared)
    return MOE_ERR_INVALID_ARG;
  // int32 words read one at a time: 4-byte alignment is enough for these
  auto ptr4 = [](const void* q) { return q != nullptr && ((uintptr_t)q & 3u) == 0; };
  MOE_CHECK_PTR(local_offsets);
  if (!ptr4(done)) return MOE_ERR_INVALID_ARG;
  MOE_CHECK_PTR(status);
  if (peers->cap == 0) {
    return cuda_status(launch_ep_signal_returned(*peers, rank, epoch, as_stream(stream)));
  }
  MOE_CHECK_PTR(recv_x);
  if (!ptr4(recv_src) || !ptr4(recv_rank)) return MOE_ERR_INVALID_ARG;
  MOE_CHECK_PTR(packed);
  MOE_CHECK_PTR(act);
  MOE_CHECK_PTR(workspace);
  cudaStream_t s = as_stream(stream);
  // MOE_EP_FUSED_RETURN=0: the FFN into y_recv, then the separate return copy (for
  // comparison; also the form taken where the down GEMM does not run as a pair launch)
  const char* env = getenv("MOE_EP_FUSED_RETURN");
  if (!(env && env[0] == '0')) {
    const FfnScatter sc{(bf16* const*)peers->y_back, recv_rank, recv_src, peers->P, c.T * c.top_k};
    const int32_t* off = local_offsets;
    st = ffn_run(local_cfg, recv_x, nullptr, off, packed, act, nullptr, nullptr, workspace, status, stream,
                 true, false, false, &sc);
    if (st == MOE_OK) return cuda_status(launch_ep_signal_returned(*peers, rank, epoch, s));
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  MOE_CHECK_PTR(y_recv);
  st = ffn_run(local_cfg, recv_x, nullptr, local_offsets, packed, act, y_recv, nullptr, workspace, status,
               stream, true, false);
  if (st != MOE_OK) return st;
  return cuda_status(launch_ep_return_rows(c, *peers, rank, 1, y_recv, local_offsets, done, epoch, s));
}

moe_status moe_ep_wait_returned(const moe_config* cfg, const moe_ep_peers* peers, int32_t rank0,
                                int32_t nlocal, uint32_t epoch, int32_t* status, void* stream) {
  moe_status st = ep_check(cfg, peers, rank0, nlocal);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(status);
  return cuda_status(launch_ep_wait_returned(*peers, rank0, nlocal, status, epoch, as_stream(stream)));
}

moe_status moe_check_wait_timeout(uint32_t* barrier, int32_t* status, void* stream) {
  MOE_CHECK_PTR(barrier);
  MOE_CHECK_PTR(status);
  return cuda_status(launch_barrier_timeout_check(barrier, status, as_stream(stream)));
}

moe_status moe_router_filter_view(const moe_config* cfg, size_t* approx_offset, int32_t* approx_ld,
                                  size_t* wmax_offset, float* coef) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(approx_offset);
  MOE_CHECK_PTR(approx_ld);
  MOE_CHECK_PTR(wmax_offset);
  MOE_CHECK_PTR(coef);
  const moe_config& c = *cfg;
  const WsLayout L = ws_layout(c);
  if (!route_takes_filter(c, L.r_wmax - L.r_split, false)) return MOE_ERR_UNSUPPORTED;
  *approx_offset = L.r_approx;
  *approx_ld = (c.E + 127) / 128 * 128;
  *wmax_offset = L.r_wmax;
  *coef = route_filter_coef(c.D);
  return MOE_OK;
}

// A group's last <= 128 rows run as an M = 128 tile in the MXFP8 GEMMs (MOE_MX_HALF=0: as
// M = 256, for comparison); the quantiser of their A rows must lay the scales out the same way.
static int mx_half_tiles() {
  const char* env = getenv("MOE_MX_HALF");
  return (env && env[0] == '0') ? 0 : 1;
}
// A single-band group of 257..320 rows runs as one folded tile (the remainder as a product
// with the weights as M); MOE_MX_FOLD=0: as a full tile and a second one, for comparison.
// The folding kernel's ring has 5 stages instead of 6 (the remainder rows take shared
// memory), which costs 5-7 % where no group folds; so it runs only where groups of about
// 256 rows are expected: at most 512 routed rows per expert on average.  The quantiser
// of the A rows and both GEMMs take the same decision from the same config.
static int mx_fold(const moe_config& c) {
  const char* env = getenv("MOE_MX_FOLD");
  if (env && env[0] == '0') return 0;
  if (env && env[0] == '1') return 64;
  return (int64_t)c.T * c.top_k <= 512LL * c.E ? 64 : 0;
}

// MXFP8 routed experts: 256-wide N tiles on both GEMMs (gate_up width and D multiples of
// 256) and 128-deep K steps (D and F multiples of 128).
static moe_status mx_check(const moe_config* cfg) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const int nup = cfg->act == MOE_ACT_SWIGLU ? 2 * cfg->F : cfg->F;
  if (cfg->D % 256 != 0 || cfg->F % 128 != 0 || nup % 256 != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

size_t moe_packed_weights_mxfp8_size(const moe_config* cfg) {
  if (mx_check(cfg) != MOE_OK) return 0;
  return mx_pack_layout(*cfg).total;
}

size_t moe_workspace_mxfp8_size(const moe_config* cfg) {
  if (mx_check(cfg) != MOE_OK) return 0;
  return mx_ws_layout(*cfg).total;
}

moe_status moe_prepare_weights_mxfp8(const moe_config* cfg, const void* packed, void* packed_mx,
                                     void* stream) {
  moe_status st = mx_check(cfg);
  if (st != MOE_OK) return st;
  MOE_CHECK_PTR(packed);
  MOE_CHECK_PTR(packed_mx);
  const moe_config& c = *cfg;
  const PackLayout P = pack_layout(c);
  const MxPackLayout Q = mx_pack_layout(c);
  const uint8_t* pk = (const uint8_t*)packed;
  uint8_t* mx = (uint8_t*)packed_mx;
  cudaStream_t s = as_stream(stream);
  const int64_t nup = c.act == MOE_ACT_SWIGLU ? 2 * (int64_t)c.F : c.F;
  cudaError_t err = launch_mx_quant_rows((const bf16*)(pk + P.w_up), (int64_t)c.E * nup, c.D, mx + Q.w_up,
                                         mx + Q.sf_scratch, s);
  if (err == cudaSuccess) err = launch_mx_block_scales(mx + Q.sf_scratch, mx + Q.sf_up, (int64_t)c.E * nup, c.D, s);
  if (err == cudaSuccess)
    err = launch_mx_quant_rows((const bf16*)(pk + P.w_down), (int64_t)c.E * c.D, c.F, mx + Q.w_down,
                               mx + Q.sf_scratch, s);
  if (err == cudaSuccess) err = launch_mx_block_scales(mx + Q.sf_scratch, mx + Q.sf_down, (int64_t)c.E * c.D, c.F, s);
  return cuda_status(err);
}

moe_status moe_expert_ffn_mxfp8(const moe_config* cfg, const void* x_perm, const void* x,
                                const int32_t* expert_offsets, const void* packed, const void* packed_mx,
                                void* y_perm, void* shared_out, void* workspace, int32_t* status,
                                void* stream) {
  moe_status st = mx_check(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  MOE_CHECK_PTR(expert_offsets);
  MOE_CHECK_PTR(packed_mx);
  MOE_CHECK_PTR(workspace);
  MOE_CHECK_PTR(status);
  const int64_t R = (int64_t)c.T * c.top_k;
  if (R > 0) {
    if (x_perm != nullptr) MOE_CHECK_PTR(x_perm);
    MOE_CHECK_PTR(y_perm);
  }
  cudaStream_t s = as_stream(stream);
  const MxPackLayout Q = mx_pack_layout(c);
  const MxWsLayout L = mx_ws_layout(c);
  const uint8_t* mx = (const uint8_t*)packed_mx;
  uint8_t* ws = (uint8_t*)workspace;
  const int nup = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  int32_t* ctr = (int32_t*)(ws + L.counters);
  if (R > 0) {
    const int half = mx_half_tiles(), fold = mx_fold(c);
    cudaError_t err = cudaMemsetAsync(ctr, 0, 2 * sizeof(int32_t), s);
    // x_perm NULL: moe_dispatch_mxfp8 has already put the quantised rows in the workspace
    if (err == cudaSuccess && x_perm != nullptr)
      err = launch_mx_quant_a((const bf16*)x_perm, nullptr, 1, R, expert_offsets, c.E, c.D, half, fold,
                              ws + L.xq, ws + L.xsf, s);
    // gate_up (or W1): the activation comes out quantised, with the down projection's scales
    MxProblem up;
    memset(&up, 0, sizeof(up));
    up.A = ws + L.xq; up.a_rows = R; up.sa = ws + L.xsf;
    up.B = mx + Q.w_up; up.G = c.E; up.sb = mx + Q.sf_up;
    up.N = nup; up.K = c.D;
    up.group_offsets = expert_offsets;
    up.q_out = ws + L.aq; up.q_sf = ws + L.asf; up.ldo = c.F;
    up.epi = c.act == MOE_ACT_SWIGLU ? EPI_SWIGLU : EPI_GELU;
    up.half_tiles = half;
    up.fold = fold;
    up.status = status; up.counter = ctr;
    if (err == cudaSuccess) err = launch_grouped_mx(up, s);
    MxProblem dn = up;
    dn.A = ws + L.aq; dn.sa = ws + L.asf;
    dn.B = mx + Q.w_down; dn.sb = mx + Q.sf_down;
    dn.N = c.D; dn.K = c.F;
    dn.q_out = nullptr; dn.q_sf = nullptr;
    dn.out = (bf16*)y_perm; dn.ldo = c.D;
    dn.epi = EPI_STORE; dn.counter = ctr + 1;
    if (err == cudaSuccess) err = launch_grouped_mx(dn, s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  // the shared experts stay bf16 (the MXFP8 option covers the routed experts)
  if (c.n_shared > 0 && shared_out != nullptr)
    return moe_shared_ffn(cfg, x, packed, shared_out, workspace, status, stream);
  return MOE_OK;
}

moe_status moe_dispatch_mxfp8(const moe_config* cfg, const void* x, const int32_t* src,
                              const int32_t* expert_offsets, void* workspace, void* stream) {
  moe_status st = mx_check(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.x_dtype != MOE_DT_BF16) return MOE_ERR_UNSUPPORTED;
  MOE_CHECK_PTR(expert_offsets);
  MOE_CHECK_PTR(workspace);
  const int64_t R = (int64_t)c.T * c.top_k;
  if (R == 0) return MOE_OK;
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(src);
  const MxWsLayout L = mx_ws_layout(c);
  uint8_t* ws = (uint8_t*)workspace;
  return cuda_status(launch_mx_quant_a((const bf16*)x, src, c.top_k, R, expert_offsets, c.E, c.D,
                                       mx_half_tiles(), mx_fold(c), ws + L.xq, ws + L.xsf, as_stream(stream)));
}

moe_status moe_mxfp8_quantize(const void* x, int64_t rows, int32_t K, void* q, void* scales,
                              void* stream) {
  if (rows < 0 || K <= 0 || K % 32 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(q);
  if (scales == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_mx_quant_rows((const bf16*)x, rows, K, (uint8_t*)q, (uint8_t*)scales,
                                          as_stream(stream)));
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_INDEX_OOB: return "expert index out of range";
    case MOE_ERR_TIMEOUT: return "bounded wait expired in a kernel";
    case MOE_ERR_SCRATCH_LIMIT: return "configuration exceeds the no-alloc preprocess scratch";
  }
  return "unknown status";
}

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status moe_instr_read(int32_t kernel, uint64_t* counters, int32_t n) {
  if (counters == nullptr || n < 0 || (kernel != 0 && kernel != 1)) return MOE_ERR_INVALID_ARG;
  unsigned long long* h = reinterpret_cast<unsigned long long*>(counters);
  const cudaError_t e = kernel == 0 ? instr_read_pair(h, n) : instr_read_mx(h, n);
  if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return cuda_status(e);
}

}  // extern "C"
