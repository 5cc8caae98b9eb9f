// Preprocess: per-expert counts, split sizes over the virtual EP ranks, and the
// deterministic dispatch order.
//
// "Expert Parallel (EP)", Communication Pattern step 1 (per-expert token counts
// and split sizes) and step 2 (permute tokens by expert assignment); section
// Overview, shard_experts(): experts split evenly and contiguously over ranks.
// "Worked Example: Tracing a Token Through Expert Parallelism", Steps 2-3.
//
// Three small kernels over the R = T*k flat (token, slot) pairs:
//  1. hist:    each block counts its chunk of pairs per expert (smem atomics;
//              counts are order-independent, so atomics keep them exact).
//  2. scan:    one block turns the [block, expert] histogram into per-block
//              bases (a column scan), counts, expert offsets, rank splits,
//              rank offsets and the per-expert GEMM M-tile prefix.
//  3. scatter: each block re-reads its chunk in order; a pair's row is
//              offset[e] + (pairs of e in earlier blocks) + (earlier pairs of e
//              in this block), the last term from __match_any_sync ranks within
//              a warp plus per-warp counts of earlier warps.  Rows follow the flat
//              index, so tokens ascend inside each expert: no atomics decide order.
#include "moe_internal.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(kPreThreads)
pre_hist_kernel(const int32_t* __restrict__ idx, int R, int E, int32_t* __restrict__ block_counts,
                int32_t* status) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kPreChunk;
  bool bad = false;
  for (int i = threadIdx.x; i < kPreChunk; i += blockDim.x) {
    const int f = base + i;
    if (f >= R) break;
    const int e = __ldg(idx + f);
    if ((unsigned)e >= (unsigned)E) { bad = true; continue; }
    atomicAdd(&hist[e], 1);
  }
  if (bad) atomicCAS(status, 0, (int)MOE_ERR_INDEX_OOB);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    block_counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// Exclusive scan of one value per thread over a block of up to 1024 threads.
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    if (lane < nwarps) warp_sums[lane] = s;     // inclusive prefix of warp sums
    if (lane == 31) *total = s;
  }
  __syncthreads();
  const int before = warp > 0 ? warp_sums[warp - 1] : 0;
  const int r = before + inc - v;
  __syncthreads();
  return r;
}

// One block of 1024 threads; thread e owns expert e (E <= 1024).
__global__ void __launch_bounds__(1024)
pre_scan_kernel(int32_t* __restrict__ block_counts, int nblk, int E, int ep,
                int32_t* __restrict__ counts, int32_t* __restrict__ expert_offsets,
                int32_t* __restrict__ rank_splits, int32_t* __restrict__ rank_offsets,
                int32_t* __restrict__ mt_start) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  __shared__ int cnt_s[kMaxExperts];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {           // column scan: per-block base of expert e
      const size_t i = (size_t)b * E + e;
      const int c = block_counts[i];
      block_counts[i] = run;
      run += c;
    }
    counts[e] = run;
    cnt_s[e] = run;
  }
  const int off = block_exclusive_scan(e < E ? run : 0, warp_sums, &total);
  if (e < E) expert_offsets[e] = off;
  if (e == 0) expert_offsets[E] = total;
  // GEMM M-tile prefixes: [0, E] for 128-row tiles, [E+1, 2E+1] for 256-row tiles
  const int tiles = e < E ? (run + kTileM - 1) / kTileM : 0;
  const int toff = block_exclusive_scan(tiles, warp_sums, &total);
  if (e < E) mt_start[e] = toff;
  if (e == 0) mt_start[E] = total;
  const int tiles2 = e < E ? (run + 2 * kTileM - 1) / (2 * kTileM) : 0;
  const int toff2 = block_exclusive_scan(tiles2, warp_sums, &total);
  if (e < E) mt_start[E + 1 + e] = toff2;
  if (e == 0) mt_start[2 * E + 1] = total;
  __syncthreads();
  const int El = E / ep;
  int split = 0;
  if (e < ep)
    for (int i = 0; i < El; ++i) split += cnt_s[e * El + i];
  const int roff = block_exclusive_scan(e < ep ? split : 0, warp_sums, &total);
  if (e < ep) { rank_splits[e] = split; rank_offsets[e] = roff; }
  if (e == 0) rank_offsets[ep] = total;
}

__global__ void __launch_bounds__(kPreThreads)
pre_scatter_kernel(const int32_t* __restrict__ idx, int R, int E,
                   const int32_t* __restrict__ block_base, const int32_t* __restrict__ expert_offsets,
                   int32_t* __restrict__ pos, int32_t* __restrict__ src) {
  constexpr int kWarps = kPreThreads / 32;
  extern __shared__ int sm[];
  int* running = sm;                 // [E]
  int* warp_cnt = sm + E;            // [kWarps][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += kPreThreads)
    running[e] = expert_offsets[e] + block_base[(size_t)blockIdx.x * E + e];
  const unsigned lt_mask = (1u << lane) - 1u;
  const int base = blockIdx.x * kPreChunk;
  for (int r0 = 0; r0 < kPreChunk; r0 += kPreThreads) {
    for (int i = tid; i < kWarps * E; i += kPreThreads) warp_cnt[i] = 0;
    __syncthreads();
    const int f = base + r0 + tid;
    int e = -1;
    if (f < R) {
      e = __ldg(idx + f);
      if ((unsigned)e >= (unsigned)E) e = -1;   // reported by the histogram pass
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_in_warp = __popc(peers & lt_mask);
    if (e >= 0 && rank_in_warp == 0) warp_cnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w * E + e];
      const int p = running[e] + before + rank_in_warp;
      pos[f] = p;
      src[p] = f;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPreThreads) {
      int s = 0;
      for (int w = 0; w < kWarps; ++w) s += warp_cnt[w * E + ee];
      running[ee] += s;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_preprocess(const moe_config& c, const int32_t* topk_idx, int32_t* counts,
                              int32_t* expert_offsets, int32_t* rank_splits,
                              int32_t* rank_offsets, int32_t* pos, int32_t* src,
                              int32_t* block_counts, int nblk, int32_t* mt_start,
                              int32_t* status, cudaStream_t s) {
  const int R = c.T * c.top_k;
  const int E = c.E;
  if (nblk > 0) {
    pre_hist_kernel<<<nblk, kPreThreads, E * sizeof(int), s>>>(topk_idx, R, E, block_counts, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  pre_scan_kernel<<<1, 1024, 0, s>>>(block_counts, nblk, E, c.ep_size, counts, expert_offsets,
                                     rank_splits, rank_offsets, mt_start);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || nblk == 0) return err;
  const size_t smem = (size_t)E * sizeof(int) * (1 + kPreThreads / 32);
  pre_scatter_kernel<<<nblk, kPreThreads, smem, s>>>(topk_idx, R, E, block_counts, expert_offsets,
                                                      pos, src);
  return cudaGetLastError();
}

}  // namespace moe
