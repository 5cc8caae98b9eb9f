// Preprocess: per-expert counts, split sizes over the virtual EP ranks, and the
// deterministic dispatch order.
//
// "Expert Parallel (EP)", Communication Pattern step 1 (per-expert token counts
// and split sizes) and step 2 (permute tokens by expert assignment); section
// Overview, shard_experts(): experts split evenly and contiguously over ranks.
// "Worked Example: Tracing a Token Through Expert Parallelism", Steps 2-3.
//
// One cooperative launch over the R = T*k flat (token, slot) pairs, one block per
// contiguous chunk (at most one block per SM, so all blocks are resident):
//  1. each block counts its chunk per expert (warp-aggregated smem atomics:
//     counts are order-independent, so atomics keep them exact) and publishes
//     its row of the [block, expert] histogram;
//  2. a grid barrier (bounded wait; a stuck barrier reports MOE_ERR_TIMEOUT);
//  3. every block reads the histogram, forms its per-expert base (pairs of e in
//     earlier blocks) and the global exclusive scan; block 0 writes counts,
//     expert offsets and rank splits/offsets;
//  4. each block walks its chunk in order; a pair's row is offset[e] + base[e] +
//     (earlier pairs of e in this block), the last term from __match_any_sync
//     ranks within a warp plus per-warp counts of earlier warps.  Rows follow
//     the flat index, so tokens ascend inside each expert: no atomic decides order.
#include "device_util.cuh"

namespace moe {

namespace {

constexpr int kPreWarps = kPreThreads / 32;

struct PreArgs {
  const int32_t* idx;
  int R, E, ep, chunk;
  int32_t* block_counts;   // [gridDim.x][E]
  unsigned* barrier;       // [2], zero at launch
  int32_t *counts, *expert_offsets, *rank_splits, *rank_offsets, *pos, *src, *status;
};

__global__ void __launch_bounds__(kPreThreads)
pre_fused_kernel(const PreArgs a) {
  extern __shared__ int sm[];
  const int E = a.E;
  int* cnt = sm;                       // [E]  histogram, then running row base
  int* tmp = sm + E;                   // [E]  scan scratch
  int* warp_cnt = sm + 2 * E;          // [kPreWarps][E]
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int tid = threadIdx.x;
  const int base = blockIdx.x * a.chunk;
  const int end = min(base + a.chunk, a.R);

  // 1. histogram of this block's chunk
  for (int e = tid; e < E; e += kPreThreads) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int f = base + tid; f < end; f += kPreThreads) {
    const int e = __ldg(a.idx + f);
    if ((unsigned)e >= (unsigned)E) { bad = true; continue; }
    atomicAdd(&cnt[e], 1);
  }
  if (bad) atomicCAS(a.status, 0, (int)MOE_ERR_INDEX_OOB);
  __syncthreads();
  for (int e = tid; e < E; e += kPreThreads)
    a.block_counts[(size_t)blockIdx.x * E + e] = cnt[e];

  // 2. all histograms published
  if (!grid_barrier(a.barrier, gridDim.x, a.status)) return;

  // 3. per-expert base of this block, global totals and the block-0 outputs
  pre_totals<kPreThreads>(a.block_counts, E, a.ep, cnt, tmp, warp_sums, &total, a.counts,
                          a.expert_offsets, a.rank_splits, a.rank_offsets);

  // 4. in-order scatter of this block's chunk, kPreThreads pairs per round
  pre_positions<kPreThreads>(
      base, end,
      [&](int f) {
        const int e = __ldg(a.idx + f);
        return (unsigned)e < (unsigned)E ? e : -1;   // out of range: reported in step 1
      },
      E, cnt, warp_cnt, a.pos, a.src, nullptr);
}

// One block waits at a grid barrier sized for two blocks: nothing completes it, so the
// bounded wait of grid_barrier (the one the cooperative kernels use) runs out, records
// MOE_ERR_TIMEOUT in *status and the kernel returns.
__global__ void barrier_timeout_check_kernel(unsigned* bar, int32_t* status) {
  grid_barrier(bar, 2u, status);
}

}  // namespace

cudaError_t launch_barrier_timeout_check(unsigned* barrier, int32_t* status, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(barrier, 0, 2 * sizeof(unsigned), s);
  if (err != cudaSuccess) return err;
  barrier_timeout_check_kernel<<<1, 32, 0, s>>>(barrier, status);
  return cudaGetLastError();
}

int preprocess_blocks(int64_t R) {
  const int64_t want = (R + kPreThreads - 1) / kPreThreads;
  return (int)(want < kPreMaxBlocks ? (want > 0 ? want : 1) : kPreMaxBlocks);
}

cudaError_t launch_preprocess(const moe_config& c, const int32_t* topk_idx, int32_t* counts,
                              int32_t* expert_offsets, int32_t* rank_splits,
                              int32_t* rank_offsets, int32_t* pos, int32_t* src,
                              int32_t* block_counts, int max_blocks,
                              unsigned* barrier, int32_t* status, cudaStream_t s) {
  const int R = c.T * c.top_k;
  const int sms = sm_count();
  int nblk = preprocess_blocks(R);
  if (nblk > max_blocks) nblk = max_blocks;
  if (nblk > sms) nblk = sms;                   // one block per SM: all resident
  const int chunk = ((R + nblk - 1) / nblk + kPreThreads - 1) / kPreThreads * kPreThreads;
  cudaError_t err = cudaMemsetAsync(barrier, 0, 2 * sizeof(unsigned), s);
  if (err != cudaSuccess) return err;
  PreArgs a;
  a.idx = topk_idx; a.R = R; a.E = c.E; a.ep = c.ep_size; a.chunk = chunk;
  a.block_counts = block_counts; a.barrier = barrier;
  a.counts = counts; a.expert_offsets = expert_offsets; a.rank_splits = rank_splits;
  a.rank_offsets = rank_offsets; a.pos = pos; a.src = src; a.status = status;
  const size_t smem = (size_t)c.E * sizeof(int) * (2 + kPreWarps);
  if (smem > (48u << 10)) {
    err = cudaFuncSetAttribute(pre_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  void* args[] = {&a};
  err = cudaLaunchCooperativeKernel((const void*)pre_fused_kernel, dim3(nblk), dim3(kPreThreads),
                                    args, smem, s);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
