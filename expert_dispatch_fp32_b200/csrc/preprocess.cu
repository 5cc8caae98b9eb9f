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
//     expert offsets, rank splits/offsets and the GEMM M-tile prefixes;
//  4. each block walks its chunk in order; a pair's row is offset[e] + base[e] +
//     (earlier pairs of e in this block), the last term from __match_any_sync
//     ranks within a warp plus per-warp counts of earlier warps.  Rows follow
//     the flat index, so tokens ascend inside each expert: no atomic decides order.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr long long kBarrierLimitCycles = 2000000000ll;   // ~1 s at 2 GHz
constexpr int kPreWarps = kPreThreads / 32;

// Grid-wide barrier for a cooperative launch.  bar[0] counts arrivals, bar[1] is a
// generation the last arrival bumps; both start at zero (set on the stream before
// the launch).  Bounded: after kBarrierLimitCycles a waiting block reports
// MOE_ERR_TIMEOUT and the kernel returns without touching the outputs further.
__device__ bool grid_barrier(unsigned* bar, unsigned nblocks, int32_t* status) {
  __threadfence();
  __syncthreads();
  int ok = 1;
  if (threadIdx.x == 0) {
    volatile unsigned* gen = bar + 1;
    const unsigned g = *gen;
    if (atomicAdd(bar, 1u) == nblocks - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const long long t0 = clock64();
      while (*gen == g) {
        if (clock64() - t0 > kBarrierLimitCycles) {
          atomicCAS(status, 0, (int)MOE_ERR_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(100);
      }
    }
    __threadfence();
  }
  return __syncthreads_and(ok) != 0;
}

// Exclusive scan over the block of one value per thread; *total gets the sum.
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
    if (lane < nwarps) warp_sums[lane] = s;
    if (lane == 31) *total = s;
  }
  __syncthreads();
  const int before = warp > 0 ? warp_sums[warp - 1] : 0;
  const int r = before + inc - v;
  __syncthreads();
  return r;
}

// Exclusive scan of vals[0..n) in place (n <= kMaxExperts), returns the total.
// Thread i scans the contiguous run [i*per, (i+1)*per).
__device__ int block_scan_array(int* vals, int n, int* warp_sums, int* total) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per, hi = min(lo + per, n);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += vals[i];
  int run = block_exclusive_scan(local, warp_sums, total);
  for (int i = lo; i < hi; ++i) {
    const int v = vals[i];
    vals[i] = run;
    run += v;
  }
  __syncthreads();
  return *total;
}

struct PreArgs {
  const int32_t* idx;
  int R, E, ep, chunk;
  int32_t* block_counts;   // [gridDim.x][E]
  unsigned* barrier;       // [2], zero at launch
  int32_t *counts, *expert_offsets, *rank_splits, *rank_offsets, *mt_start, *pos, *src, *status;
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
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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

  // 3. per-expert base of this block and global totals (rows of other blocks are
  //    read past L1, which is not coherent across SMs)
  for (int e = tid; e < E; e += kPreThreads) {
    int before = 0, after = 0;
    for (int b = 0; b < (int)gridDim.x; ++b) {
      const int c = __ldcg(a.block_counts + (size_t)b * E + e);
      if (b < (int)blockIdx.x) before += c; else after += c;
    }
    cnt[e] = before;
    tmp[e] = before + after;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e < E; e += kPreThreads) a.counts[e] = tmp[e];
  const int R_all = block_scan_array(tmp, E, warp_sums, &total);   // tmp = expert offsets
  for (int e = tid; e < E; e += kPreThreads) cnt[e] += tmp[e];      // running row of e
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += kPreThreads) a.expert_offsets[e] = tmp[e];
    if (tid == 0) a.expert_offsets[E] = R_all;
    const int El = E / a.ep;
    for (int r = tid; r < a.ep; r += kPreThreads) {
      const int lo = tmp[r * El];
      const int hi = (r + 1) * El < E ? tmp[(r + 1) * El] : R_all;
      a.rank_splits[r] = hi - lo;
      a.rank_offsets[r] = lo;
    }
    if (tid == 0) a.rank_offsets[a.ep] = R_all;
    // GEMM M-tile prefixes: [0, E] for 128-row tiles, [E+1, 2E+1] for 256-row tiles
    for (int half = 0; half < 2; ++half) {
      const int tm = half ? 2 * kTileM : kTileM;
      int* outp = a.mt_start + half * (E + 1);
      __syncthreads();
      for (int e = tid; e < E; e += kPreThreads) {
        const int ce = (e + 1 < E ? tmp[e + 1] : R_all) - tmp[e];
        warp_cnt[e] = (ce + tm - 1) / tm;        // warp_cnt is free until step 4
      }
      __syncthreads();
      const int tiles = block_scan_array(warp_cnt, E, warp_sums, &total);
      for (int e = tid; e < E; e += kPreThreads) outp[e] = warp_cnt[e];
      if (tid == 0) outp[E] = tiles;
    }
  }
  __syncthreads();

  // 4. in-order scatter of this block's chunk, kPreThreads pairs per round
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r0 = base; r0 < end; r0 += kPreThreads) {
    for (int i = tid; i < kPreWarps * E; i += kPreThreads) warp_cnt[i] = 0;
    __syncthreads();
    const int f = r0 + tid;
    int e = -1;
    if (f < end) {
      e = __ldg(a.idx + f);
      if ((unsigned)e >= (unsigned)E) e = -1;   // reported in step 1
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_in_warp = __popc(peers & lt_mask);
    if (e >= 0 && rank_in_warp == 0) warp_cnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w * E + e];
      const int p = cnt[e] + before + rank_in_warp;
      a.pos[f] = p;
      a.src[p] = f;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPreThreads) {
      int s = 0;
      for (int w = 0; w < kPreWarps; ++w) s += warp_cnt[w * E + ee];
      cnt[ee] += s;
    }
    __syncthreads();
  }
}

}  // namespace

int preprocess_blocks(int64_t R) {
  const int64_t want = (R + kPreThreads - 1) / kPreThreads;
  return (int)(want < kPreMaxBlocks ? (want > 0 ? want : 1) : kPreMaxBlocks);
}

cudaError_t launch_preprocess(const moe_config& c, const int32_t* topk_idx, int32_t* counts,
                              int32_t* expert_offsets, int32_t* rank_splits,
                              int32_t* rank_offsets, int32_t* pos, int32_t* src,
                              int32_t* block_counts, int max_blocks, int32_t* mt_start,
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
  a.rank_offsets = rank_offsets; a.mt_start = mt_start; a.pos = pos; a.src = src; a.status = status;
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
