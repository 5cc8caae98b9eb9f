// Device helpers shared by the router, the preprocess and the fused
// route + preprocess + dispatch kernel (each translation unit gets its own copy).
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr long long kBarrierLimitCycles = 2000000000ll;   // ~1 s at 2 GHz

// Eight terms of a router dot product, added to `acc` in order.  x (bf16 or fp32) and
// w (fp32) convert exactly to fp64 and their product needs at most 48 significant
// bits, so every term is exact and only the fp64 sums round: the logit, rounded once
// to fp32 at the end, is the exact dot product's fp32 value unless the fp64 rounding
// (relative 2^-53 of the largest partial sum) moves it across an fp32 rounding
// boundary.  With fp32 partial products, inputs whose partial sums are orders of
// magnitude above the logit (heavy cancellation) lost the digits that rank experts.
__device__ __forceinline__ double dot8_exact(const float (&x)[8], const float4& w0, const float4& w1,
                                             double acc) {
  acc = fma((double)x[0], (double)w0.x, acc);
  acc = fma((double)x[1], (double)w0.y, acc);
  acc = fma((double)x[2], (double)w0.z, acc);
  acc = fma((double)x[3], (double)w0.w, acc);
  acc = fma((double)x[4], (double)w1.x, acc);
  acc = fma((double)x[5], (double)w1.y, acc);
  acc = fma((double)x[6], (double)w1.z, acc);
  acc = fma((double)x[7], (double)w1.w, acc);
  return acc;
}

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

// Exclusive scan of vals[0..n) in place, returns the total (the whole block calls):
// one warp's shuffles for n <= 32, else block_scan_array.
__device__ __forceinline__ int scan_array(int* vals, int n, int* warp_sums, int* total) {
  if (n > 32) return block_scan_array(vals, n, warp_sums, total);
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    const int v = lane < n ? vals[lane] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane < n) vals[lane] = inc - v;
    if (lane == 31) *total = inc;
  }
  __syncthreads();
  const int t = *total;
  __syncthreads();            // every thread has read *total before a next call rewrites it
  return t;
}

// After the grid barrier of a cooperative preprocess over NB = gridDim.x blocks, each
// holding a contiguous chunk of the flat (token, slot) pairs and having published its
// per-expert histogram row in block_counts[blockIdx.x][E]: cnt[e] becomes the first
// row of expert e for this block's pairs (expert offset + pairs of e in earlier
// blocks); block 0 also writes counts, expert offsets and rank splits / offsets.
// tmp[E] is scratch.
template <int NT>
__device__ void pre_totals(const int32_t* block_counts, int E, int ep, int* cnt, int* tmp,
                           int* warp_sums, int* total, int32_t* counts,
                           int32_t* expert_offsets, int32_t* rank_splits, int32_t* rank_offsets) {
  const int tid = threadIdx.x;
  // rows of other blocks are read past L1, which is not coherent across SMs.  With
  // E < NT the blocks' rows of an expert are split over NT / E threads (their partial
  // sums added in shared memory), so few experts over many blocks still take only a
  // few dependent loads per thread; integer sums, exact in any order.
  const int tpe = E < NT ? NT / E : 1;
  if (tpe > 1) {
    for (int e = tid; e < E; e += NT) { cnt[e] = 0; tmp[e] = 0; }
    __syncthreads();
  }
  const int nb = (int)gridDim.x, me = (int)blockIdx.x;
  constexpr int kBatch = 16;                  // loads in flight per thread
  for (int i = tid; i < E * tpe; i += NT) {
    const int e = i % E, part = i / E;
    int before = 0, after = 0;
    for (int b0 = part; b0 < nb; b0 += tpe * kBatch) {
      int c[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int b = b0 + u * tpe;
        c[u] = b < nb ? __ldcg(block_counts + (size_t)b * E + e) : 0;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (b0 + u * tpe < me) before += c[u]; else after += c[u];
      }
    }
    if (tpe > 1) {
      atomicAdd(&cnt[e], before);
      atomicAdd(&tmp[e], before + after);
    } else {
      cnt[e] = before;
      tmp[e] = before + after;
    }
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e < E; e += NT) counts[e] = tmp[e];
  const int R_all = scan_array(tmp, E, warp_sums, total);          // tmp = expert offsets
  for (int e = tid; e < E; e += NT) cnt[e] += tmp[e];              // running row of e
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += NT) expert_offsets[e] = tmp[e];
    if (tid == 0) expert_offsets[E] = R_all;
    const int El = E / ep;
    for (int r = tid; r < ep; r += NT) {
      const int lo = tmp[r * El];
      const int hi = (r + 1) * El < E ? tmp[(r + 1) * El] : R_all;
      rank_splits[r] = hi - lo;
      rank_offsets[r] = lo;
    }
    if (tid == 0) rank_offsets[ep] = R_all;
  }
  __syncthreads();
}

// In-order rows of the block's pairs [base, end), NT pairs per round: a pair's row is
// cnt[e] + (pairs of e in earlier warps of the round) + (its rank among the lanes of
// its warp with the same expert, from __match_any_sync); cnt advances by the round's
// counts.  get_e(f) gives the pair's expert (< 0: skipped).  Writes pos[f] and src[row]
// (and pos_s[f - base] when given).  warp_cnt needs (NT / 32) * E ints.
template <int NT, class GetE>
__device__ void pre_positions(int base, int end, GetE get_e, int E, int* cnt, int* warp_cnt,
                              int32_t* pos, int32_t* src, int* pos_s) {
  constexpr int kWarps = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r0 = base; r0 < end; r0 += NT) {
    for (int i = tid; i < kWarps * E; i += NT) warp_cnt[i] = 0;
    __syncthreads();
    const int f = r0 + tid;
    const int e = f < end ? get_e(f) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_in_warp = __popc(peers & lt_mask);
    if (e >= 0 && rank_in_warp == 0) warp_cnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w * E + e];
      const int p = cnt[e] + before + rank_in_warp;
      pos[f] = p;
      src[p] = f;
      if (pos_s != nullptr) pos_s[f - base] = p;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += NT) {
      int s = 0;
      for (int w = 0; w < kWarps; ++w) s += warp_cnt[w * E + ee];
      cnt[ee] += s;
    }
    __syncthreads();
  }
}

// Warp argmax top-k over one logit per lane (lanes >= E hold none); returns the
// expert of selection `lane` (lanes < k).
__device__ __forceinline__ int warp_topk_write(float l, int E, int k, int renorm, size_t t,
                                                int32_t* __restrict__ topk_idx,
                                                float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  bool avail = lane < E;
  int my_idx = 0;
  float my_val = 0.f, top = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = avail ? l : -INFINITY;
    int bi = avail ? lane : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == bi) avail = false;
    if (lane == j) { my_idx = bi; my_val = bv; }
    if (j == 0) top = bv;
  }
  const float num = (lane < k) ? expf(my_val - top) : 0.f;
  float den = renorm ? num : (lane < E ? expf(l - top) : 0.f);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    topk_idx[t * k + lane] = my_idx;
    topk_w[t * k + lane] = num / den;
  }
  return my_idx;
}

}  // namespace
}  // namespace moe
