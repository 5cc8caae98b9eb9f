// Router, preprocess and dispatch in one cooperative launch, for few experts.
//
// "Expert Parallel (EP)", Communication Pattern steps 1-2 (gate + top-k, per-expert
// counts and split sizes, tokens permuted by expert assignment); "Worked Example:
// Tracing a Token Through Expert Parallelism", Steps 1-2.
//
// Block b owns tokens [b * tpb, (b + 1) * tpb) and, for the preprocess, the flat
// (token, slot) pairs of those tokens:
//  1. W_r and the block's x rows are brought into shared memory by bulk copies, each
//     warp's rows on a barrier of its own, so routing starts as its rows land;
//  2. each warp routes TW tokens at a time with the arithmetic of the few-expert
//     router (exact fp64 terms summed in fp64, lane-parallel over D, exact
//     argmax top-k, renormalised softmax weights) and keeps the selections;
//  3. the block's per-expert histogram goes out, then one grid barrier;
//  4. the totals, expert offsets and rank splits, and the in-order
//     rows of the block's pairs, exactly as the preprocess computes them;
//  5. each pair's x row is written to x_perm from shared memory (bf16).
// Every output is bit-identical to moe_route + moe_preprocess +
// moe_dispatch_permute; x is read from HBM once.
#include "device_util.cuh"

namespace moe {

namespace {

constexpr int kFuseThreads = 512;
constexpr int kFuseWarps = kFuseThreads / 32;

struct FuseArgs {
  const void* x;
  const float* w;
  const float* bias;
  float* logits_out;
  int32_t* topk_idx;
  float* topk_w;
  int T, D, E, k, renorm, ep, tpb;
  int32_t* block_counts;   // [gridDim.x][E]
  unsigned* barrier;       // [2], zero at launch
  int32_t *counts, *expert_offsets, *rank_splits, *rank_offsets, *pos, *src, *status;
  bf16* x_perm;
};

__device__ __forceinline__ void x8(const bf16* p, float (&v)[8]) {
  const uint4 t = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&t);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(h[q]);
    v[2 * q] = f.x; v[2 * q + 1] = f.y;
  }
}
__device__ __forceinline__ void x8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr long long kFuseWaitLimitCycles = 2000000000ll;   // about 1 s at 2 GHz

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase 0 of a staging barrier: false (and MOE_ERR_TIMEOUT) on expiry.
__device__ __noinline__ bool mbar_wait0(uint32_t bar, int32_t* status) {
  const long long t0 = clock64();
  while (!mbar_test(bar, 0)) {
    if (clock64() - t0 > kFuseWaitLimitCycles) {
      atomicCAS(status, 0, (int)MOE_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// Bulk copy (the copy engine) of `bytes` from shared to global memory (bulk group).
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_addr(src)), "r"(bytes)
               : "memory");
}
// Bulk copy (the copy engine) of `bytes` from global to shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <int EP, int TW, typename XT>
__global__ void __launch_bounds__(kFuseThreads, 1) route_pre_dispatch_kernel(const FuseArgs a) {
  extern __shared__ uint4 fsm[];
  const int E = a.E, D = a.D, k = a.k;
  const int t_lo = blockIdx.x * a.tpb;
  const int ntok = max(min(t_lo + a.tpb, a.T) - t_lo, 0);
  float* w_s = reinterpret_cast<float*>(fsm);                          // [E * D]
  XT* x_s = reinterpret_cast<XT*>(w_s + (size_t)E * D);               // [tpb * D]
  int* sel = reinterpret_cast<int*>(x_s + (size_t)a.tpb * D);         // [tpb * k]
  int* pos_s = sel + a.tpb * k;                                       // [tpb * k]
  int* cnt = pos_s + a.tpb * k;                                       // [E]
  int* tmp = cnt + E;                                                 // [E]
  int* warp_cnt = tmp + E;                                            // [kFuseWarps * E]
  __shared__ int warp_sums[32];
  __shared__ int total;
  __shared__ __align__(8) uint64_t bars[1 + kFuseWarps];              // W_r, each warp's x rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // 1. bulk copies into shared memory: W_r on bars[0], warp w's token rows on bars[1 + w],
  //    so a warp starts routing once W_r and its own rows are in
  if (tid == 0) {
    for (int i = 0; i <= kFuseWarps; ++i) mbar_init(smem_addr(&bars[i]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const uint32_t xrow = (uint32_t)D * (uint32_t)sizeof(XT);
  if (tid == 0) {
    mbar_expect(smem_addr(&bars[0]), (uint32_t)E * D * 4);
    bulk_g2s(w_s, a.w, (uint32_t)E * D * 4, smem_addr(&bars[0]));
    const XT* xg = static_cast<const XT*>(a.x) + (size_t)t_lo * D;
    for (int w = 0; w < kFuseWarps; ++w) {
      uint32_t n = 0;
      for (int g0 = w * TW; g0 < ntok; g0 += kFuseWarps * TW) n += (uint32_t)min(TW, ntok - g0);
      const uint32_t bar = smem_addr(&bars[1 + w]);
      mbar_expect(bar, n * xrow);
      for (int g0 = w * TW; g0 < ntok; g0 += kFuseWarps * TW)
        for (int i = 0; i < TW && g0 + i < ntok; ++i)
          bulk_g2s(x_s + (size_t)(g0 + i) * D, xg + (size_t)(g0 + i) * D, xrow, bar);
    }
  }
  {
    bool ok = true;
    if (lane == 0) ok = mbar_wait0(smem_addr(&bars[0]), a.status) && mbar_wait0(smem_addr(&bars[1 + warp]), a.status);
    // on a timeout (reported) the warp goes on with whatever shared memory holds
    __syncwarp();
    (void)ok;
  }

  // 2. route: the few-expert router's arithmetic, x from shared memory
  for (int g0 = warp * TW; g0 < ntok; g0 += kFuseWarps * TW) {
    double acc[TW][EP];
#pragma unroll
    for (int i = 0; i < TW; ++i)
#pragma unroll
      for (int e = 0; e < EP; ++e) acc[i][e] = 0.0;
    for (int d0 = lane * 8; d0 < D; d0 += 256) {
      float xv[TW][8];
#pragma unroll
      for (int i = 0; i < TW; ++i) {
        if (g0 + i < ntok) {
          x8(x_s + (size_t)(g0 + i) * D + d0, xv[i]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) xv[i][q] = 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E) {
          const float4 w0 = *reinterpret_cast<const float4*>(w_s + (size_t)e * D + d0);
          const float4 w1 = *reinterpret_cast<const float4*>(w_s + (size_t)e * D + d0 + 4);
#pragma unroll
          for (int i = 0; i < TW; ++i) {
            acc[i][e] = dot8_exact(xv[i], w0, w1, acc[i][e]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TW; ++i)
#pragma unroll
      for (int e = 0; e < EP; ++e)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], o);
#pragma unroll
    for (int i = 0; i < TW; ++i) {
      if (g0 + i >= ntok) break;
      const int t = t_lo + g0 + i;
      float l = -INFINITY;
#pragma unroll
      for (int e = 0; e < EP; ++e)
        if (lane == e) l = (float)acc[i][e];
      if (lane < E && a.bias != nullptr) l = l + a.bias[lane];
      if (a.logits_out != nullptr && lane < E) a.logits_out[(size_t)t * E + lane] = l;
      const int s = warp_topk_write(l, E, k, a.renorm, (size_t)t, a.topk_idx, a.topk_w);
      if (lane < k) {
        // an expert id out of range (only NaN logits give one) is what the preprocess
        // reports as MOE_ERR_INDEX_OOB and skips; so here
        const bool ok = (unsigned)s < (unsigned)E;
        sel[(g0 + i) * k + lane] = ok ? s : -1;
        if (!ok) atomicCAS(a.status, 0, (int)MOE_ERR_INDEX_OOB);
      }
    }
  }
  __syncthreads();

  // 3. this block's histogram, then every block's
  for (int e = tid; e < E; e += kFuseThreads) cnt[e] = 0;
  __syncthreads();
  for (int f = tid; f < ntok * k; f += kFuseThreads)
    if (sel[f] >= 0) atomicAdd(&cnt[sel[f]], 1);
  __syncthreads();
  for (int e = tid; e < E; e += kFuseThreads) a.block_counts[(size_t)blockIdx.x * E + e] = cnt[e];
  if (!grid_barrier(a.barrier, gridDim.x, a.status)) return;

  // 4. totals and block-0 outputs, then the in-order rows of the block's pairs
  pre_totals<kFuseThreads>(a.block_counts, E, a.ep, cnt, tmp, warp_sums, &total, a.counts,
                           a.expert_offsets, a.rank_splits, a.rank_offsets);
  const int base = t_lo * k;
  pre_positions<kFuseThreads>(base, base + ntok * k, [&](int f) { return sel[f - base]; }, E, cnt,
                              warp_cnt, a.pos, a.src, pos_s);

  // the expert FFN (launched as a programmatic dependent) may start launching now
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // 5. dispatch from shared memory.  bf16 x: the row is already x_perm's bytes, one bulk
  //    copy per pair (issued by lane 0 of a warp, which waits until its copies have read
  //    shared memory before the block may exit); fp32 x: a warp per pair converts.
  if (sizeof(XT) == 2) {
    if (lane == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      int issued = 0;
      for (int f = warp; f < ntok * k; f += kFuseWarps) {
        if (sel[f] < 0) continue;                    // no row (reported above)
        bulk_s2g(a.x_perm + (size_t)pos_s[f] * D, x_s + (size_t)(f / k) * D, (uint32_t)D * 2);
        ++issued;
      }
      if (issued) {
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      }
    }
    return;
  }
  const int cpr = D >> 3;
  for (int f = warp; f < ntok * k; f += kFuseWarps) {
    if (sel[f] < 0) continue;                        // no row (reported above)
    const XT* row = x_s + (size_t)(f / k) * D;
    bf16* dst = a.x_perm + (size_t)pos_s[f] * D;
    for (int ch = lane; ch < cpr; ch += 32) {
      float v[8];
      x8(row + ch * 8, v);
      uint4 o;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
      *reinterpret_cast<uint4*>(dst + ch * 8) = o;
    }
  }
}

size_t fuse_smem(const moe_config& c, int tpb) {
  const size_t sx = c.x_dtype == MOE_DT_F32 ? 4 : 2;
  return (size_t)c.E * c.D * 4 + (size_t)tpb * c.D * sx + 2 * (size_t)tpb * c.top_k * 4 +
         (size_t)(2 + kFuseWarps) * c.E * 4;
}

template <int EP, int TW, typename XT>
cudaError_t launch_fused(const FuseArgs& a, int grid, size_t smem, cudaStream_t s) {
  auto kern = route_pre_dispatch_kernel<EP, TW, XT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int occ = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kFuseThreads, smem);
  if (err != cudaSuccess) return err;
  if ((int64_t)occ * sm_count() < grid) return cudaErrorCooperativeLaunchTooLarge;
  FuseArgs args = a;
  void* p[] = {&args};
  err = cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(kFuseThreads), p, smem, s);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

// Shared-memory budget of the fused kernel (W_r, the block's x rows, selections, rows).
constexpr size_t kFuseSmemLimit = 200u << 10;

bool route_pre_dispatch_applies(const moe_config& c, int max_blocks) {
  if (c.T <= 0 || c.E > 32) return false;
  int grid = sm_count();
  if (grid > max_blocks) grid = max_blocks;
  if (grid > c.T) grid = c.T;
  const int tpb = (c.T + grid - 1) / grid;
  return fuse_smem(c, tpb) <= kFuseSmemLimit;
}

cudaError_t launch_route_pre_dispatch(const moe_config& c, const void* x, const float* w,
                                      const float* bias, float* logits_out, int32_t* topk_idx,
                                      float* topk_w, int32_t* counts, int32_t* expert_offsets,
                                      int32_t* rank_splits, int32_t* rank_offsets, int32_t* pos,
                                      int32_t* src, int32_t* block_counts, int max_blocks,
                                      unsigned* barrier, bool barrier_zeroed,
                                      bf16* x_perm, int32_t* status, cudaStream_t s) {
  int grid = sm_count();
  if (grid > max_blocks) grid = max_blocks;
  if (grid > c.T) grid = c.T;
  if (grid < 1) return cudaErrorInvalidValue;
  const int tpb = (c.T + grid - 1) / grid;
  grid = (c.T + tpb - 1) / tpb;                    // no empty block
  const size_t smem = fuse_smem(c, tpb);
  if (smem > kFuseSmemLimit || c.E > 32) return cudaErrorInvalidValue;
  if (!barrier_zeroed) {
    const cudaError_t err = cudaMemsetAsync(barrier, 0, 2 * sizeof(unsigned), s);
    if (err != cudaSuccess) return err;
  }
  FuseArgs a;
  a.x = x; a.w = w; a.bias = bias; a.logits_out = logits_out; a.topk_idx = topk_idx; a.topk_w = topk_w;
  a.T = c.T; a.D = c.D; a.E = c.E; a.k = c.top_k; a.renorm = c.renormalize; a.ep = c.ep_size;
  a.tpb = tpb;
  a.block_counts = block_counts; a.barrier = barrier;
  a.counts = counts; a.expert_offsets = expert_offsets; a.rank_splits = rank_splits;
  a.rank_offsets = rank_offsets; a.pos = pos; a.src = src; a.status = status;
  a.x_perm = x_perm;
  const bool f32 = c.x_dtype == MOE_DT_F32;
  if (c.E <= 8)
    return f32 ? launch_fused<8, 2, float>(a, grid, smem, s) : launch_fused<8, 2, bf16>(a, grid, smem, s);
  if (c.E <= 16)
    return f32 ? launch_fused<16, 1, float>(a, grid, smem, s) : launch_fused<16, 1, bf16>(a, grid, smem, s);
  return f32 ? launch_fused<32, 1, float>(a, grid, smem, s) : launch_fused<32, 1, bf16>(a, grid, smem, s);
}

}  // namespace moe
