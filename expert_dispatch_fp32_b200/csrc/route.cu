// Router: fp32 logits over all experts, then softmax + top-k per token.
//
// "Worked Example: Tracing a Token Through Expert Parallelism", Step 1: the gate
// scores all E experts for the token, softmax-normalises, keeps the top-k.
// "Expert Parallel (EP)", Configuration: router_dtype 'fp32'.
//
// Every router path forms each term x_d * W_r[e,d] exactly in fp64 (both operands
// convert exactly and the product needs at most 48 bits), sums the terms in fp64 and
// rounds the total once to fp32 (dot8_exact in device_util.cuh): the stored logit is
// the exact dot product's fp32 value up to the fp64 sums' rounding, whatever the
// magnitudes and cancellation in x.
//
// Logits kernel: a token-tiled SIMT GEMM (x[T,D] . W_r[E,D]^T).  W_r does not fit in
// shared memory for large E*D, so tiles of BM tokens x BN experts stream 32-wide K
// slices of both operands through shared memory; each thread keeps fp64 totals of its
// register tile.  With few tokens the K range is split across blocks (fp64 slice
// totals, added in order by a second kernel before the single rounding).
//
// Top-k kernel: one warp per token; selection j is an exact warp argmax on
// (logit, -index), so ties go to the lower expert index; lane j keeps pick j.
//
// Few experts (E <= 32 and W_r small enough for shared memory): one fused kernel.
// W_r is staged in shared memory once per block; each warp streams TW tokens of x
// with coalesced 16-byte loads (lane l holds columns 8l..8l+7 of every 256), adds
// their exact terms to an fp64 per-lane accumulator, then
// an fp64 butterfly leaves every lane with all E dot products; lane e keeps logit
// e and the warp runs the same exact argmax top-k without a logits round trip.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "device_util.cuh"

namespace moe {

namespace {

constexpr int kRouteBK = 32;
constexpr int kRouteThreads = 256;

__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  float4 t = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}
__device__ __forceinline__ void load4(const bf16* p, float (&v)[4]) {
  uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&t.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&t.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}

template <int BN, int BM, typename XT>
__global__ void __launch_bounds__(kRouteThreads)
route_logits_kernel(const XT* __restrict__ x, const float* __restrict__ w,
                    const float* __restrict__ bias, float* __restrict__ logits, int T, int D,
                    int E, int kchunk, double* __restrict__ part) {
  constexpr int BK = kRouteBK;
  constexpr int NTN = BN / 4;                 // thread columns, 4 experts each
  constexpr int NTM = kRouteThreads / NTN;    // thread rows
  constexpr int TM = BM / NTM;                // tokens per thread
  static_assert(TM >= 1 && BM % NTM == 0, "tile");
  __shared__ __align__(16) float xs[BK][BM + 4];
  __shared__ __align__(16) float ws[BK][BN + 4];

  const int tid = threadIdx.x;
  const int tx = tid % NTN, ty = tid / NTN;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;

  double tot[TM][4];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tot[i][j] = 0.0;

  // K range of this block: all of D, or slice blockIdx.z of a split launch.  The next
  // slice's global loads go to registers before the current slice's math, so their
  // latency overlaps it (the values and the arithmetic are those of a plain loop).
  const int kbeg = blockIdx.z * kchunk, kend = kbeg + kchunk;
  constexpr int XN = BM * (BK / 4), WN = BN * (BK / 4);
  constexpr int XL = (XN + kRouteThreads - 1) / kRouteThreads;
  constexpr int WL = (WN + kRouteThreads - 1) / kRouteThreads;
  float xr[XL][4], wr[WL][4];
  auto load_slice = [&](int k0) {
#pragma unroll
    for (int l = 0; l < XL; ++l) {
      const int i = tid + l * kRouteThreads;
      const int r = i / (BK / 4), c4 = (i % (BK / 4)) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) xr[l][q] = 0.f;
      if (i < XN && m0 + r < T) load4(x + (size_t)(m0 + r) * D + k0 + c4, xr[l]);
    }
#pragma unroll
    for (int l = 0; l < WL; ++l) {
      const int i = tid + l * kRouteThreads;
      const int r = i / (BK / 4), c4 = (i % (BK / 4)) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) wr[l][q] = 0.f;
      if (i < WN && n0 + r < E) load4(w + (size_t)(n0 + r) * D + k0 + c4, wr[l]);
    }
  };
  if (kbeg < kend) load_slice(kbeg);
  for (int k0 = kbeg; k0 < kend; k0 += BK) {
#pragma unroll
    for (int l = 0; l < XL; ++l) {
      const int i = tid + l * kRouteThreads;
      const int r = i / (BK / 4), c4 = (i % (BK / 4)) * 4;
      if (i < XN) {
#pragma unroll
        for (int q = 0; q < 4; ++q) xs[c4 + q][r] = xr[l][q];
      }
    }
#pragma unroll
    for (int l = 0; l < WL; ++l) {
      const int i = tid + l * kRouteThreads;
      const int r = i / (BK / 4), c4 = (i % (BK / 4)) * 4;
      if (i < WN) {
#pragma unroll
        for (int q = 0; q < 4; ++q) ws[c4 + q][r] = wr[l][q];
      }
    }
    __syncthreads();
    if (k0 + BK < kend) load_slice(k0 + BK);
    // every term exact in fp64 (see dot8_exact), summed in K order
#pragma unroll 4
    for (int kk = 0; kk < BK; ++kk) {
      double a[TM];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = (double)xs[kk][ty * TM + i];
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      const double b0 = b.x, b1 = b.y, b2 = b.z, b3 = b.w;
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        tot[i][0] = fma(a[i], b0, tot[i][0]);
        tot[i][1] = fma(a[i], b1, tot[i][1]);
        tot[i][2] = fma(a[i], b2, tot[i][2]);
        tot[i][3] = fma(a[i], b3, tot[i][3]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int t = m0 + ty * TM + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = n0 + tx * 4 + j;
      if (e >= E) continue;
      if (part != nullptr) {
        // split launch: the slice's fp64 total; route_reduce_kernel adds the slices
        part[((size_t)blockIdx.z * T + t) * E + e] = tot[i][j];
        continue;
      }
      float l = (float)tot[i][j];
      if (bias != nullptr) l = l + bias[e];
      logits[(size_t)t * E + e] = l;
    }
  }
}

__global__ void __launch_bounds__(256)
route_topk_kernel(const float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                  float* __restrict__ topk_w, int T, int E, int k, int renorm) {
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  uint32_t taken = 0;                 // bit c: element c*32+lane already chosen
  int my_idx = 0;
  float my_val = 0.f, top = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = 0; c * 32 + lane < E; ++c) {
      if ((taken >> c) & 1u) continue;
      const int e = c * 32 + lane;
      const float v = row[e];
      if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) { my_idx = bi; my_val = bv; }
    if (j == 0) top = bv;
  }
  const float num = (lane < k) ? expf(my_val - top) : 0.f;
  float den;
  if (renorm) {
    den = num;
  } else {
    den = 0.f;
    for (int e = lane; e < E; e += 32) den += expf(row[e] - top);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = my_idx;
    topk_w[(size_t)t * k + lane] = num / den;
  }
}

// Split logits launch, second step: one thread per (token, expert) adds the fp64 slice
// totals in slice order, rounds once and adds the bias, as the unsplit kernel does.
__global__ void __launch_bounds__(256)
route_reduce_kernel(const double* __restrict__ part, int nsplit, const float* __restrict__ bias,
                    float* __restrict__ logits, int T, int E) {
  const size_t n = (size_t)T * E;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    double sum = 0.0;
#pragma unroll 8
    for (int z = 0; z < nsplit; ++z) sum += __ldg(part + (size_t)z * n + i);
    float l = (float)sum;
    if (bias != nullptr) l = l + bias[i % E];
    logits[i] = l;
  }
}

constexpr int kSmallThreads = 512;

template <int EP, int TW, typename XT>
__global__ void __launch_bounds__(kSmallThreads, 1)
route_small_kernel(const XT* __restrict__ x, const float* __restrict__ w,
                   const float* __restrict__ bias, float* __restrict__ logits_out,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int T, int D, int E,
                   int k, int renorm) {
  extern __shared__ float4 w_s4[];
  const float* w_s = reinterpret_cast<const float*>(w_s4);
  const int n4 = E * D / 4;
  {
    // stage W_r with 8 independent 16-byte loads in flight per thread (a plain
    // load-store loop waits out one L2 round trip per vector)
    constexpr int U = 8;
    for (int i0 = threadIdx.x; i0 < n4; i0 += blockDim.x * U) {
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + u * (int)blockDim.x < n4) v[u] = __ldg(reinterpret_cast<const float4*>(w) + i0 + u * blockDim.x);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + u * (int)blockDim.x < n4) w_s4[i0 + u * blockDim.x] = v[u];
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int gwarp = blockIdx.x * wpb + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * wpb;
  for (int t0 = gwarp * TW; t0 < T; t0 += nwarps * TW) {
    double acc[TW][EP];
#pragma unroll
    for (int i = 0; i < TW; ++i)
#pragma unroll
      for (int e = 0; e < EP; ++e) acc[i][e] = 0.0;
    for (int d0 = lane * 8; d0 < D; d0 += 256) {
      float xv[TW][8];
#pragma unroll
      for (int i = 0; i < TW; ++i) {
        if (t0 + i < T) {
          float a[4], b[4];
          load4(x + (size_t)(t0 + i) * D + d0, a);
          load4(x + (size_t)(t0 + i) * D + d0 + 4, b);
#pragma unroll
          for (int q = 0; q < 4; ++q) { xv[i][q] = a[q]; xv[i][4 + q] = b[q]; }
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
      const int t = t0 + i;
      if (t >= T) break;
      float l = -INFINITY;
#pragma unroll
      for (int e = 0; e < EP; ++e)
        if (lane == e) l = (float)acc[i][e];
      if (lane < E && bias != nullptr) l = l + bias[lane];
      if (logits_out != nullptr && lane < E) logits_out[(size_t)t * E + lane] = l;
      warp_topk_write(l, E, k, renorm, (size_t)t, topk_idx, topk_w);
    }
  }
}

template <int EP, int TW, typename XT>
cudaError_t launch_small(const moe_config& c, const XT* x, const float* w, const float* bias,
                         float* logits_out, int32_t* topk_idx, float* topk_w, cudaStream_t s) {
  const int threads = kSmallThreads;
  const size_t smem = (size_t)c.E * c.D * sizeof(float);
  auto kern = route_small_kernel<EP, TW, XT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int warps = threads / 32;
  const int need = (c.T + warps * TW - 1) / (warps * TW);
  int occ = 1;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem);
  if (err != cudaSuccess) return err;
  const int cap = sm_count() * (occ > 0 ? occ : 1);
  kern<<<need < cap ? need : cap, threads, smem, s>>>(x, w, bias, logits_out, topk_idx, topk_w,
                                                      c.T, c.D, c.E, c.top_k, c.renormalize);
  return cudaGetLastError();
}

constexpr size_t kSmallRouterSmem = 200u << 10;

// Tile shape of the logits kernel: BN experts x BM tokens per block.
struct LogitsTiles {
  int bn, bm, m_blocks, n_blocks;
};
LogitsTiles logits_tiles(const moe_config& c) {
  LogitsTiles g;
  g.bn = c.E >= 64 ? 64 : c.E > 16 ? 32 : c.E > 8 ? 16 : 8;
  const int m_blocks128 = (c.T + 127) / 128;
  g.n_blocks = (c.E + g.bn - 1) / g.bn;
  // 64-token tiles when 128-token tiles leave SMs idle (needs >= 2 tokens per thread row)
  const bool small_m = g.bn >= 32 && (int64_t)m_blocks128 * g.n_blocks < 2 * sm_count();
  g.bm = small_m ? 64 : 128;
  g.m_blocks = (c.T + g.bm - 1) / g.bm;
  return g;
}

// With few tokens the logits kernel has too few blocks to stream W_r (and the
// tensor-core filter GEMM too few tiles: 2 for deepseek_v3's 256 x 7168 router, ~150 us
// for 32 tokens), so the K range is split over blockIdx.z: each block stores the fp64
// total of its 32-wide slices and route_reduce_kernel adds the slices in order.  Split
// count: the largest divisor of D/32 that brings the grid to ~2 blocks per SM and whose
// slice totals (nsplit * T * E doubles) fit in `cap` bytes.  Taken when every block has
// at most kSplitMaxSlices slices, or twice that with at least one block per SM, and never
// past kSplitRouteMaxFma multiply-adds (T * E * D).  Measured against the tensor-core
// router: 256 x 7168 router 42 vs 150 us for 32 tokens, 52 vs 131 for 128, 71 vs 131 for
// 256, 114 vs 143 for 512 (32 slices, 224 blocks); 64 x 2048 router 28 vs 53 us for 32
// tokens, 34 vs 53 for 256, 48 vs 53 for 512, but 77 vs 53 for 1024 (32 slices, 32 blocks).
constexpr int kSplitMaxSlices = 16;
constexpr double kSplitRouteMaxFma = 1.0e9;
int split_route_count(const moe_config& c, size_t cap) {
  // MOE_ROUTE_SPLIT=0 keeps the unsplit paths (read at each call; for comparison)
  const char* env = getenv("MOE_ROUTE_SPLIT");
  if (env && env[0] == '0') return 1;
  if (cap == 0 || (double)c.T * c.E * c.D > kSplitRouteMaxFma) return 1;
  const LogitsTiles g = logits_tiles(c);
  const int64_t blocks = (int64_t)g.m_blocks * g.n_blocks;
  const int64_t target = (2 * sm_count() + blocks - 1) / blocks;
  const int slices = c.D / kRouteBK;
  int best = 1;
  for (int d = 2; d <= slices && d <= target; ++d)
    if (slices % d == 0 && (size_t)d * c.T * c.E * sizeof(double) <= cap) best = d;
  const int per_block = slices / best;
  const bool ok = per_block <= kSplitMaxSlices ||
                  (per_block <= 2 * kSplitMaxSlices && blocks * best >= sm_count());
  return ok ? best : 1;
}

template <typename XT>
cudaError_t launch_logits(const moe_config& c, const XT* x, const float* w, const float* bias,
                          float* logits, int nsplit, double* part, cudaStream_t s) {
  const LogitsTiles g = logits_tiles(c);
  const bool small_m = g.bm == 64;
  const int kchunk = c.D / nsplit;
  if (nsplit < 2) part = nullptr;
  dim3 grid(g.m_blocks, g.n_blocks, nsplit);
#define MOE_ROUTE_ARGS x, w, bias, logits, c.T, c.D, c.E, kchunk, part
#define MOE_ROUTE_TILE(BN_)                                                                        \
  if (small_m) route_logits_kernel<BN_, 64, XT><<<grid, kRouteThreads, 0, s>>>(MOE_ROUTE_ARGS); \
  else route_logits_kernel<BN_, 128, XT><<<grid, kRouteThreads, 0, s>>>(MOE_ROUTE_ARGS);
  switch (g.bn) {
    case 64: MOE_ROUTE_TILE(64) break;
    case 32: MOE_ROUTE_TILE(32) break;
    case 16: route_logits_kernel<16, 128, XT><<<grid, kRouteThreads, 0, s>>>(MOE_ROUTE_ARGS); break;
    default: route_logits_kernel<8, 128, XT><<<grid, kRouteThreads, 0, s>>>(MOE_ROUTE_ARGS); break;
  }
#undef MOE_ROUTE_TILE
#undef MOE_ROUTE_ARGS
  return cudaGetLastError();
}

template <typename XT>
cudaError_t launch_route_t(const moe_config& c, const XT* x, const float* w_router,
                           const float* bias, float* logits, bool keep_logits, int32_t* topk_idx,
                           float* topk_w, double* part, size_t part_bytes, cudaStream_t s) {
  const size_t wbytes = (size_t)c.E * c.D * sizeof(float);
  if (c.E <= 32 && wbytes <= kSmallRouterSmem) {
    float* lo = keep_logits ? logits : nullptr;
    // Four tokens per warp read W_r from shared memory half as often as two, which pays
    // once the 64-token blocks still cover most SMs (mixtral_8x7b: 45 vs 59 us); with
    // fewer tokens the two-token form keeps more SMs busy (small_e8_d2048: 22.5 vs 28.7 us)
    if (c.E <= 8 && 4 * ((c.T + 63) / 64) >= 3 * sm_count())
      return launch_small<8, 4, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
    if (c.E <= 8) return launch_small<8, 2, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
    if (c.E <= 16) return launch_small<16, 1, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
    return launch_small<32, 1, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
  }
  const int nsplit = part != nullptr ? split_route_count(c, part_bytes) : 1;
  cudaError_t err = launch_logits(c, x, w_router, bias, logits, nsplit, part, s);
  if (err != cudaSuccess) return err;
  if (nsplit > 1) {
    const int64_t n = (int64_t)c.T * c.E;
    const int64_t rb = (n + 255) / 256, cap = 8 * (int64_t)sm_count();
    route_reduce_kernel<<<(int)(rb < cap ? rb : cap), 256, 0, s>>>(part, nsplit, bias, logits, c.T, c.E);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const int warps_per_block = 8;
  const int blocks = (c.T + warps_per_block - 1) / warps_per_block;
  route_topk_kernel<<<blocks, warps_per_block * 32, 0, s>>>(logits, topk_idx, topk_w, c.T, c.E,
                                                             c.top_k, c.renormalize);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Tensor-core router for bf16 x (filter and refine)
// ---------------------------------------------------------------------------
// 1. router_split_kernel: W_r (fp32) = hi + mid + lo with hi = bf16(W_r),
//    mid = bf16(W_r - hi), |lo| <= 2^-18 |W_r|.  hi and mid rows are packed K-major
//    for the grouped GEMM in 64-expert groups (a 256-row block holds, for experts
//    128b + [0, 64), the hi rows then the mid rows, then the same for 128b + [64,
//    128)), the layout the GEMM's paired epilogue reads; wmax[d] = max_e |W_r[e,d]|.
// 2. The grouped GEMM (dense group, EPI_PAIRSUM_F32) gives approx[t,e] = x.hi + x.mid
//    in fp32 on the tensor cores (x is bf16, so every product is exact; only the
//    fp32 accumulation and the dropped lo part differ from the exact value).
// 3. route_refine_kernel, one warp per token: with S_t = sum_d |x_d| wmax_d, every
//    approximate logit is within eps_t = coef * S_t of the exact one (coef covers
//    one fp32 rounding per MMA instruction in each of the two chains plus the lo
//    part, with a factor 2 of margin).  Experts whose approx is below the k-th
//    largest approx minus 2 eps_t cannot be in the exact top-k; the others
//    (usually k plus one or two) get an exact logit (exact fp64 terms summed in fp64,
//    as in the SIMT paths), and the top-k and weights are taken from those.
constexpr int kRouterRowBlock = 128;      // experts per 256-row (hi, mid) block
constexpr int kRefineWarps = 4;

constexpr int kSplitRows = 8;       // expert rows per thread of the W_r split
__global__ void __launch_bounds__(128)
router_split_kernel(const float* __restrict__ w, int E, int Epad, int D, bf16* __restrict__ bsplit,
                    unsigned* __restrict__ wmax_bits) {
  const int dq = blockIdx.x * blockDim.x + threadIdx.x;     // 8-column chunk
  if (dq * 8 >= D) return;
  const int d = dq * 8;
  const int e0 = blockIdx.y * kSplitRows;
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = 0.f;
  // all kSplitRows rows' loads first (in flight together), then split and store
  float4 va[kSplitRows], vb[kSplitRows];
#pragma unroll
  for (int r = 0; r < kSplitRows; ++r) {
    const int e = e0 + r;
    if (e < E) {
      va[r] = __ldg(reinterpret_cast<const float4*>(w + (size_t)e * D + d));
      vb[r] = __ldg(reinterpret_cast<const float4*>(w + (size_t)e * D + d + 4));
    } else {
      va[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      vb[r] = va[r];
    }
  }
#pragma unroll
  for (int r = 0; r < kSplitRows; ++r) {
    const int e = e0 + r;
    if (e >= Epad) break;
    const float v[8] = {va[r].x, va[r].y, va[r].z, va[r].w, vb[r].x, vb[r].y, vb[r].z, vb[r].w};
    uint4 hi, mid;
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(&hi);
    __nv_bfloat16* m = reinterpret_cast<__nv_bfloat16*>(&mid);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      h[i] = __float2bfloat16_rn(v[i]);
      m[i] = __float2bfloat16_rn(v[i] - __bfloat162float(h[i]));
      mx[i] = fmaxf(mx[i], fabsf(v[i]));
    }
    const int j = e % kRouterRowBlock;
    const size_t row_hi = (size_t)(e / kRouterRowBlock) * (2 * kRouterRowBlock) + (j / 64) * 128 + (j % 64);
    *reinterpret_cast<uint4*>(bsplit + row_hi * D + d) = hi;
    *reinterpret_cast<uint4*>(bsplit + (row_hi + 64) * D + d) = mid;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) atomicMax(wmax_bits + d + i, __float_as_uint(mx[i]));   // |w| >= 0
}

__global__ void __launch_bounds__(32 * kRefineWarps)
route_refine_kernel(const bf16* __restrict__ x, const float* __restrict__ w,
                    const float* __restrict__ bias, const float* __restrict__ approx, int ld_approx,
                    const float* __restrict__ wmax, float coef, int32_t* __restrict__ topk_idx,
                    float* __restrict__ topk_w, int T, int D, int E, int k) {
  extern __shared__ int refine_sm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * kRefineWarps + warp;
  if (t >= T) return;                          // warps are independent: no block barrier below
  int* cidx = refine_sm + (size_t)warp * 2 * E;
  float* cval = reinterpret_cast<float*>(cidx + E);
  const bf16* xr = x + (size_t)t * D;
  const float* ar = approx + (size_t)t * ld_approx;

  // a. S_t = sum_d |x_d| wmax_d
  float S = 0.f;
  for (int d0 = lane * 8; d0 < D; d0 += 256) {
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + d0));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&xv);
    const float4 m0 = __ldg(reinterpret_cast<const float4*>(wmax + d0));
    const float4 m1 = __ldg(reinterpret_cast<const float4*>(wmax + d0 + 4));
    const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      S = fmaf(fabsf(f.x), mm[2 * i], S);
      S = fmaf(fabsf(f.y), mm[2 * i + 1], S);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);

  // b. the k-th largest approximate logit (+ bias) and the candidate set
  uint32_t taken = 0;
  float vk = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = 0; c * 32 + lane < E; ++c) {
      if ((taken >> c) & 1u) continue;
      const int e = c * 32 + lane;
      const float v = ar[e] + (bias != nullptr ? bias[e] : 0.f);
      if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    vk = bv;
  }
  const float eps = coef * S * 1.01f + 1e-6f * (fabsf(vk) + 1.f);
  const float thr = vk - 2.f * eps;
  int n = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int c = 0; c * 32 < E; ++c) {
    const int e = c * 32 + lane;
    const bool is = e < E && ar[e] + (bias != nullptr ? bias[e] : 0.f) >= thr;
    const unsigned m = __ballot_sync(0xffffffffu, is);
    if (is) cidx[n + __popc(m & lt)] = e;
    n += __popc(m);
  }
  __syncwarp();

  // c. exact logits of the candidates, four at a time
  for (int i0 = 0; i0 < n; i0 += 4) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    int ce[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) ce[q] = i0 + q < n ? cidx[i0 + q] : -1;
    for (int d0 = lane * 8; d0 < D; d0 += 256) {
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + d0));
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&xv);
      float xf[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        xf[2 * i] = f.x; xf[2 * i + 1] = f.y;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (ce[q] < 0) continue;
        const float* wr = w + (size_t)ce[q] * D + d0;
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wr));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wr + 4));
        acc[q] = dot8_exact(xf, w0, w1, acc[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (ce[q] < 0) continue;
        float l = (float)acc[q];
        if (bias != nullptr) l = l + bias[ce[q]];
        cval[i0 + q] = l;
      }
    }
  }
  __syncwarp();

  // d. exact top-k among the candidates (logit descending, ties to the lower index)
  taken = 0;
  int my_idx = 0;
  float my_val = 0.f, top = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff, bs = -1;
    for (int c = 0; c * 32 + lane < n; ++c) {
      if ((taken >> c) & 1u) continue;
      const int s = c * 32 + lane;
      const float v = cval[s];
      const int e = cidx[s];
      if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; bs = s; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const int os = __shfl_xor_sync(0xffffffffu, bs, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; bs = os; }
    }
    if ((bs & 31) == lane) taken |= 1u << (bs >> 5);
    if (lane == j) { my_idx = bi; my_val = bv; }
    if (j == 0) top = bv;
  }
  // e. renormalised weights over the top-k
  const float num = (lane < k) ? expf(my_val - top) : 0.f;
  float den = num;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = my_idx;
    topk_w[(size_t)t * k + lane] = num / den;
  }
}

cudaError_t launch_route_tc(const moe_config& c, const bf16* x, const float* w, const float* bias,
                            const RouterScratch& rs, int32_t* topk_idx, float* topk_w,
                            cudaStream_t s) {
  const int Epad = (c.E + kRouterRowBlock - 1) / kRouterRowBlock * kRouterRowBlock;
  cudaError_t err = cudaMemsetAsync(rs.wmax, 0, (size_t)c.D * sizeof(float), s);
  if (err != cudaSuccess) return err;
  err = cudaMemsetAsync(rs.counter, 0, sizeof(int32_t), s);
  if (err != cudaSuccess) return err;
  dim3 sgrid((c.D / 8 + 63) / 64, (Epad + kSplitRows - 1) / kSplitRows);
  router_split_kernel<<<sgrid, 64, 0, s>>>(w, c.E, Epad, c.D, rs.bsplit,
                                            reinterpret_cast<unsigned*>(rs.wmax));
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  GemmProblem g;
  memset(&g, 0, sizeof(g));
  g.A = x; g.a_rows = c.T;
  g.B = rs.bsplit; g.G = 1;
  g.N = 2 * Epad; g.K = c.D;
  g.group_offsets = nullptr; g.dense_rows = c.T;
  g.tile_n = 256;
  g.pair = rs.pair;
  const int tm = g.pair ? 2 * kTileM : kTileM;
  g.max_tiles = ((int64_t)(c.T + tm - 1) / tm) * (2 * Epad / 256);
  g.outf = rs.approx; g.ldo = Epad;
  g.epi = EPI_PAIRSUM_F32;
  g.status = rs.status;
  g.counter = rs.counter;
  g.dep = -1;
  err = launch_grouped_gemm(g, s);
  if (err != cudaSuccess) return err;
  // every approximate logit is within coef * S_t of the exact one (see above)
  const float coef = route_filter_coef(c.D);
  const size_t smem = (size_t)kRefineWarps * 2 * c.E * sizeof(int);
  route_refine_kernel<<<(c.T + kRefineWarps - 1) / kRefineWarps, 32 * kRefineWarps, smem, s>>>(
      x, w, bias, rs.approx, Epad, rs.wmax, coef, topk_idx, topk_w, c.T, c.D, c.E, c.top_k);
  return cudaGetLastError();
}

}  // namespace

float route_filter_coef(int D) {
  // per D: one fp32 rounding (<= 2^-23 relative, doubled) of a magnitude <= S_t per
  // 16-deep MMA instruction in each of the hi and mid chains, two more for their sum,
  // plus the dropped lo part (<= 2^-18 S_t, doubled)
  return (float)(4.0 * (D / 16 + 2) * 0x1p-23 + 0x1p-17);
}

bool route_takes_filter(const moe_config& c, size_t part_bytes, bool keep_logits) {
  if (c.x_dtype != MOE_DT_BF16) return false;
  const char* env = getenv("MOE_ROUTER_TC");
  const bool tc_ok = !(env && env[0] == '0');
  const bool few = c.E <= 32 && (size_t)c.E * c.D * sizeof(float) <= kSmallRouterSmem;
  // few tokens: the split SIMT logits (exact) beat the tensor-core filter's fixed cost
  const bool split = !few && split_route_count(c, part_bytes) > 1;
  return tc_ok && !few && !split && c.renormalize && !keep_logits;
}

cudaError_t launch_route(const moe_config& c, const void* x, const float* w_router,
                         const float* bias, float* logits, bool keep_logits, int32_t* topk_idx,
                         float* topk_w, const RouterScratch& rs, cudaStream_t s) {
  if (c.x_dtype == MOE_DT_F32)
    return launch_route_t(c, static_cast<const float*>(x), w_router, bias, logits, keep_logits,
                          topk_idx, topk_w, rs.part, rs.part_bytes, s);
  // bf16 x with renormalised weights and no logits to return, too many experts for the
  // fused shared-memory router: tensor-core filter and exact refine (MOE_ROUTER_TC=0
  // selects the SIMT paths, which compute every logit exactly)
  if (route_takes_filter(c, rs.part_bytes, keep_logits) && rs.bsplit != nullptr)
    return launch_route_tc(c, static_cast<const bf16*>(x), w_router, bias, rs, topk_idx, topk_w, s);
  return launch_route_t(c, static_cast<const bf16*>(x), w_router, bias, logits, keep_logits,
                        topk_idx, topk_w, rs.part, rs.part_bytes, s);
}

}  // namespace moe
