// Router: fp32 logits over all experts, then softmax + top-k per token.
//
// "Worked Example: Tracing a Token Through Expert Parallelism", Step 1: the gate
// scores all E experts for the token, softmax-normalises, keeps the top-k.
// "Expert Parallel (EP)", Configuration: router_dtype 'fp32'.
//
// Logits kernel (many experts): a token-tiled SIMT fp32 GEMM (x[T,D] . W_r[E,D]^T).
// W_r does not fit in shared memory for large E*D, so tiles of BM tokens x 64
// experts stream 16-wide K slices of both operands through shared memory.  Each
// thread sums a 16-term slice in fp32 and folds it into an fp64 running total, so
// the stored fp32 logit is the dot product rounded once, to within fp32 round-off
// of a 16-term partial (~1e-8 relative), far inside the 1e-5 near-tie margin.
//
// Top-k kernel: one warp per token; selection j is an exact warp argmax on
// (logit, -index), so ties go to the lower expert index; lane j keeps pick j.
//
// Few experts (E <= 32): one fused kernel, logits and top-k together (see
// route_small_kernel below).
#include <math.h>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kRouteThreads = 256;

// Raw 8-element K slice of one x row (bf16: one 16-byte load; fp32: two).
struct XSlice { uint4 a, b; };
__device__ __forceinline__ void ld_slice(const bf16* p, XSlice& s) {
  s.a = __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void ld_slice(const float* p, XSlice& s) {
  s.a = __ldg(reinterpret_cast<const uint4*>(p));
  s.b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
}
__device__ __forceinline__ void unpack_slice(const XSlice& s, float (&v)[8], const bf16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&s.a);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x; v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void unpack_slice(const XSlice& s, float (&v)[8], const float*) {
  v[0] = __uint_as_float(s.a.x); v[1] = __uint_as_float(s.a.y);
  v[2] = __uint_as_float(s.a.z); v[3] = __uint_as_float(s.a.w);
  v[4] = __uint_as_float(s.b.x); v[5] = __uint_as_float(s.b.y);
  v[6] = __uint_as_float(s.b.z); v[7] = __uint_as_float(s.b.w);
}

// Tiled router logits for many experts: BM tokens x 64 experts per block, K in
// slices of 16 double-buffered through shared memory (the next slice is fetched
// into registers while the current one is multiplied).  Thread (ty, tx) owns TM
// tokens x 4 experts; each 16-term slice is summed in fp32 and folded into fp64.
template <int BM, typename XT>
__global__ void __launch_bounds__(kRouteThreads)
route_logits_kernel(const XT* __restrict__ x, const float* __restrict__ w,
                    const float* __restrict__ bias, float* __restrict__ logits, int T, int D,
                    int E) {
  constexpr int BN = 64, BK = 16;
  constexpr int TM = BM / 16;                     // 16 x 16 threads
  constexpr int NXS = BM * BK / 8;                         // 8-element x slices per tile
  constexpr int XLOADS = (NXS + kRouteThreads - 1) / kRouteThreads;
  __shared__ __align__(16) float xs[2][BK][BM + 4];
  __shared__ __align__(16) float ws[2][BK][BN + 4];

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  // global -> register assignment: x slice i covers token xr[i], k offset xc[i]
  int xr[XLOADS], xc[XLOADS];
#pragma unroll
  for (int i = 0; i < XLOADS; ++i) {
    const int q = tid + i * kRouteThreads;
    xr[i] = q >> 1;
    xc[i] = (q & 1) * 8;
  }
  const int wr = tid >> 2, wc = (tid & 3) * 4;    // 64 experts x 16 k = 256 float4
  XSlice xv[XLOADS];
  float4 wv;

  auto fetch = [&](int k0) {
#pragma unroll
    for (int i = 0; i < XLOADS; ++i) {
      const int t = m0 + xr[i];
      if (t < T && tid + i * kRouteThreads < NXS) ld_slice(x + (size_t)t * D + k0 + xc[i], xv[i]);
      else { xv[i].a = make_uint4(0, 0, 0, 0); xv[i].b = make_uint4(0, 0, 0, 0); }
    }
    const int e = n0 + wr;
    wv = e < E ? __ldg(reinterpret_cast<const float4*>(w + (size_t)e * D + k0 + wc))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int i = 0; i < XLOADS; ++i) {
      if (tid + i * kRouteThreads >= NXS) continue;
      float v[8];
      unpack_slice(xv[i], v, x);
#pragma unroll
      for (int q = 0; q < 8; ++q) xs[buf][xc[i] + q][xr[i]] = v[q];
    }
    ws[buf][wc + 0][wr] = wv.x;
    ws[buf][wc + 1][wr] = wv.y;
    ws[buf][wc + 2][wr] = wv.z;
    ws[buf][wc + 3][wr] = wv.w;
  };

  double tot[TM][4];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tot[i][j] = 0.0;

  fetch(0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < D; k0 += BK) {
    const bool more = k0 + BK < D;
    if (more) fetch(k0 + BK);
    float acc[TM][4];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[TM];
#pragma unroll
      for (int i = 0; i < TM; i += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(&xs[buf][kk][ty * TM + i]);
        a[i] = t4.x; a[i + 1] = t4.y; a[i + 2] = t4.z; a[i + 3] = t4.w;
      }
      const float4 b = *reinterpret_cast<const float4*>(&ws[buf][kk][tx * 4]);
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        acc[i][0] = fmaf(a[i], b.x, acc[i][0]);
        acc[i][1] = fmaf(a[i], b.y, acc[i][1]);
        acc[i][2] = fmaf(a[i], b.z, acc[i][2]);
        acc[i][3] = fmaf(a[i], b.w, acc[i][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) tot[i][j] += (double)acc[i][j];
    if (more) {
      stash(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int t = m0 + ty * TM + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = n0 + tx * 4 + j;
      if (e >= E) continue;
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

// Warp argmax top-k over one logit per lane (lanes >= E hold none).
__device__ __forceinline__ void warp_topk_write(float l, int E, int k, int renorm, size_t t,
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
}

// Few experts (E <= 32): one token per lane, K split across the warps of a block.
// Lane l of warp w accumulates token t0 + l over K range w*D/W .. (w+1)*D/W, 16
// elements per step: two 16-byte loads of its own x row, and warp-uniform (all
// lanes same address, one transaction) float4 loads of W_r[e][k..k+3] from L1/L2,
// so each W_r value read serves 32 tokens.  Each 16-element step is summed in fp32
// and folded into fp64; the W warps' fp64 partials meet in shared memory and are
// added in warp order (deterministic), then the block's tokens run the warp top-k.
constexpr int kSmallWarps = 16;
constexpr int kSmallThreads = 32 * kSmallWarps;

template <int EP, typename XT>
__global__ void __launch_bounds__(kSmallThreads, 1)
route_small_kernel(const XT* __restrict__ x, const float* __restrict__ w,
                   const float* __restrict__ bias, float* __restrict__ logits_out,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int T, int D, int E,
                   int k, int renorm) {
  extern __shared__ double part[];            // [kSmallWarps][32][EP]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 32 + lane;
  const int kspan = D / kSmallWarps;          // multiple of 4 (D % 64 == 0)
  const int kb = warp * kspan, ke = kb + kspan;
  double tot[EP];
#pragma unroll
  for (int e = 0; e < EP; ++e) tot[e] = 0.0;
  const XT* xrow = x + (size_t)(t < T ? t : 0) * D;
  // 16-byte x loads need every span start on a 16-byte boundary: kspan % 16 == 0
  // (all D >= 256 that are multiples of 256); otherwise elements are read one by one.
  const bool vec = (kspan & 15) == 0;
  for (int k0 = kb; k0 < ke; k0 += 16) {
    float xv[16];
    const int n = min(16, ke - k0);           // 16, or 4/8/12 at the end of a short span
    if (t < T && vec) {
      XSlice s0, s1;
      ld_slice(xrow + k0, s0);
      ld_slice(xrow + k0 + 8, s1);
      float a[8], b[8];
      unpack_slice(s0, a, x);
      unpack_slice(s1, b, x);
#pragma unroll
      for (int q = 0; q < 8; ++q) { xv[q] = a[q]; xv[8 + q] = b[q]; }
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) xv[q] = (t < T && q < n) ? (float)xrow[k0 + q] : 0.f;
    }
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      if (e < E) {
        const float* wr = w + (size_t)e * D + k0;
        float acc = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          if (q4 * 4 < n) {
            const float4 wv = __ldg(reinterpret_cast<const float4*>(wr) + q4);
            acc = fmaf(xv[4 * q4 + 0], wv.x, acc);
            acc = fmaf(xv[4 * q4 + 1], wv.y, acc);
            acc = fmaf(xv[4 * q4 + 2], wv.z, acc);
            acc = fmaf(xv[4 * q4 + 3], wv.w, acc);
          }
        }
        tot[e] += (double)acc;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EP; ++e) part[((size_t)warp * 32 + lane) * EP + e] = tot[e];
  __syncthreads();
  // token i of the block: lane e sums expert e's partials over the warps in order
  for (int i = warp; i < 32; i += kSmallWarps) {
    const int tt = blockIdx.x * 32 + i;
    if (tt >= T) break;
    float l = -INFINITY;
    if (lane < E) {
      double sum = 0.0;
      for (int ww = 0; ww < kSmallWarps; ++ww) sum += part[((size_t)ww * 32 + i) * EP + lane];
      l = (float)sum;
      if (bias != nullptr) l = l + bias[lane];
      if (logits_out != nullptr) logits_out[(size_t)tt * E + lane] = l;
    }
    warp_topk_write(l, E, k, renorm, (size_t)tt, topk_idx, topk_w);
  }
}

template <int EP, typename XT>
cudaError_t launch_small(const moe_config& c, const XT* x, const float* w, const float* bias,
                         float* logits_out, int32_t* topk_idx, float* topk_w, cudaStream_t s) {
  const size_t smem = (size_t)kSmallWarps * 32 * EP * sizeof(double);
  auto kern = route_small_kernel<EP, XT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<(c.T + 31) / 32, kSmallThreads, smem, s>>>(x, w, bias, logits_out, topk_idx, topk_w, c.T,
                                                    c.D, c.E, c.top_k, c.renormalize);
  return cudaGetLastError();
}

template <typename XT>
cudaError_t launch_logits(const moe_config& c, const XT* x, const float* w, const float* bias,
                          float* logits, cudaStream_t s) {
  const int n_blocks = (c.E + 63) / 64;
  // 64-token tiles when 128-token tiles would leave SMs idle
  const bool small_m = (int64_t)((c.T + 127) / 128) * n_blocks < 2 * sm_count();
  if (small_m) {
    dim3 grid((c.T + 63) / 64, n_blocks);
    route_logits_kernel<64, XT><<<grid, kRouteThreads, 0, s>>>(x, w, bias, logits, c.T, c.D, c.E);
  } else {
    dim3 grid((c.T + 127) / 128, n_blocks);
    route_logits_kernel<128, XT><<<grid, kRouteThreads, 0, s>>>(x, w, bias, logits, c.T, c.D, c.E);
  }
  return cudaGetLastError();
}

template <typename XT>
cudaError_t launch_route_t(const moe_config& c, const XT* x, const float* w_router,
                           const float* bias, float* logits, bool keep_logits, int32_t* topk_idx,
                           float* topk_w, cudaStream_t s) {
  if (c.E <= 32) {
    float* lo = keep_logits ? logits : nullptr;
    if (c.E <= 8) return launch_small<8, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
    if (c.E <= 16) return launch_small<16, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
    return launch_small<32, XT>(c, x, w_router, bias, lo, topk_idx, topk_w, s);
  }
  cudaError_t err = launch_logits(c, x, w_router, bias, logits, s);
  if (err != cudaSuccess) return err;
  const int warps_per_block = 8;
  const int blocks = (c.T + warps_per_block - 1) / warps_per_block;
  route_topk_kernel<<<blocks, warps_per_block * 32, 0, s>>>(logits, topk_idx, topk_w, c.T, c.E,
                                                             c.top_k, c.renormalize);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const moe_config& c, const void* x, const float* w_router,
                         const float* bias, float* logits, bool keep_logits, int32_t* topk_idx,
                         float* topk_w, cudaStream_t s) {
  if (c.x_dtype == MOE_DT_F32)
    return launch_route_t(c, static_cast<const float*>(x), w_router, bias, logits, keep_logits,
                          topk_idx, topk_w, s);
  return launch_route_t(c, static_cast<const bf16*>(x), w_router, bias, logits, keep_logits,
                        topk_idx, topk_w, s);
}

}  // namespace moe
