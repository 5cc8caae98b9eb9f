// Dispatch (token pre-all-to-all) and combine (post-all-to-all + unpermute +
// routing weights + residual) as HBM-bound gather kernels.
//
// "Expert Parallel (EP)", Communication Pattern steps 2 and 4; "Worked Example:
// Tracing a Token Through Expert Parallelism", Step 2 (each chosen expert gets a
// copy of the token), Step 4 (weighted sum of the expert outputs) and Step 5
// (residual add).  On one GPU the exchange is the gather itself.
#include <string.h>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;

struct Vec8 { float v[8]; };

__device__ __forceinline__ void ld8(const bf16* p, Vec8& o) {
  uint4 t = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&t);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    o.v[2 * i] = f.x; o.v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void ld8(const float* p, Vec8& o) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  o.v[0] = a.x; o.v[1] = a.y; o.v[2] = a.z; o.v[3] = a.w;
  o.v[4] = b.x; o.v[5] = b.y; o.v[6] = b.z; o.v[7] = b.w;
}
__device__ __forceinline__ uint4 pack_bf16(const Vec8& o) {
  uint4 t;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&t);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o.v[2 * i], o.v[2 * i + 1]);
  return t;
}
__device__ __forceinline__ void st8(bf16* p, const Vec8& o) {
  *reinterpret_cast<uint4*>(p) = pack_bf16(o);
}
__device__ __forceinline__ void st8(float* p, const Vec8& o) {
  reinterpret_cast<float4*>(p)[0] = make_float4(o.v[0], o.v[1], o.v[2], o.v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(o.v[4], o.v[5], o.v[6], o.v[7]);
}

// Token pre-all-to-all as a scatter in token order.  Block b handles token t = b
// (strided by the grid) and each thread one 16-byte chunk of the row: the chunk
// of x[t, :] is read once and written, as bf16, to its k destinations
// x_perm[pos[t*k + j], :] (a warp touches 512 contiguous bytes per store).  Every
// byte of x is read from HBM once and every byte of x_perm written once.
template <typename XT>
__global__ void __launch_bounds__(1024)
dispatch_kernel(const XT* __restrict__ x, const int32_t* __restrict__ pos, bf16* __restrict__ x_perm,
                int T, int D, int k, uint32_t R) {
  const int cpr = D >> 3;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const int32_t* pr = pos + (size_t)t * k;
    for (int ch = threadIdx.x; ch < cpr; ch += blockDim.x) {
      Vec8 f;
      ld8(x + (size_t)t * D + ch * 8, f);
      const uint4 v = pack_bf16(f);
      for (int j = 0; j < k; ++j) {
        const uint32_t p = (uint32_t)__ldg(pr + j);
        if (p < R) *reinterpret_cast<uint4*>(x_perm + (size_t)p * D + ch * 8) = v;   // else skipped pair
      }
    }
  }
}

// The same scatter with U token rows per block: every thread loads its chunk of all U
// rows before the first store (U loads in flight per thread instead of one).
template <int U>
__global__ void __launch_bounds__(1024)
dispatch_u_kernel(const bf16* __restrict__ x, const int32_t* __restrict__ pos, bf16* __restrict__ x_perm,
                  int T, int D, int k, uint32_t R) {
  const int cpr = D >> 3;
  for (int t0 = blockIdx.x * U; t0 < T; t0 += gridDim.x * U) {
    for (int ch = threadIdx.x; ch < cpr; ch += blockDim.x) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (t0 + u < T) v[u] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + u) * D + ch * 8));
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (t0 + u >= T) break;
        const int32_t* pr = pos + (size_t)(t0 + u) * k;
        for (int j = 0; j < k; ++j) {
          const uint32_t p = (uint32_t)__ldg(pr + j);
          if (p < R) *reinterpret_cast<uint4*>(x_perm + (size_t)p * D + ch * 8) = v[u];   // else skipped pair
        }
      }
    }
  }
}

// Token post-all-to-all + unpermute + routing weights + residual, warp per token:
// out[t] = x[t] + shared[t] + sum_j w[t,j] * y_perm[pos[t*k+j]]   (fp32 accumulate,
// slots in order j = 0..k-1).  pos and w are read once per token into lanes;
// each of the k row reads is 512 contiguous bytes per warp instruction.  Row
// indices are clamped to [0, R): pos is only undefined after the preprocess
// reported an out-of-range expert, and then the output is unspecified anyway.
template <typename XT>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const bf16* __restrict__ y_perm, const int32_t* __restrict__ pos,
               const float* __restrict__ topk_w, const XT* __restrict__ x,
               const bf16* __restrict__ shared, XT* __restrict__ out, int T, int D, int k,
               uint32_t R) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // see launch_pdl
  constexpr int U = 2;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    const uint32_t my_pos = lane < k ? min((uint32_t)__ldg(pos + (size_t)t * k + lane), R - 1) : 0u;
    const float my_w = lane < k ? __ldg(topk_w + (size_t)t * k + lane) : 0.f;
    for (int c0 = lane * 8; c0 < D; c0 += 256 * U) {
      Vec8 acc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 256;
        if (c < D) {
          ld8(x + (size_t)t * D + c, acc[u]);
          if (shared != nullptr) {
            Vec8 s;
            ld8(shared + (size_t)t * D + c, s);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[u].v[i] += s.v[i];
          }
        }
      }
      for (int j = 0; j < k; ++j) {
        const uint32_t p = __shfl_sync(0xffffffffu, my_pos, j);
        const float w = __shfl_sync(0xffffffffu, my_w, j);
        const bf16* yrow = y_perm + (size_t)p * D;
        Vec8 y[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (c0 + u * 256 < D) ld8(yrow + c0 + u * 256, y[u]);
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[u].v[i] = fmaf(w, y[u].v[i], acc[u].v[i]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + u * 256 < D) st8(out + (size_t)t * D + c0 + u * 256, acc[u]);
    }
  }
}

// Raw 8-element bf16 chunks, converted to fp32 only where they are used (half the
// registers of converting at the load, so more loads stay in flight per lane).
template <typename T> struct Raw8;
template <> struct Raw8<bf16> { uint4 a; };
__device__ __forceinline__ void ldr(const bf16* p, Raw8<bf16>& r) {
  r.a = __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void cvt(const Raw8<bf16>& r, Vec8& o) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.a);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    o.v[2 * i] = f.x; o.v[2 * i + 1] = f.y;
  }
}

// Combine with every row chunk of a step in flight: x, shared and the KC routed rows,
// U 256-column chunks each, loaded before the first multiply-add; the arithmetic and
// its order are those of combine_kernel.  Measured after an L2 flush (same bits as the
// slot-by-slot walk): mixtral_8x7b (k = 2, U = 2) 57.4 -> 45.1 us (5.96 TB/s),
// small_e8_d2048 18.4 -> 14.3 us, deepseek_v3 (k = 8, U = 1) 227 -> 205 us, zipf_skew_e64
// 111 -> 98 us; U = 4 at k = 2 (90 registers, half the resident warps) was slower than 2.
template <typename XT, int KC, int U>
__global__ void __launch_bounds__(kCombineThreads)
combine_k_kernel(const bf16* __restrict__ y_perm, const int32_t* __restrict__ pos,
                 const float* __restrict__ topk_w, const XT* __restrict__ x,
                 const bf16* __restrict__ shared, XT* __restrict__ out, int T, int D, uint32_t R) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // see launch_pdl
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    const uint32_t my_pos = lane < KC ? min((uint32_t)__ldg(pos + (size_t)t * KC + lane), R - 1) : 0u;
    const float my_w = lane < KC ? __ldg(topk_w + (size_t)t * KC + lane) : 0.f;
    uint32_t p[KC];
#pragma unroll
    for (int j = 0; j < KC; ++j) p[j] = __shfl_sync(0xffffffffu, my_pos, j);
    for (int c0 = lane * 8; c0 < D; c0 += 256 * U) {
      Raw8<XT> xr[U];
      Raw8<bf16> sr[U], yr[KC][U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 256;
        if (c < D) {
          ldr(x + (size_t)t * D + c, xr[u]);
          if (shared != nullptr) ldr(shared + (size_t)t * D + c, sr[u]);
#pragma unroll
          for (int j = 0; j < KC; ++j) ldr(y_perm + (size_t)p[j] * D + c, yr[j][u]);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (c0 + u * 256 < D) {
          Vec8 acc;
          cvt(xr[u], acc);
          if (shared != nullptr) {
            Vec8 sv;
            cvt(sr[u], sv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc.v[i] += sv.v[i];
          }
#pragma unroll
          for (int j = 0; j < KC; ++j) {
            const float w = __shfl_sync(0xffffffffu, my_w, j);
            Vec8 yv;
            cvt(yr[j][u], yv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc.v[i] = fmaf(w, yv.v[i], acc.v[i]);
          }
          st8(out + (size_t)t * D + c0 + u * 256, acc);
        }
      }
    }
  }
}

// Launch as a programmatic dependent of the previous kernel on the stream: the grid may
// be scheduled while that kernel finishes; the kernel's first instruction
// (griddepcontrol.wait) waits until it has completed and its writes are visible.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const char* pdl_env = getenv("MOE_PDL");       // MOE_PDL=0: plain stream order
  cfg.attrs = attr;
  cfg.numAttrs = (pdl_env && pdl_env[0] == '0') ? 0 : 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

int combine_grid(int T) {
  const int wpb = kCombineThreads / 32;
  const int need = (T + wpb - 1) / wpb;
  const int cap = sm_count() * 8;
  return need < cap ? (need > 0 ? need : 1) : cap;
}

// Dispatch: one block per token row (strided when T exceeds the grid limit); the
// block covers the row's D/8 chunks with up to 1024 threads.
dim3 row_block(int D) {
  const int cpr = D >> 3;
  const int th = cpr < 1024 ? ((cpr + 31) / 32) * 32 : 1024;
  return dim3(th);
}
dim3 row_grid(int T) { return dim3(T < 65535 ? (T > 0 ? T : 1) : 65535); }

}  // namespace

cudaError_t launch_dispatch(const moe_config& c, const void* x, const int32_t* pos, bf16* x_perm,
                            cudaStream_t s) {
  const uint32_t R = (uint32_t)c.T * c.top_k;
  if (c.x_dtype == MOE_DT_F32)
    dispatch_kernel<float><<<row_grid(c.T), row_block(c.D), 0, s>>>(static_cast<const float*>(x), pos,
                                                               x_perm, c.T, c.D, c.top_k, R);
  else if (c.top_k <= 4)
    // two rows per block: mixtral_8x7b (k = 2) 35.8 -> 31.8 us after an L2 flush; with
    // k = 6..8 (each load feeds 6-8 stores) one row per block measured ~1 % faster
    dispatch_u_kernel<2><<<row_grid((c.T + 1) / 2), row_block(c.D), 0, s>>>(
        static_cast<const bf16*>(x), pos, x_perm, c.T, c.D, c.top_k, R);
  else
    dispatch_kernel<bf16><<<row_grid(c.T), row_block(c.D), 0, s>>>(static_cast<const bf16*>(x), pos,
                                                              x_perm, c.T, c.D, c.top_k, R);
  return cudaGetLastError();
}

cudaError_t launch_combine(const moe_config& c, const bf16* y_perm, const int32_t* pos,
                           const float* topk_w, const void* x, const bf16* shared_out, void* out,
                           cudaStream_t s) {
  const uint32_t R = (uint32_t)c.T * c.top_k;
  // bf16 x: every row chunk of a step in flight, U chunks per row (k = 1: 4; k <= 4: 2;
  // else 1); MOE_PERMUTE_V=0 selects the slot-by-slot walk (for comparison)
  const char* env = getenv("MOE_PERMUTE_V");
  const bool hoist = !(env && env[0] == '0') && c.x_dtype == MOE_DT_BF16;
#define MOE_COMBINE_K(KC, U)                                                                       \
  if (hoist && c.top_k == KC)                                                                      \
    return launch_pdl(combine_k_kernel<bf16, KC, U>, combine_grid(c.T), kCombineThreads, s, y_perm, \
                      pos, topk_w, static_cast<const bf16*>(x), shared_out,                         \
                      static_cast<bf16*>(out), c.T, c.D, R);
  MOE_COMBINE_K(1, 4)
  MOE_COMBINE_K(2, 2)
  MOE_COMBINE_K(3, 2)
  MOE_COMBINE_K(4, 2)
  MOE_COMBINE_K(5, 1)
  MOE_COMBINE_K(6, 1)
  MOE_COMBINE_K(7, 1)
  MOE_COMBINE_K(8, 1)
#undef MOE_COMBINE_K
  if (c.x_dtype == MOE_DT_F32)
    return launch_pdl(combine_kernel<float>, combine_grid(c.T), kCombineThreads, s, y_perm, pos,
                      topk_w, static_cast<const float*>(x), shared_out, static_cast<float*>(out),
                      c.T, c.D, c.top_k, R);
  return launch_pdl(combine_kernel<bf16>, combine_grid(c.T), kCombineThreads, s, y_perm, pos, topk_w,
                    static_cast<const bf16*>(x), shared_out, static_cast<bf16*>(out), c.T, c.D,
                    c.top_k, R);
}

}  // namespace moe
