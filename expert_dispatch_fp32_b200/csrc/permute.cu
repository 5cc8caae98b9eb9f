// Dispatch (token pre-all-to-all) and combine (post-all-to-all + unpermute +
// routing weights + residual) as HBM-bound gather kernels.
//
// "Expert Parallel (EP)", Communication Pattern steps 2 and 4; "Worked Example:
// Tracing a Token Through Expert Parallelism", Step 2 (each chosen expert gets a
// copy of the token), Step 4 (weighted sum of the expert outputs) and Step 5
// (residual add).  On one GPU the exchange is the gather itself.
//
// Both kernels walk a flat index over 16-byte output vectors (8 bf16 or 8 fp32
// elements of one row), so consecutive threads touch consecutive bytes of a row;
// each thread handles kUnroll vectors with all loads issued before any store.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kUnroll = 4;
constexpr int kThreads = 256;

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

// x_perm[row, :] = bf16(x[src[row] / k, :])
template <typename XT>
__global__ void __launch_bounds__(kThreads)
dispatch_kernel(const XT* __restrict__ x, const int32_t* __restrict__ src, bf16* __restrict__ x_perm,
                uint32_t total_vec, uint32_t vec_per_row, int D, int k, int T) {
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t v0 = blockIdx.x * blockDim.x + threadIdx.x; v0 < total_vec; v0 += stride * kUnroll) {
    Vec8 buf[kUnroll];
    uint32_t row[kUnroll], col[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t v = v0 + u * stride;
      row[u] = v / vec_per_row;
      col[u] = (v - row[u] * vec_per_row) * 8;
      if (v < total_vec) {
        const uint32_t t = (uint32_t)__ldg(src + row[u]) / (uint32_t)k;
        if (t < (uint32_t)T) ld8(x + (size_t)t * D + col[u], buf[u]);
        else for (int i = 0; i < 8; ++i) buf[u].v[i] = 0.f;   // a pair the preprocess skipped
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t v = v0 + u * stride;
      if (v < total_vec) st8(x_perm + (size_t)row[u] * D + col[u], buf[u]);
    }
  }
}

// out[t] = x[t] + shared[t] + sum_j w[t,j] * y_perm[pos[t,j]]   (fp32 accumulate)
// Row indices are clamped to [0, R): pos is only undefined after the preprocess
// reported an out-of-range expert, and then the output is unspecified anyway.
template <typename XT>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const bf16* __restrict__ y_perm, const int32_t* __restrict__ pos,
               const float* __restrict__ topk_w, const XT* __restrict__ x,
               const bf16* __restrict__ shared, XT* __restrict__ out, uint32_t total_vec,
               uint32_t vec_per_row, int D, int k, uint32_t R) {
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t v = blockIdx.x * blockDim.x + threadIdx.x; v < total_vec; v += stride) {
    const uint32_t t = v / vec_per_row;
    const uint32_t col = (v - t * vec_per_row) * 8;
    Vec8 acc;
    ld8(x + (size_t)t * D + col, acc);
    if (shared != nullptr) {
      Vec8 s;
      ld8(shared + (size_t)t * D + col, s);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc.v[i] += s.v[i];
    }
    const int32_t* pt = pos + (size_t)t * k;
    const float* wt = topk_w + (size_t)t * k;
    int j = 0;
    for (; j + 2 <= k; j += 2) {               // two rows in flight per step
      const uint32_t p0 = min((uint32_t)__ldg(pt + j), R - 1), p1 = min((uint32_t)__ldg(pt + j + 1), R - 1);
      const float w0 = __ldg(wt + j), w1 = __ldg(wt + j + 1);
      Vec8 y0, y1;
      ld8(y_perm + (size_t)p0 * D + col, y0);
      ld8(y_perm + (size_t)p1 * D + col, y1);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc.v[i] = fmaf(w0, y0.v[i], acc.v[i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc.v[i] = fmaf(w1, y1.v[i], acc.v[i]);
    }
    if (j < k) {
      const uint32_t p0 = min((uint32_t)__ldg(pt + j), R - 1);
      const float w0 = __ldg(wt + j);
      Vec8 y0;
      ld8(y_perm + (size_t)p0 * D + col, y0);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc.v[i] = fmaf(w0, y0.v[i], acc.v[i]);
    }
    st8(out + (size_t)t * D + col, acc);
  }
}

int grid_for(uint32_t total_vec) {
  const int max_blocks = sm_count() * 8;
  const uint32_t need = (total_vec + kThreads - 1) / kThreads;
  return (int)(need < (uint32_t)max_blocks ? (need > 0 ? need : 1) : max_blocks);
}

}  // namespace

cudaError_t launch_dispatch(const moe_config& c, const void* x, const int32_t* src, bf16* x_perm,
                            cudaStream_t s) {
  const uint32_t vpr = c.D / 8;
  const uint32_t total = (uint32_t)c.T * c.top_k * vpr;
  const int grid = grid_for((total + kUnroll - 1) / kUnroll);
  if (c.x_dtype == MOE_DT_F32)
    dispatch_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(x), src, x_perm,
                                                     total, vpr, c.D, c.top_k, c.T);
  else
    dispatch_kernel<bf16><<<grid, kThreads, 0, s>>>(static_cast<const bf16*>(x), src, x_perm,
                                                    total, vpr, c.D, c.top_k, c.T);
  return cudaGetLastError();
}

cudaError_t launch_combine(const moe_config& c, const bf16* y_perm, const int32_t* pos,
                           const float* topk_w, const void* x, const bf16* shared_out, void* out,
                           cudaStream_t s) {
  const uint32_t vpr = c.D / 8;
  const uint32_t total = (uint32_t)c.T * vpr;
  const int grid = grid_for(total);
  if (c.x_dtype == MOE_DT_F32)
    combine_kernel<float><<<grid, kThreads, 0, s>>>(y_perm, pos, topk_w,
                                                    static_cast<const float*>(x), shared_out,
                                                    static_cast<float*>(out), total, vpr, c.D,
                                                    c.top_k, (uint32_t)c.T * c.top_k);
  else
    combine_kernel<bf16><<<grid, kThreads, 0, s>>>(y_perm, pos, topk_w, static_cast<const bf16*>(x),
                                                   shared_out, static_cast<bf16*>(out), total, vpr,
                                                   c.D, c.top_k, (uint32_t)c.T * c.top_k);
  return cudaGetLastError();
}

}  // namespace moe
