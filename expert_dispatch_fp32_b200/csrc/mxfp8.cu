// MXFP8 quantisation of bf16 rows: E4M3 elements with one E8M0 power-of-two scale per
// 32 consecutive elements along the row.
//
// torchtitan issue 5554 (shared-expert overlap) names MXFP8 routed experts as a
// training option; the format is the OCP Microscaling (MX) v1.0 "MXFP8 (E4M3)" one:
// a block's scale exponent is s = floor(log2 amax) - 8 (8: the largest E4M3 normal
// exponent), clamped to [-127, 127], -127 for an all-zero block; every element is
// v / 2^s rounded to the nearest E4M3 value, ties to even, magnitudes above 448
// clamped to 448.  v / 2^s is exact in fp32 (a power-of-two scaling of a bf16 value
// that stays in fp32's normal range), so the conversion's single rounding is the
// element's rounding and the result is the oracle's bit for bit.
//
// Layout: q [rows, K] E4M3 bytes (row-major, K-major for the tensor cores); scales
// [rows, K/32] bytes holding s + 127 (the E8M0 encoding).  One thread per 32-element
// block: four 16-byte loads, the block maximum, two 16-byte stores and one byte.
#include <cuda_fp8.h>

#include "moe_internal.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256)
mx_quant_rows_kernel(const bf16* __restrict__ x, int64_t nblocks, int kb, uint8_t* __restrict__ q,
                     uint8_t* __restrict__ scales) {
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks;
       b += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + b * 32);
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = __ldg(src + c);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[8 * c + 2 * i] = f.x;
        v[8 * c + 2 * i + 1] = f.y;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    int s = -127;
    if (amax > 0.f) {
      int e;
      frexpf(amax, &e);              // amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
      s = e - 1 - 8;
      s = s < -127 ? -127 : (s > 127 ? 127 : s);
    }
    const float inv = __int_as_float((127 - s) << 23);   // 2^-s (s <= 119 for finite input)
    uint4 out[2];
    uint8_t* ob = reinterpret_cast<uint8_t*>(out);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      ob[i] = (uint8_t)__nv_cvt_float_to_fp8(v[i] * inv, __NV_SATFINITE, __NV_E4M3);
    uint4* dst = reinterpret_cast<uint4*>(q + b * 32);
    dst[0] = out[0];
    dst[1] = out[1];
    scales[b] = (uint8_t)(s + 127);
    (void)kb;
  }
}

}  // namespace

cudaError_t launch_mx_quant_rows(const bf16* x, int64_t rows, int K, uint8_t* q, uint8_t* scales,
                                 cudaStream_t s) {
  const int64_t nblocks = rows * (K / 32);
  if (nblocks == 0) return cudaSuccess;
  int64_t grid = (nblocks + 255) / 256;
  const int64_t cap = 8 * (int64_t)sm_count();
  if (grid > cap) grid = cap;
  mx_quant_rows_kernel<<<(int)grid, 256, 0, s>>>(x, nblocks, K / 32, q, scales);
  return cudaGetLastError();
}

}  // namespace moe
