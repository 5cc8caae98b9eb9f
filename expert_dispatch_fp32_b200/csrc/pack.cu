// One-time repack of expert weights into the K-major layout the grouped GEMMs
// read with TMA ("Expert Parallel (EP)", Requirements: tensor-style experts with
// fused gate_up_proj [E, D, 2F] and down_proj [E, F, D]).
//
// Every output is B[g][n][kk] (kk contiguous), gathered from an input laid out
// [*, rows = K, cols = N] (n contiguous), through a 64 x 64 shared-memory tile so
// both the read (along n) and the write (along kk) are coalesced.
//   GU_SWIGLU   routed gate_up -> [E, 2F, D]; output column block b (256 wide)
//               holds, for intermediate columns b*128 + [0, 64): gate then up, and
//               for b*128 + [64, 128): gate then up.  Every 128-row half of a block
//               therefore carries both factors of 64 SwiGLU outputs, so a 256-wide
//               accumulator tile (one CTA, or a CTA pair whose CTAs each hold a
//               128-row half of B) keeps each gate column beside its up column.
//   TRANSPOSE   W1 [E, D, F] -> [E, F, D];  down [E, F, D] -> [E, D, F].
//   GU_SHARED   S shared gate_up [S, D, 2Fs] -> one [2*S*Fs, D] expert whose gate
//               (and up) columns are the S experts' gates (ups) concatenated,
//               interleaved in 64-column groups like GU_SWIGLU.
//   DOWN_SHARED S shared down [S, Fs, D] -> one [D, S*Fs] expert (rows concatenated).
// Summing S SwiGLU experts equals one SwiGLU expert with the concatenated
// intermediate dim, so the shared experts run as a single GEMM pair.
#include "moe_internal.cuh"

namespace moe {

namespace {

enum PackMode { GU_SWIGLU = 0, TRANSPOSE = 1, GU_SHARED = 2, DOWN_SHARED = 3 };

// Source element index of B[g][n][kk].  N, K: output dims; P: F or Fs.
__device__ __forceinline__ size_t pack_src(int mode, int g, int n, int kk, int N, int K, int P) {
  switch (mode) {
    case GU_SWIGLU: {
      const int blk = n >> 8, w = n & 255;
      const int f = blk * 128 + (w >> 7) * 64 + (w & 63);     // intermediate column
      const int col = ((w >> 6) & 1) ? P + f : f;             // up : gate
      return ((size_t)g * K + kk) * (size_t)(2 * P) + col;
    }
    case TRANSPOSE:
      return ((size_t)g * K + kk) * (size_t)N + n;
    case GU_SHARED: {
      const int blk = n >> 8, w = n & 255;
      const int c = blk * 128 + (w >> 7) * 64 + (w & 63);   // concatenated column
      const int i = c / P;                                  // shared expert
      const int col = ((w >> 6) & 1) * P + (c - i * P);
      return ((size_t)i * K + kk) * (size_t)(2 * P) + col;
    }
    default: {                                  // DOWN_SHARED, input [S, Fs, D]
      const int i = kk / P, f = kk - i * P;
      return ((size_t)i * P + f) * (size_t)N + n;
    }
  }
}

__global__ void __launch_bounds__(256)
pack_kernel(const bf16* __restrict__ in, bf16* __restrict__ out, int mode, int N, int K, int P) {
  __shared__ bf16 tile[64][64 + 2];
  const int g = blockIdx.z;
  const int n0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;   // 64 x 4
  for (int r = ty; r < 64; r += 4)           // r: kk offset; tx: n offset (coalesced read)
    tile[r][tx] = in[pack_src(mode, g, n0 + tx, k0 + r, N, K, P)];
  __syncthreads();
  for (int r = ty; r < 64; r += 4)           // r: n offset; tx: kk offset (coalesced write)
    out[((size_t)g * N + n0 + r) * K + k0 + tx] = tile[tx][r];
}

cudaError_t pack_one(const bf16* in, bf16* out, int mode, int G, int N, int K, int P,
                     cudaStream_t s) {
  dim3 grid(N / 64, K / 64, G);
  pack_kernel<<<grid, 256, 0, s>>>(in, out, mode, N, K, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack(const moe_config& c, const bf16* w_up, const bf16* w_down,
                        const bf16* ws_up, const bf16* ws_down, uint8_t* packed, cudaStream_t s) {
  const PackLayout L = pack_layout(c);
  cudaError_t err;
  if (c.act == MOE_ACT_SWIGLU)
    err = pack_one(w_up, (bf16*)(packed + L.w_up), GU_SWIGLU, c.E, 2 * c.F, c.D, c.F, s);
  else
    err = pack_one(w_up, (bf16*)(packed + L.w_up), TRANSPOSE, c.E, c.F, c.D, c.F, s);
  if (err != cudaSuccess) return err;
  err = pack_one(w_down, (bf16*)(packed + L.w_down), TRANSPOSE, c.E, c.D, c.F, c.F, s);
  if (err != cudaSuccess || c.n_shared == 0) return err;
  const int Fc = c.n_shared * c.F_shared;
  err = pack_one(ws_up, (bf16*)(packed + L.ws_up), GU_SHARED, 1, 2 * Fc, c.D, c.F_shared, s);
  if (err != cudaSuccess) return err;
  return pack_one(ws_down, (bf16*)(packed + L.ws_down), DOWN_SHARED, 1, c.D, Fc, c.F_shared, s);
}

}  // namespace moe
