// Helpers of the multi-rank expert-parallel forward ("Expert Parallel (EP)",
// Communication Pattern steps 2-4): the row bookkeeping around the two
// all-to-all exchanges that torch.distributed performs between the stages.
//
//   moe_ep_local_ids  before the exchange: the local expert (on its destination
//                     rank) of every row of the rank-major dispatch buffer, sent
//                     along with the rows so the receiver can group them.
//   moe_gather_rows   after the local experts ran on the receiver's rows grouped
//                     by local expert: put the output rows back in received order
//                     for the return exchange.
#include "moe_internal.cuh"

namespace moe {

namespace {

// ids[row] = topk_idx.flat[src[row]] % El; rows with src outside [0, R) get -1.
__global__ void __launch_bounds__(256)
local_ids_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ src,
                 int32_t* __restrict__ ids, int R, int El) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
    const int s = __ldg(src + r);
    ids[r] = (s >= 0 && s < R) ? __ldg(topk_idx + s) % El : -1;
  }
}

// dst[i, :] = src[index[i], :] for bf16 rows of D elements (D % 8 == 0): one block
// per row (strided), one 16-byte chunk per thread.  index outside [0, n_src) leaves
// the row unwritten.
__global__ void __launch_bounds__(1024)
gather_rows_kernel(const bf16* __restrict__ src, const int32_t* __restrict__ index,
                   bf16* __restrict__ dst, int n, int n_src, int D) {
  const int cpr = D >> 3;
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int j = __ldg(index + i);
    if (j < 0 || j >= n_src) continue;
    for (int ch = threadIdx.x; ch < cpr; ch += blockDim.x)
      reinterpret_cast<uint4*>(dst + (size_t)i * D)[ch] =
          __ldg(reinterpret_cast<const uint4*>(src + (size_t)j * D) + ch);
  }
}

}  // namespace

cudaError_t launch_local_ids(const int32_t* topk_idx, const int32_t* src, int32_t* ids, int R, int El,
                             cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  const int blocks = (R + 255) / 256 < 4 * sm_count() ? (R + 255) / 256 : 4 * sm_count();
  local_ids_kernel<<<blocks, 256, 0, s>>>(topk_idx, src, ids, R, El);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const bf16* src, const int32_t* index, bf16* dst, int n, int n_src,
                               int D, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int cpr = D >> 3;
  const int th = cpr < 1024 ? ((cpr + 31) / 32) * 32 : 1024;
  gather_rows_kernel<<<n < 65535 ? n : 65535, th, 0, s>>>(src, index, dst, n, n_src, D);
  return cudaGetLastError();
}

}  // namespace moe
