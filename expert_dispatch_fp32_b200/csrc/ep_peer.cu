// Expert-parallel exchange over peer memory: the two all-to-all steps of the layer
// written as stores into the other ranks' buffers.
//
// "Expert Parallel (EP)", Communication Pattern: rank r owns experts
// [r*El, (r+1)*El); step 2 sends every dispatched row to the rank owning its expert
// (token pre-all-to-all), step 3 runs the local experts, step 4 sends the output
// rows back (token post-all-to-all).  "Worked Example: Tracing a Token Through
// Expert Parallelism", Step 2: the entry for expert 11 goes to device 2 tagged with
// its local expert 11 mod 4 = 3; Step 4: the outputs come back to the token's device.
//
// Every rank's buffers are reachable from every rank through tables of device
// pointers (moe_ep_peers): on a multi-GPU node the entries are peer mappings of
// the other GPUs' memory (NVLink / NVSwitch), with several ranks on one GPU they are
// buffers of that GPU.  A call covers the ranks [rank0, rank0 + nlocal) that run on
// the calling device (nlocal = 1 with one rank per GPU).
//
//   send_counts   each rank writes its per-expert counts [E] into row r of every
//                 rank's count matrix [P, E], then raises its count flag there;
//   send_rows     after every rank's counts have arrived, each rank knows where its
//                 rows go: in destination d, local expert l's rows are those of
//                 source 0, then source 1, ... (token order inside a source), so a
//                 row (t, j) of expert e = d*El + l lands at
//                   sum_{l' < l} sum_s cnt[s][d*El + l'] + sum_{s < r} cnt[s][e]
//                   + (pos[t*k + j] - expert_offsets[e]);
//                 one block per token reads x[t] once and stores its k copies (16-byte
//                 stores into the destinations' memory), with the sender's row and
//                 rank beside each; the last block of a rank raises its row flags;
//   recv_layout   after every sender's row flag: the rank's local expert offsets
//                 (the grouped FFN then runs on the received rows as they lie);
//   return_rows   each received output row goes back to its sender's y_back at the
//                 sender's dispatch row; the last block raises the return flags;
//   wait_returned until every destination has returned this rank's rows; then the
//                 ordinary combine reads y_back exactly as it reads y_perm on one GPU.
// Flags hold the exchange's epoch (a number the caller increases per forward), so
// nothing is reset between forwards; stores to other ranks are ordered before a flag
// by a system-scope fence and the flag itself is a release store, read with an
// acquire load.  Every wait is bounded (~1 s of SM cycles) and reports
// MOE_ERR_TIMEOUT in the status word instead of hanging.  No TMA and no multicast:
// plain 16-byte stores, so the same code runs on one GPU and across GPUs.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr long long kPeerWaitCycles = 2000000000ll;   // ~1 s at 2 GHz
constexpr int kPeerThreads = 256;

// Row stride of the stacked per-rank int32 arguments: n rounded up to 4 (16 bytes),
// so that every rank's row starts 16-byte aligned, as the single-rank calls require.
__host__ __device__ constexpr int ep_stride(int n) { return (n + 3) & ~3; }

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One thread: bounded wait until flags[i] == epoch for every i < n.
__device__ bool wait_epoch(const uint32_t* flags, int n, uint32_t epoch, int32_t* status) {
  const long long t0 = clock64();
  for (int i = 0; i < n; ++i) {
    while (ld_acquire_sys(flags + i) != epoch) {
      if (clock64() - t0 > kPeerWaitCycles) {
        if (status != nullptr) atomicCAS(status, 0, (int32_t)MOE_ERR_TIMEOUT);
        return false;
      }
      __nanosleep(100);
    }
  }
  return true;
}

// Block-wide: every thread's earlier stores are visible system-wide before thread 0
// goes on (the caller then raises flags from thread 0).
__device__ __forceinline__ void block_release_point() {
  __threadfence_system();
  __syncthreads();
}

// The last of a rank's blocks to finish raises flags[d][slot * P + r] for every rank
// d; the completion counter is left at zero for the next exchange.
__device__ void last_block_signal(int32_t* done, uint32_t* const* flags, int P, int slot, int r,
                                  uint32_t epoch) {
  block_release_point();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(done, 1);
    if (prev == (int)gridDim.x - 1) {
      __threadfence_system();
      atomicExch(done, 0);
      for (int d = 0; d < P; ++d) st_release_sys(flags[d] + slot * P + r, epoch);
    }
  }
}

__global__ void __launch_bounds__(kPeerThreads)
ep_send_counts_kernel(int32_t* const* cnt, uint32_t* const* flags, const int32_t* __restrict__ counts,
                      int rank0, int P, int E, uint32_t epoch) {
  const int r = rank0 + (int)blockIdx.x;
  const int32_t* c = counts + (size_t)blockIdx.x * ep_stride(E);
  for (int d = 0; d < P; ++d)
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[d][(size_t)r * E + e] = __ldg(c + e);
  block_release_point();
  if (threadIdx.x == 0)
    for (int d = 0; d < P; ++d) st_release_sys(flags[d] + r, epoch);
}

// Shared memory of send_rows: base[E] (first destination row of this rank's rows of
// each expert), then the current token's k destinations.
template <typename XT>
__global__ void __launch_bounds__(1024)
ep_send_rows_kernel(int32_t* const* cnt, uint32_t* const* flags, void* const* recv_x,
                    int32_t* const* recv_src, int32_t* const* recv_rank, const XT* __restrict__ x,
                    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ pos,
                    const int32_t* __restrict__ expert_offsets, int32_t* done, int32_t* status,
                    int rank0, int P, int E, int T, int D, int k, int cap, uint32_t epoch) {
  extern __shared__ int ep_sm[];
  int* base = ep_sm;                      // [E]
  int* dst_row = base + E;                // [k]
  int* dst_rank = dst_row + k;            // [k]
  const int li = (int)blockIdx.y, r = rank0 + li;
  const int El = E / P;
  const XT* xr = x + (size_t)li * T * D;
  const int32_t* idx = topk_idx + (size_t)li * ep_stride(T * k);
  const int32_t* ps = pos + (size_t)li * ep_stride(T * k);
  const int32_t* eo = expert_offsets + (size_t)li * ep_stride(E + 1);

  // every rank's counts must be in this rank's matrix before the layout is known
  __shared__ int ok;
  if (threadIdx.x == 0) ok = wait_epoch(flags[r], P, epoch, status) ? 1 : 0;
  __syncthreads();
  if (!ok) return;
  const int32_t* m = cnt[r];              // [P, E], row s from rank s
  // base[e]: experts of the destination before e (all sources), then sources before r
  for (int d = threadIdx.x; d < P; d += blockDim.x) {
    int run = 0;
    for (int l = 0; l < El; ++l) {
      const int e = d * El + l;
      int tot = 0, mine = 0;
      for (int s = 0; s < P; ++s) {
        const int v = __ldcg(m + (size_t)s * E + e);
        tot += v;
        if (s < r) mine += v;
      }
      base[e] = run + mine;
      run += tot;
    }
  }
  __syncthreads();

  const int cpr = D >> 3;                 // 16-byte chunks of a bf16 row
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      const int f = t * k + threadIdx.x;
      const int e = __ldg(idx + f);
      int row = -1, d = -1;
      if (e >= 0 && e < E) {
        d = e / El;
        row = base[e] + (__ldg(ps + f) - __ldg(eo + e));
        if (row < 0 || row >= cap) {    // more rows than the buffer holds
          atomicCAS(status, 0, (int32_t)MOE_ERR_INVALID_ARG);
          row = -1;
        }
      }
      dst_row[threadIdx.x] = row;
      dst_rank[threadIdx.x] = d;
      if (row >= 0) {
        recv_src[d][row] = __ldg(ps + f);
        recv_rank[d][row] = r;
      }
    }
    __syncthreads();
    for (int ch = threadIdx.x; ch < cpr; ch += blockDim.x) {
      uint4 v;
      if constexpr (sizeof(XT) == 2) {
        v = __ldg(reinterpret_cast<const uint4*>(xr + (size_t)t * D) + ch);
      } else {
        const float4 a = __ldg(reinterpret_cast<const float4*>(xr + (size_t)t * D) + 2 * ch);
        const float4 b = __ldg(reinterpret_cast<const float4*>(xr + (size_t)t * D) + 2 * ch + 1);
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
        h[0] = __floats2bfloat162_rn(a.x, a.y);
        h[1] = __floats2bfloat162_rn(a.z, a.w);
        h[2] = __floats2bfloat162_rn(b.x, b.y);
        h[3] = __floats2bfloat162_rn(b.z, b.w);
      }
      for (int j = 0; j < k; ++j) {
        const int row = dst_row[j];
        if (row < 0) continue;
        reinterpret_cast<uint4*>(static_cast<bf16*>(recv_x[dst_rank[j]]) + (size_t)row * D)[ch] = v;
      }
    }
    __syncthreads();
  }
  last_block_signal(done + li, flags, P, 1, r, epoch);
}

__global__ void __launch_bounds__(kPeerThreads)
ep_recv_layout_kernel(const int32_t* const* cnt, uint32_t* const* flags, int32_t* __restrict__ offsets,
                      int32_t* status, int rank0, int P, int E, uint32_t epoch) {
  const int li = (int)blockIdx.x, d = rank0 + li;
  const int El = E / P;
  int32_t* off = offsets + (size_t)li * ep_stride(El + 1);
  __shared__ int ok;
  // every sender's rows (and so its counts) are in
  if (threadIdx.x == 0) ok = wait_epoch(flags[d] + P, P, epoch, status) ? 1 : 0;
  __syncthreads();
  if (!ok) return;
  if (threadIdx.x == 0) {
    const int32_t* m = cnt[d];
    int run = 0;
    for (int l = 0; l < El; ++l) {
      off[l] = run;
      for (int s = 0; s < P; ++s) run += __ldcg(m + (size_t)s * E + d * El + l);
    }
    off[El] = run;
  }
}

__global__ void __launch_bounds__(1024)
ep_return_rows_kernel(uint32_t* const* flags, const int32_t* const* recv_src,
                      const int32_t* const* recv_rank, void* const* y_back,
                      const bf16* __restrict__ y_recv, const int32_t* __restrict__ offsets,
                      int32_t* done, int rank0, int P, int E, int D, int cap, int R_src,
                      uint32_t epoch) {
  const int li = (int)blockIdx.y, d = rank0 + li;
  const int El = E / P;
  const int n = __ldg(offsets + (size_t)li * ep_stride(El + 1) + El);
  const bf16* yr = y_recv + (size_t)li * cap * D;
  const int cpr = D >> 3;
  for (int i = blockIdx.x; i < n && i < cap; i += gridDim.x) {
    const int s = recv_rank[d][i], row = recv_src[d][i];
    if (s < 0 || s >= P || row < 0 || row >= R_src) continue;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(y_back[s]) + (size_t)row * D);
    const uint4* src = reinterpret_cast<const uint4*>(yr + (size_t)i * D);
    for (int ch = threadIdx.x; ch < cpr; ch += blockDim.x) dst[ch] = __ldg(src + ch);
  }
  last_block_signal(done + li, flags, P, 2, d, epoch);
}

__global__ void ep_signal_returned_kernel(uint32_t* const* flags, int r, int P, uint32_t epoch) {
  if (threadIdx.x == 0) {
    __threadfence_system();
    for (int d = 0; d < P; ++d) st_release_sys(flags[d] + 2 * P + r, epoch);
  }
}

__global__ void ep_wait_returned_kernel(uint32_t* const* flags, int32_t* status, int rank0, int P,
                                        uint32_t epoch) {
  if (threadIdx.x == 0) wait_epoch(flags[rank0 + (int)blockIdx.x] + 2 * P, P, epoch, status);
}

int row_threads(int D) {
  const int cpr = D >> 3;
  return cpr < 1024 ? ((cpr + 31) / 32) * 32 : 1024;
}

int blocks_per_rank(int n) {
  const int cap = 4 * sm_count();
  return n < 1 ? 1 : (n < cap ? n : cap);
}

}  // namespace

cudaError_t launch_ep_send_counts(const moe_ep_peers& p, int rank0, int nlocal, const int32_t* counts,
                                  int E, uint32_t epoch, cudaStream_t s) {
  ep_send_counts_kernel<<<nlocal, kPeerThreads, 0, s>>>(p.cnt, p.flags, counts, rank0, p.P, E, epoch);
  return cudaGetLastError();
}

cudaError_t launch_ep_send_rows(const moe_config& c, const moe_ep_peers& p, int rank0, int nlocal,
                                const void* x, const int32_t* topk_idx, const int32_t* pos,
                                const int32_t* expert_offsets, int32_t* done, int32_t* status,
                                uint32_t epoch, cudaStream_t s) {
  dim3 grid(blocks_per_rank(c.T), nlocal);
  const size_t smem = (size_t)(c.E + 2 * c.top_k) * sizeof(int);
  const int th = row_threads(c.D);
  if (c.x_dtype == MOE_DT_F32)
    ep_send_rows_kernel<float><<<grid, th, smem, s>>>(
        p.cnt, p.flags, p.recv_x, p.recv_src, p.recv_rank, static_cast<const float*>(x), topk_idx, pos,
        expert_offsets, done, status, rank0, p.P, c.E, c.T, c.D, c.top_k, p.cap, epoch);
  else
    ep_send_rows_kernel<bf16><<<grid, th, smem, s>>>(
        p.cnt, p.flags, p.recv_x, p.recv_src, p.recv_rank, static_cast<const bf16*>(x), topk_idx, pos,
        expert_offsets, done, status, rank0, p.P, c.E, c.T, c.D, c.top_k, p.cap, epoch);
  return cudaGetLastError();
}

cudaError_t launch_ep_recv_layout(const moe_config& c, const moe_ep_peers& p, int rank0, int nlocal,
                                  int32_t* local_offsets, int32_t* status, uint32_t epoch,
                                  cudaStream_t s) {
  ep_recv_layout_kernel<<<nlocal, 32, 0, s>>>(p.cnt, p.flags, local_offsets, status, rank0, p.P, c.E,
                                              epoch);
  return cudaGetLastError();
}

cudaError_t launch_ep_return_rows(const moe_config& c, const moe_ep_peers& p, int rank0, int nlocal,
                                  const void* y_recv, const int32_t* local_offsets, int32_t* done,
                                  uint32_t epoch, cudaStream_t s) {
  dim3 grid(blocks_per_rank(p.cap), nlocal);
  ep_return_rows_kernel<<<grid, row_threads(c.D), 0, s>>>(
      p.flags, p.recv_src, p.recv_rank, p.y_back, static_cast<const bf16*>(y_recv), local_offsets, done,
      rank0, p.P, c.E, c.D, p.cap, c.T * c.top_k, epoch);
  return cudaGetLastError();
}

cudaError_t launch_ep_signal_returned(const moe_ep_peers& p, int r, uint32_t epoch, cudaStream_t s) {
  ep_signal_returned_kernel<<<1, 32, 0, s>>>(p.flags, r, p.P, epoch);
  return cudaGetLastError();
}

cudaError_t launch_ep_wait_returned(const moe_ep_peers& p, int rank0, int nlocal, int32_t* status,
                                    uint32_t epoch, cudaStream_t s) {
  ep_wait_returned_kernel<<<nlocal, 32, 0, s>>>(p.flags, status, rank0, p.P, epoch);
  return cudaGetLastError();
}

}  // namespace moe
