// moe_preprocess_noalloc: the preprocess stage for callers that cannot allocate
// device memory.
//
// moe_preprocess needs a caller-allocated workspace for its per-block expert
// histograms.  Some callers cannot provide one: code running inside a host
// framework that owns every device allocation and hands out only the tensors it
// already has, or a latency-critical loop where a cudaMalloc (which may
// synchronise the device) is not acceptable.  This entry point takes no
// workspace and allocates nothing; its scratch is one file-scope device array of
// MOE_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds until
// the process exits.  The pages describe no such call: it exists for deployment.
//
// The kernels are the ones moe_preprocess launches; only the scratch differs.
// Every call shares the array and leaves its contents behind.  Each call zeroes
// the barrier words on its stream and writes every histogram entry before reading
// it; calls that overlap on the GPU (two streams with no ordering between them)
// race on it.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

// Scratch: two grid-barrier words, then the block histograms.
constexpr size_t kNoAllocScratchInts = MOE_NOALLOC_SCRATCH_BYTES / sizeof(int32_t);
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};   // context id the address belongs to

// Unique id of the calling thread's current context (0 if none is current yet).  Ids
// are never reused in a process, so a device reset, which destroys the context and
// reloads the library's device array when the next one is made, shows as a new id.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = []() -> GetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<GetCurrentFn>(p);
  }();
  static GetIdFn get_id = []() -> GetIdFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<GetIdFn>(p);
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, with the device current: once per device, and again only if
// the device's context has changed since (the array then lives in the new context).
cudaError_t scratch_for_current_device(int32_t** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // makes the context current if needed
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_preprocess_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                             int32_t* counts, int32_t* expert_offsets,
                                             int32_t* rank_splits, int32_t* rank_offsets,
                                             int32_t* pos, int32_t* src, int32_t* status,
                                             void* stream) {
  moe_status st = moe_validate_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  const int32_t* ptrs_small[] = {counts, expert_offsets, rank_splits, rank_offsets, status};
  for (const int32_t* p : ptrs_small)
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u)) return MOE_ERR_INVALID_ARG;
  if (c.T > 0) {
    const int32_t* ptrs_big[] = {topk_idx, pos, src};
    for (const int32_t* p : ptrs_big)
      if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u)) return MOE_ERR_INVALID_ARG;
  }
  const size_t R = (size_t)c.T * c.top_k;
  const size_t nblk = (size_t)preprocess_blocks((int64_t)R);
  // barrier words [2], block histograms [nblk * E]
  const size_t need = 2 + nblk * (size_t)c.E;
  if (need > kNoAllocScratchInts) return MOE_ERR_SCRATCH_LIMIT;
  int32_t* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned* barrier = reinterpret_cast<unsigned*>(scratch);
  int32_t* block_counts = scratch + 2;
  // The barrier words are zeroed on the stream before each launch; every histogram
  // entry is written before it is read, so nothing else needs clearing.
  const cudaError_t err = launch_preprocess(c, topk_idx, counts, expert_offsets, rank_splits,
                                            rank_offsets, pos, src, block_counts, (int)nblk,
                                            barrier, status,
                                            reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
