// Mappings of another process's device buffers, for the peer-memory exchange
// (moe_ep_peers) with one process per GPU.
//
// "Expert Parallel (EP)", Communication Pattern, steps 2 and 4: each rank stores rows
// straight into the owning rank's receive buffer.  With one process per GPU those
// buffers live in another process, so each rank exports its exchange buffers once
// (a CUDA IPC handle of the allocation that holds the buffer, plus the buffer's
// offset in it), the handles travel over the process group (host bytes), and every
// rank opens the others' handles; the opened pointers fill its pointer tables.  The
// mapping is made once, before the first forward, and closed after the last; nothing
// here runs per forward.
//
// A caching allocator hands out pieces of larger device allocations, and a handle
// names a whole allocation, so export reports the buffer's offset in its allocation
// (cuMemGetAddressRange) and import adds it back.
#include <string.h>

#include "moe_internal.cuh"

namespace {

typedef CUresult (*GetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

GetAddressRangeFn address_range_fn() {
  static GetAddressRangeFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<GetAddressRangeFn>(p);
  }
  return fn;
}

}  // namespace

extern "C" {

int32_t moe_ipc_handle_bytes(void) { return (int32_t)sizeof(cudaIpcMemHandle_t); }

moe_status moe_ipc_export(const void* ptr, void* handle, uint64_t* offset) {
  if (ptr == nullptr || handle == nullptr || offset == nullptr) return MOE_ERR_INVALID_ARG;
  GetAddressRangeFn range = address_range_fn();
  if (range == nullptr) return MOE_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, (CUdeviceptr)(uintptr_t)ptr) != CUDA_SUCCESS) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, (void*)(uintptr_t)base) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  memcpy(handle, &h, sizeof(h));
  *offset = (uint64_t)((uintptr_t)ptr - (uintptr_t)base);
  return MOE_OK;
}

moe_status moe_ipc_import(const void* handle, uint64_t offset, void** ptr) {
  if (handle == nullptr || ptr == nullptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *ptr = (void*)((uintptr_t)base + offset);
  return MOE_OK;
}

moe_status moe_ipc_close(void* ptr, uint64_t offset) {
  if (ptr == nullptr) return MOE_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle((void*)((uintptr_t)ptr - offset)) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // extern "C"
