// Device-memory sharing between the processes of one node (CUDA IPC), so that each rank
// of the expert-parallel layer can address its peers' receive buffers, outputs and home
// weights directly: the pointer tables of the moe_ep_* calls.  Host code only.
//
// A buffer handed out by a caching allocator usually sits inside a larger allocation; the
// handle names the whole allocation (its base, found with cuMemGetAddressRange), and the
// buffer's offset inside it travels next to the handle.
#include <cuda.h>
#include <string.h>

#include "common.cuh"

static_assert(sizeof(cudaIpcMemHandle_t) <= MOE_IPC_HANDLE_BYTES, "IPC handle size");

namespace {

typedef CUresult (*MemGetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

MemGetAddressRangeFn address_range_fn() {
  static MemGetAddressRangeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<MemGetAddressRangeFn>(nullptr);
    return reinterpret_cast<MemGetAddressRangeFn>(p);
  }();
  return fn;
}

}  // namespace

extern "C" {

int moe_ipc_export(const void* ptr, void* handle, int64_t* offset) {
  if (!ptr || !handle || !offset) return MOE_ERR_ARG;
  MemGetAddressRangeFn range = address_range_fn();
  if (!range) return MOE_ERR_DEVICE;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  memset(handle, 0, MOE_IPC_HANDLE_BYTES);
  memcpy(handle, &h, sizeof(h));
  *offset = (int64_t)(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return MOE_OK;
}

int moe_ipc_import(const void* handle, int64_t offset, void** ptr, void** base) {
  if (!handle || !ptr || !base || offset < 0) return MOE_ERR_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* b = nullptr;
  if (cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  *base = b;
  *ptr = static_cast<char*>(b) + offset;
  return MOE_OK;
}

int moe_ipc_close(void* base) {
  if (!base) return MOE_ERR_ARG;
  if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  return MOE_OK;
}

}  // extern "C"
