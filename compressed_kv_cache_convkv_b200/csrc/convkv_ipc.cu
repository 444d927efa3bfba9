// CUDA IPC helpers for the sequence-parallel form: one process per GPU maps the
// other ranks' shard buffers so the fused kernels can read and write them.
#include <cstring>

#include "../../include/convkv.h"
#include "convkv_internal.h"

namespace {

typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

AddressRangeFn get_address_range() {
  static AddressRangeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  }
  return fn;
}

}  // namespace

extern "C" {

int convkv_ipc_export(const void* dev_ptr, void* handle64, size_t* offset) {
  if (!dev_ptr || !handle64 || !offset) return CONVKV_ERR_INVALID_ARG;
  AddressRangeFn range = get_address_range();
  if (!range) return CONVKV_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return CONVKV_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return CONVKV_ERR_CUDA;
  }
  static_assert(sizeof(h) == 64, "CUDA IPC handles are 64 bytes");
  std::memcpy(handle64, &h, sizeof(h));
  *offset = static_cast<size_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return CONVKV_OK;
}

int convkv_ipc_open(const void* handle64, void** dev_ptr) {
  if (!handle64 || !dev_ptr) return CONVKV_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle64, sizeof(h));
  if (cudaIpcOpenMemHandle(dev_ptr, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    *dev_ptr = nullptr;
    return CONVKV_ERR_CUDA;
  }
  return CONVKV_OK;
}

int convkv_ipc_close(void* dev_ptr) {
  if (!dev_ptr) return CONVKV_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(dev_ptr) != cudaSuccess) {
    cudaGetLastError();
    return CONVKV_ERR_CUDA;
  }
  return CONVKV_OK;
}

}  // extern "C"
