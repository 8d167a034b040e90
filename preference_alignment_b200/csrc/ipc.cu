// Interprocess mapping of device buffers (CUDA IPC), for the data-parallel exchange fused
// into the dW GEMM: each rank exports its receive buffer, the other ranks map it into
// their own address space and store their dW rows into it directly (over NVLink peer
// memory when the ranks run on different GPUs). The buffer may sit anywhere inside an
// allocation (a caching allocator's block): the handle names the whole allocation and
// the offset says where the buffer starts in it.
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "dpo.h"
#include "internal.h"

static_assert(sizeof(dpo_ipc_handle) == sizeof(cudaIpcMemHandle_t),
              "dpo_ipc_handle must hold a cudaIpcMemHandle_t");

namespace {

// The driver's cuMemGetAddressRange (reached without linking libcuda): the allocation
// that contains a device address.
PFN_cuMemGetAddressRange_v3020 address_range_fn() {
  static PFN_cuMemGetAddressRange_v3020 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(p);
  });
  return fn;
}

}  // namespace

extern "C" {

dpo_status dpo_ipc_export(const void* ptr, dpo_ipc_handle* handle, size_t* offset) {
  if (ptr == nullptr || handle == nullptr || offset == nullptr) return DPO_ERR_INVALID_ARG;
  auto range = address_range_fn();
  if (range == nullptr) return DPO_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
    return DPO_ERR_INVALID_ARG;            // not device memory of this process
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    (void)cudaGetLastError();
    return DPO_ERR_CUDA;
  }
  memcpy(handle->bytes, &h, sizeof(h));
  *offset = static_cast<size_t>(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return DPO_OK;
}

dpo_status dpo_ipc_import(const dpo_ipc_handle* handle, void** base) {
  if (handle == nullptr || base == nullptr) return DPO_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle->bytes, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    (void)cudaGetLastError();
    return DPO_ERR_CUDA;
  }
  *base = p;
  return DPO_OK;
}

dpo_status dpo_ipc_close(void* base) {
  if (base == nullptr) return DPO_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
    (void)cudaGetLastError();
    return DPO_ERR_CUDA;
  }
  return DPO_OK;
}

}  // extern "C"
