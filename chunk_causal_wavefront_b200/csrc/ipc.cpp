// Sharing a pool buffer between processes: Wave Parallelism runs one process
// per stage GPU, and a stage delivers its K/V straight into the pools of the
// stages that read them ("Wave Forcing: Towards Speed-of-Light Streaming Video
// Generation", Method section and Figure 3c; thelatestinai listing, Table 10).
// A receiver exports its pool buffer with wf_ipc_get_mem_handle; a sender maps
// it with wf_ipc_open_mem and passes the mapped pointer to wf_deliver_kv.
//
// A handle names a whole CUDA allocation, while a pool buffer may sit at an
// offset inside one (PyTorch's caching allocator carves tensors out of larger
// segments), so the export also returns the buffer's offset from the start of
// its allocation, found with cuMemGetAddressRange.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "wf_internal.h"

namespace {

PFN_cuMemGetAddressRange_v3020 get_range_fn() {
  static PFN_cuMemGetAddressRange_v3020 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
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

wf_status wf_ipc_get_mem_handle(const void *dev_ptr, wf_ipc_handle *handle, size_t *offset) {
  if (!dev_ptr || !handle || !offset) return WF_ERR_INVALID_ARG;
  auto range = get_range_fn();
  if (!range) return WF_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return WF_ERR_INVALID_ARG;   // not device memory of this context
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return WF_ERR_CUDA;
  static_assert(sizeof(h) == sizeof(handle->bytes), "IPC handle size");
  std::memcpy(handle->bytes, &h, sizeof(h));
  *offset = static_cast<size_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return WF_OK;
}

wf_status wf_ipc_open_mem(const wf_ipc_handle *handle, size_t offset, void **dev_ptr) {
  if (!handle || !dev_ptr) return WF_ERR_INVALID_ARG;
  *dev_ptr = nullptr;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle->bytes, sizeof(h));
  void *base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();   // reset the (non-sticky) last error so later launch checks pass
    return WF_ERR_CUDA;
  }
  *dev_ptr = static_cast<char *>(base) + offset;
  return WF_OK;
}

wf_status wf_ipc_close_mem(void *dev_ptr, size_t offset) {
  if (!dev_ptr) return WF_ERR_INVALID_ARG;
  void *base = static_cast<char *>(dev_ptr) - offset;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

}  // extern "C"
