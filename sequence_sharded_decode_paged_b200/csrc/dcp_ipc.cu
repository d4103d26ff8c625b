// dcp_ipc.cu -- mapping another process's device buffer into this one (CUDA IPC), for the
// one-shard-per-GPU form whose decode kernels store each head owner's partial rows straight
// into that owner's receive buffer ("Efficient Decode Context Parallelism with vLLM for Long
// Context Workloads", A2 方法细节, step 3: the partials travel to the rank that merges them).
//
// A buffer is exported as (handle of the allocation that holds it, byte offset inside that
// allocation): allocators hand out pieces of larger allocations, and an IPC handle always
// names a whole allocation.  The importer maps the allocation (peer access enabled on demand)
// and adds the offset.  Plain device memory only: no multicast objects are involved.
#include <string.h>

#include <mutex>

#include "dcp_internal.h"

namespace dcp {

typedef CUresult (*PointerGetAttributeFn)(void*, CUpointer_attribute, CUdeviceptr);

static PointerGetAttributeFn pointer_attr_fn() {
  static std::once_flag once;
  static PointerGetAttributeFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuPointerGetAttribute", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PointerGetAttributeFn>(p);
  });
  return fn;
}

}  // namespace dcp

using namespace dcp;

extern "C" {

size_t dcp_ipc_handle_bytes(void) { return sizeof(cudaIpcMemHandle_t); }

dcp_status dcp_ipc_export(const void* device_ptr, void* handle_out, uint64_t* offset_out) {
  if (device_ptr == nullptr || handle_out == nullptr || offset_out == nullptr) return DCP_ERR_INVALID_ARG;
  PointerGetAttributeFn fn = pointer_attr_fn();
  if (fn == nullptr) return DCP_ERR_CUDA;
  CUdeviceptr base = 0;
  if (fn(&base, CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, reinterpret_cast<CUdeviceptr>(device_ptr)) != CUDA_SUCCESS)
    return DCP_ERR_INVALID_ARG;  // not device memory of this process
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();  // do not leave the failure to be reported by the next launch check
    return DCP_ERR_CUDA;
  }
  memcpy(handle_out, &h, sizeof(h));
  *offset_out = (uint64_t)(reinterpret_cast<CUdeviceptr>(device_ptr) - base);
  return DCP_OK;
}

dcp_status dcp_ipc_open(const void* handle, void** base_out) {
  if (handle == nullptr || base_out == nullptr) return DCP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return DCP_ERR_CUDA;
  }
  *base_out = p;
  return DCP_OK;
}

dcp_status dcp_ipc_close(void* base) {
  if (base == nullptr) return DCP_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
    cudaGetLastError();
    return DCP_ERR_CUDA;
  }
  return DCP_OK;
}

}  // extern "C"
