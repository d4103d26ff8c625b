// dcp_noalloc.cu -- GQA all-shard partial decode for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they run a decode step: code that is handed only its input and
// output buffers (an inference-engine plugin's enqueue, an embedded runtime
// without its own device allocator), serving loops that forbid allocation
// after start-up so that memory never fragments and no step stalls on the
// allocator, and code that must not touch the allocator while other work is
// being captured.  dcp_decode_partial_all needs a caller-provided workspace;
// this variant instead uses a fixed scratch array that lives in the library
// itself, so the caller passes only inputs and outputs.
//
// The scratch is a file-scope device array of kNoAllocScratchBytes (16 MiB).
// Every GPU that loads the library holds it until the process exits.  All
// calls share it and it keeps the last call's contents, so two calls that
// overlap on the GPU (for instance on two streams) race; serialise them.
#include <mutex>

#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for each device.  In host code the
// symbol name is only a host-side stand-in, so the real address is fetched
// once per device, with that device current, and passed to the kernels.
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

dcp_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DCP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DCP_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DCP_OK;
}

__global__ void noalloc_clear_kernel(uint32_t* words, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    words[i] = 0u;
}

}  // namespace
}  // namespace dcp

using namespace dcp;

extern "C" DCP_API dcp_status dcp_decode_partial_all_noalloc(const dcp_attn_desc* desc, const void* q,
                                                            const void* const* kv_pools, const int32_t* pool_pages,
                                                            const int32_t* const* tables, const int32_t* seq_lens,
                                                            int32_t D, float* const* O_parts,
                                                            float* const* LSE_parts, void* stream) {
  if (desc == nullptr || q == nullptr || seq_lens == nullptr || kv_pools == nullptr || pool_pages == nullptr ||
      tables == nullptr || O_parts == nullptr || LSE_parts == nullptr)
    return DCP_ERR_INVALID_ARG;
  dcp_status why;
  if (!desc_supported(*desc, D, &why)) return why;
  if (desc->layout != DCP_LAYOUT_GQA) return DCP_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) != 0) return DCP_ERR_INVALID_ARG;
  WorkspaceLayout L;
  if (!workspace_layout(*desc, D, &L)) return DCP_ERR_UNSUPPORTED;
  if (L.total > kNoAllocScratchBytes) return DCP_ERR_CAPACITY;  // needs more than the fixed 16 MiB scratch
  ShardSet set;
  set.n = D;
  for (int s = 0; s < D; ++s) {
    if (tables[s] == nullptr || O_parts[s] == nullptr || LSE_parts[s] == nullptr || pool_pages[s] < 0 ||
        (pool_pages[s] > 0 && kv_pools[s] == nullptr))
      return DCP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv_pools[s]) & 15u) != 0 || (reinterpret_cast<uintptr_t>(O_parts[s]) & 15u) != 0)
      return DCP_ERR_INVALID_ARG;
    set.shard[s] = s;
    set.pool[s] = kv_pools[s];
    set.pool_pages[s] = pool_pages[s];
    set.table[s] = tables[s];
    set.O[s] = O_parts[s];
    set.LSE[s] = LSE_parts[s];
  }
  void* scratch = nullptr;
  dcp_status st = scratch_address(&scratch);
  if (st != DCP_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // The status word and the arrival counters must start at zero; the split
  // partials behind them are always written before they are read.
  const size_t zero_words = L.slots_off / 4;
  noalloc_clear_kernel<<<(unsigned)((zero_words + 255) / 256 < 1024 ? (zero_words + 255) / 256 : 1024), 256, 0, cs>>>(
      static_cast<uint32_t*>(scratch), zero_words);
  if (cudaGetLastError() != cudaSuccess) return DCP_ERR_CUDA;
  return launch_gqa_decode(*desc, D, set, q, seq_lens, scratch, kNoAllocScratchBytes, cs);
}

// Status word of the scratch (word 0, the same bits as a workspace's): read through
// the device address looked up for this device, then cleared, like dcp_read_device_error.
extern "C" DCP_API dcp_status dcp_noalloc_read_device_error(int32_t* error_out, void* stream) {
  if (error_out == nullptr) return DCP_ERR_INVALID_ARG;
  void* scratch = nullptr;
  dcp_status st = scratch_address(&scratch);
  if (st != DCP_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return DCP_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return DCP_ERR_CUDA;
  noalloc_clear_kernel<<<1, 32, 0, cs>>>(static_cast<uint32_t*>(scratch), 1);
  if (cudaGetLastError() != cudaSuccess) return DCP_ERR_CUDA;
  *error_out = v;
  return DCP_OK;
}
