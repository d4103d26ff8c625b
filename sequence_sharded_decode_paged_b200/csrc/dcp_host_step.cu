// dcp_host_step.cu -- one whole decode step fed from, and returned to, host memory.
//
// The step of "Efficient Decode Context Parallelism with vLLM for Long Context
// Workloads" (A2 方法细节: every shard attends the full query against its local
// KV slice, then the partials are merged) with its inputs and outputs on the
// host: the query, the lengths and the D block tables are copied up, the D
// shard partials and their LSE merge run on the device, and the merged output
// is copied back -- all on one stream, in one call.  The caller passes a
// device staging buffer (dcp_host_step_staging_bytes) that holds the uploaded
// inputs, the partials and the merged output; nothing is allocated here.
#include "dcp_internal.h"

namespace dcp {
namespace {

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

struct StagingLayout {
  size_t q, lens, tables, O_parts, LSE_parts, O, LSE, total;
  size_t q_bytes, lens_bytes, tables_bytes, o_bytes, lse_bytes;  // per shard for the parts
};

bool staging_layout(const dcp_attn_desc& d, int D, StagingLayout* L) {
  dcp_status why;
  if (!desc_supported(d, D, &why)) return false;
  const size_t rows = (size_t)d.batch * d.q_len * d.num_q_heads;
  L->q_bytes = rows * d.head_dim_qk * 2;
  L->lens_bytes = (size_t)d.batch * 4;
  L->tables_bytes = (size_t)D * d.batch * d.max_local_blocks * 4;
  L->o_bytes = rows * d.head_dim_v * 4;
  L->lse_bytes = rows * 4;
  size_t off = 0;
  L->q = off;
  off += align256(L->q_bytes);
  L->lens = off;
  off += align256(L->lens_bytes);
  L->tables = off;
  off += align256(L->tables_bytes);
  L->O_parts = off;
  off += (size_t)D * align256(L->o_bytes);
  L->LSE_parts = off;
  off += (size_t)D * align256(L->lse_bytes);
  L->O = off;
  off += align256(L->o_bytes);
  L->LSE = off;
  off += align256(L->lse_bytes);
  L->total = off;
  return true;
}

}  // namespace
}  // namespace dcp

using namespace dcp;

extern "C" {

size_t dcp_host_step_staging_bytes(const dcp_attn_desc* desc, int32_t D) {
  if (desc == nullptr) return 0;
  StagingLayout L;
  return staging_layout(*desc, D, &L) ? L.total : 0;
}

dcp_status dcp_decode_step_host(const dcp_attn_desc* desc, int32_t D, const void* host_q,
                                const int32_t* host_seq_lens, const int32_t* host_tables,
                                const void* const* kv_pools, const int32_t* pool_pages, void* staging,
                                size_t staging_bytes, void* workspace, size_t workspace_bytes, float* host_O,
                                float* host_LSE, void* stream) {
  if (desc == nullptr || host_q == nullptr || host_seq_lens == nullptr || host_tables == nullptr ||
      kv_pools == nullptr || pool_pages == nullptr || staging == nullptr || workspace == nullptr ||
      host_O == nullptr)
    return DCP_ERR_INVALID_ARG;
  StagingLayout L;
  if (!staging_layout(*desc, D, &L)) {
    dcp_status why;
    desc_supported(*desc, D, &why);
    return why;
  }
  if (staging_bytes < L.total) return DCP_ERR_CAPACITY;
  if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0 || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return DCP_ERR_INVALID_ARG;
  WorkspaceLayout W;
  if (!workspace_layout(*desc, D, &W)) return DCP_ERR_UNSUPPORTED;
  if (workspace_bytes < W.total) return DCP_ERR_CAPACITY;
  uint8_t* base = static_cast<uint8_t*>(staging);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ShardSet set;
  set.n = D;
  float* O_parts[kMaxShardsHost];
  float* LSE_parts[kMaxShardsHost];
  const size_t tab_row = (size_t)desc->batch * desc->max_local_blocks;
  for (int s = 0; s < D; ++s) {
    if (pool_pages[s] < 0 || (pool_pages[s] > 0 && kv_pools[s] == nullptr) ||
        (reinterpret_cast<uintptr_t>(kv_pools[s]) & 15u) != 0)
      return DCP_ERR_INVALID_ARG;
    O_parts[s] = reinterpret_cast<float*>(base + L.O_parts + s * align256(L.o_bytes));
    LSE_parts[s] = reinterpret_cast<float*>(base + L.LSE_parts + s * align256(L.lse_bytes));
    set.shard[s] = s;
    set.pool[s] = kv_pools[s];
    set.pool_pages[s] = pool_pages[s];
    set.table[s] = reinterpret_cast<const int32_t*>(base + L.tables) + s * tab_row;
    set.O[s] = O_parts[s];
    set.LSE[s] = LSE_parts[s];
  }
  // inputs up
  if (cudaMemcpyAsync(base + L.q, host_q, L.q_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(base + L.lens, host_seq_lens, L.lens_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(base + L.tables, host_tables, L.tables_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return DCP_ERR_CUDA;
  // the D shard partials in one launch, then their merge
  const int32_t* lens = reinterpret_cast<const int32_t*>(base + L.lens);
  dcp_status r = desc->layout == DCP_LAYOUT_GQA
                     ? launch_gqa_decode(*desc, D, set, base + L.q, lens, workspace, workspace_bytes, st)
                     : launch_mla_decode(*desc, D, set, base + L.q, lens, workspace, workspace_bytes, st);
  if (r != DCP_OK) return r;
  const int rows = desc->batch * desc->q_len * desc->num_q_heads;
  float* O = reinterpret_cast<float*>(base + L.O);
  float* LSE = reinterpret_cast<float*>(base + L.LSE);
  r = launch_lse_merge(O_parts, LSE_parts, D, rows, desc->head_dim_v, O, LSE, st);
  if (r != DCP_OK) return r;
  // result down
  if (cudaMemcpyAsync(host_O, O, L.o_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return DCP_ERR_CUDA;
  if (host_LSE != nullptr &&
      cudaMemcpyAsync(host_LSE, LSE, L.lse_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return DCP_ERR_CUDA;
  return DCP_OK;
}

}  // extern "C"
