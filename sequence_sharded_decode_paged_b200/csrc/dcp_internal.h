// dcp_internal.h -- host-side interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dcp.h"

namespace dcp {

constexpr int kMaxShardsHost = 16;
constexpr int kMaxQLen = 4;  // query tokens per request (multi-token decode)

// The shards one decode launch works on: slot si computes shard shard[si].
struct ShardSet {
  int n = 0;
  int shard[kMaxShardsHost];
  const void* pool[kMaxShardsHost];
  int32_t pool_pages[kMaxShardsHost];
  const int32_t* table[kMaxShardsHost];
  float* O[kMaxShardsHost];
  float* LSE[kMaxShardsHost];
  // Output layout.  owner_heads = 0: the standard [b][j][h] rows.  Otherwise query heads are
  // owned in consecutive slices of owner_heads heads, and row (b, j, h) goes to owner
  // k = h / owner_heads at row (b * q_len + j) * owner_heads + h % owner_heads of that owner's
  // block: owner 0's O and LSE rows start at O[0] / LSE[0], owner k's (k >= 1) at owner_O[k] /
  // owner_L[k] (set only with a single shard slot; any device address this GPU can store to,
  // a peer GPU's memory included).
  int owner_heads = 0;
  float* owner_O[kMaxShardsHost] = {};
  float* owner_L[kMaxShardsHost] = {};
};

// Workspace layout shared by the decode kernels.
struct WorkspaceLayout {
  size_t status_off = 0;    // int32 status word
  size_t counters_off = 0;  // int32 [D*B][n_hg] arrival counters
  size_t slots_off = 0;     // fp32 split partials
  size_t total = 0;
  int nctas = 0;            // CTAs per head group in one launch
  int n_hg = 1;             // head groups
  int rows_per_hg = 0;      // query rows per head group
  int slot_floats = 0;      // floats per (slot, head group)
};

bool desc_supported(const dcp_attn_desc& d, int D, dcp_status* why);
bool workspace_layout(const dcp_attn_desc& d, int D, WorkspaceLayout* out);

// Device properties of the current device (cached per device ordinal).
int device_sm_count();

// cuTensorMapEncodeTiled obtained through the runtime's driver entry point.
CUresult encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t inner_elems, uint64_t rows,
                         uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, int elem_bytes = 2,
                         int swizzle_bytes = 128);  // 128: SWIZZLE_128B (rows of 128 bytes); 64: SWIZZLE_64B

dcp_status launch_gqa_decode(const dcp_attn_desc& d, int D, const ShardSet& set, const void* q,
                             const int32_t* seq_lens, void* ws, size_t ws_bytes, cudaStream_t st);
dcp_status launch_mla_decode(const dcp_attn_desc& d, int D, const ShardSet& set, const void* q,
                             const int32_t* seq_lens, void* ws, size_t ws_bytes, cudaStream_t st);
dcp_status launch_lse_merge(const float* const* O_parts, const float* const* LSE_parts, int D, int rows, int d_v,
                            float* O, float* LSE_out, cudaStream_t st);
dcp_status launch_place_kv(const dcp_attn_desc& d, int D, const void* kv_src, const int64_t* cu_seqlens,
                           const int32_t* token_begin, const int32_t* seq_lens, const int32_t* const* tables,
                           void* const* pools, const int32_t* pool_pages, int32_t* device_error, bool few_rows,
                           cudaStream_t st);

// GQA geometry helpers (shared by the workspace sizing and the launcher).
int gqa_row_tiles(int G, int q_len);
int gqa_heads_per_cta(int Hkv, int bs, int head_dim, int row_tiles, int elem_bytes);

// Bytes per cached KV element.
inline int kv_elem_bytes(const dcp_attn_desc& d) { return d.kv_dtype == DCP_KV_FP8_E4M3 ? 1 : 2; }

}  // namespace dcp
