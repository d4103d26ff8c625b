// dcp_api.cu -- the C ABI (include/dcp.h): argument checks, the host-side
// shard table builder, workspace sizing and kernel dispatch.
//
// Table rule ("vLLM长序列推理优化：DCP切分KV Cache原理与实战" §2.2, §3.2): a
// request of L tokens has nblk = ceil(L / bs) logical blocks; block g belongs
// to shard g % D as local block g / D, so shard s holds
// nloc(s) = nblk > s ? (nblk - 1 - s) / D + 1 : 0 blocks, all full except the
// request's last block when that one falls in shard s.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {

// Contiguous rule: shard s holds the blocks [chunk_begin(s), chunk_begin(s + 1)).
static int64_t chunk_begin(int64_t nblk, int D, int s) { return (int64_t)s * nblk / D; }

static int nloc_blocks(int64_t len, int bs, int D, int s, int rule = DCP_SHARD_INTERLEAVED) {
  const int64_t nblk = (len + bs - 1) / bs;
  if (rule == DCP_SHARD_CONTIGUOUS) return (int)(chunk_begin(nblk, D, s + 1) - chunk_begin(nblk, D, s));
  return nblk > s ? (int)((nblk - 1 - s) / D + 1) : 0;
}

// Tokens of a request that shard s stores: its blocks, less the unused tail of the request's last
// block when that block is the shard's.
static int64_t nloc_tokens(int64_t len, int bs, int D, int s, int rule) {
  const int64_t nblk = (len + bs - 1) / bs;
  const int n = nloc_blocks(len, bs, D, s, rule);
  if (n == 0) return 0;
  const bool has_last = rule == DCP_SHARD_CONTIGUOUS ? chunk_begin(nblk, D, s + 1) == nblk : (nblk - 1) % D == s;
  return (int64_t)n * bs - (has_last ? nblk * bs - len : 0);
}

int device_sm_count() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUresult encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t inner_elems, uint64_t rows,
                         uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, int elem_bytes,
                         int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return CUDA_ERROR_NOT_SUPPORTED;
  cuuint64_t dims[2] = {inner_elems, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

bool desc_supported(const dcp_attn_desc& d, int D, dcp_status* why) {
  *why = DCP_ERR_INVALID_ARG;
  if (D < 1 || D > kMaxShardsHost || d.batch < 1 || d.num_q_heads < 1 || d.num_kv_heads < 1 || d.block_size < 1 ||
      d.max_local_blocks < 1 || d.head_dim_qk < 1 || d.head_dim_v < 1 || !(d.softmax_scale == d.softmax_scale) ||
      d.q_len < 1)
    return false;
  if (d.kv_dtype != DCP_KV_BF16 && d.kv_dtype != DCP_KV_FP8_E4M3) return false;
  if (d.shard_rule != DCP_SHARD_INTERLEAVED && d.shard_rule != DCP_SHARD_CONTIGUOUS) return false;
  if (d.kv_dtype == DCP_KV_FP8_E4M3 &&
      !(d.k_scale > 0.f && d.k_scale < INFINITY && d.v_scale > 0.f && d.v_scale < INFINITY))
    return false;
  *why = DCP_ERR_UNSUPPORTED;
  if (d.q_len > kMaxQLen) return false;
  // MLA's latent is one tensor (key = all 576 entries, value = the first 512): one scale for both
  *why = DCP_ERR_INVALID_ARG;
  if (d.kv_dtype == DCP_KV_FP8_E4M3 && d.layout == DCP_LAYOUT_MLA && d.k_scale != d.v_scale) return false;
  *why = DCP_ERR_UNSUPPORTED;
  if (d.layout == DCP_LAYOUT_GQA) {
    if (d.head_dim_qk != d.head_dim_v || (d.head_dim_qk != 64 && d.head_dim_qk != 128)) return false;
    if (d.num_q_heads % d.num_kv_heads != 0 || d.num_q_heads / d.num_kv_heads > 16) return false;
    if (d.block_size % 16 != 0 || d.block_size > 256 || d.block_size * d.head_dim_qk > 16384) return false;
    return true;
  }
  if (d.layout == DCP_LAYOUT_MLA) {
    return d.num_q_heads == 64 && d.num_kv_heads == 1 && d.head_dim_qk == 576 && d.head_dim_v == 512 &&
           d.block_size == 64;
  }
  *why = DCP_ERR_INVALID_ARG;
  return false;
}

int mla_ctas(int q_len);

bool workspace_layout(const dcp_attn_desc& d, int D, WorkspaceLayout* L) {
  dcp_status why;
  if (!desc_supported(d, D, &why)) return false;
  const int sms = device_sm_count();
  if (d.layout == DCP_LAYOUT_GQA) {
    const int G = d.num_q_heads / d.num_kv_heads;
    const int hpc = gqa_heads_per_cta(d.num_kv_heads, d.block_size, d.head_dim_qk, gqa_row_tiles(G, d.q_len),
                                      kv_elem_bytes(d));
    L->n_hg = d.num_kv_heads / hpc;
    L->rows_per_hg = hpc * G * d.q_len;
    L->nctas = sms / L->n_hg > 0 ? sms / L->n_hg : 1;
  } else {
    L->n_hg = d.q_len;  // one group per query token (blockIdx.y)
    L->rows_per_hg = d.num_q_heads;
    L->nctas = mla_ctas(d.q_len);
  }
  L->slot_floats = (L->rows_per_hg * (d.head_dim_v + 1) + 3) & ~3;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  L->status_off = 0;
  L->counters_off = 256;
  L->slots_off = L->counters_off + up((size_t)D * d.batch * L->n_hg * sizeof(int32_t));
  L->total = L->slots_off + up((size_t)2 * L->nctas * L->n_hg * L->slot_floats * sizeof(float));
  return true;
}

__global__ void zero_words_kernel(uint32_t* p, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0u;
}

}  // namespace dcp

using namespace dcp;

extern "C" {

// 0.2.0: q_len, kv_dtype, scales and shard_rule in dcp_attn_desc; 0.3.0: FP8 pools for every layout,
// dcp_decode_partial_to_owners and the CUDA IPC helpers
int32_t dcp_version(void) { return 300; }

const char* dcp_status_string(dcp_status s) {
  switch (s) {
    case DCP_OK: return "ok";
    case DCP_ERR_INVALID_ARG: return "invalid argument";
    case DCP_ERR_UNSUPPORTED: return "unsupported shape";
    case DCP_ERR_CAPACITY: return "buffer too small";
    case DCP_ERR_CUDA: return "CUDA error";
    case DCP_ERR_DEVICE: return "device recorded an invalid page id";
  }
  return "unknown status";
}

dcp_status dcp_block_table_extent_rule(const int32_t* seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                       int32_t shard_rule, int32_t* max_local_blocks, int32_t* num_pages) {
  if (seq_lens == nullptr || max_local_blocks == nullptr || num_pages == nullptr || batch < 0 || block_size <= 0 ||
      D < 1 || D > kMaxShardsHost || (shard_rule != DCP_SHARD_INTERLEAVED && shard_rule != DCP_SHARD_CONTIGUOUS))
    return DCP_ERR_INVALID_ARG;
  int64_t mx = 0;
  std::vector<int64_t> pages(D, 0);
  for (int b = 0; b < batch; ++b) {
    if (seq_lens[b] < 0) return DCP_ERR_INVALID_ARG;
    for (int s = 0; s < D; ++s) {
      const int n = nloc_blocks(seq_lens[b], block_size, D, s, shard_rule);
      pages[s] += n;
      if (n > mx) mx = n;
    }
  }
  for (int s = 0; s < D; ++s) {
    if (pages[s] > INT32_MAX) return DCP_ERR_CAPACITY;
    num_pages[s] = (int32_t)pages[s];
  }
  *max_local_blocks = (int32_t)mx;
  return DCP_OK;
}

dcp_status dcp_block_table_extent(const int32_t* seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                  int32_t* max_local_blocks, int32_t* num_pages) {
  return dcp_block_table_extent_rule(seq_lens, batch, block_size, D, DCP_SHARD_INTERLEAVED, max_local_blocks,
                                     num_pages);
}

dcp_status dcp_build_block_table_rule(const int32_t* seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                      int32_t shard_rule, uint64_t perm_seed, int32_t max_local_blocks,
                                      int32_t* tables, int32_t* local_len) {
  if (seq_lens == nullptr || tables == nullptr || batch < 0 || block_size <= 0 || D < 1 || D > kMaxShardsHost ||
      max_local_blocks < 0 || (shard_rule != DCP_SHARD_INTERLEAVED && shard_rule != DCP_SHARD_CONTIGUOUS))
    return DCP_ERR_INVALID_ARG;
  for (int b = 0; b < batch; ++b)
    if (seq_lens[b] < 0) return DCP_ERR_INVALID_ARG;
  for (int b = 0; b < batch; ++b)
    for (int s = 0; s < D; ++s)
      if (nloc_blocks(seq_lens[b], block_size, D, s, shard_rule) > max_local_blocks) return DCP_ERR_CAPACITY;
  for (int s = 0; s < D; ++s) {
    int32_t next = 0;
    for (int b = 0; b < batch; ++b) {
      const int64_t len = seq_lens[b];
      const int n = nloc_blocks(len, block_size, D, s, shard_rule);
      int32_t* row = tables + ((size_t)s * batch + b) * max_local_blocks;
      for (int j = 0; j < max_local_blocks; ++j) row[j] = j < n ? next + j : -1;
      next += n;
      if (local_len != nullptr) local_len[(size_t)s * batch + b] = (int32_t)nloc_tokens(len, block_size, D, s, shard_rule);
    }
    if (perm_seed != 0 && next > 1) {
      std::vector<int32_t> pi(next);
      for (int32_t i = 0; i < next; ++i) pi[i] = i;
      uint64_t state = perm_seed + (uint64_t)(s + 1) * 0xD1B54A32D192ED03ull;
      for (int64_t i = next - 1; i >= 1; --i) {
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        const int64_t j = (int64_t)(z % (uint64_t)(i + 1));
        std::swap(pi[i], pi[j]);
      }
      for (int b = 0; b < batch; ++b) {
        int32_t* row = tables + ((size_t)s * batch + b) * max_local_blocks;
        for (int j = 0; j < max_local_blocks; ++j)
          if (row[j] >= 0) row[j] = pi[row[j]];
      }
    }
  }
  return DCP_OK;
}

dcp_status dcp_build_block_table(const int32_t* seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                 uint64_t perm_seed, int32_t max_local_blocks, int32_t* tables, int32_t* local_len) {
  return dcp_build_block_table_rule(seq_lens, batch, block_size, D, DCP_SHARD_INTERLEAVED, perm_seed,
                                    max_local_blocks, tables, local_len);
}

size_t dcp_kv_page_bytes(const dcp_attn_desc* desc) {
  if (desc == nullptr) return 0;
  dcp_attn_desc d = *desc;
  if (d.max_local_blocks < 1) d.max_local_blocks = 1;
  dcp_status why;
  if (!desc_supported(d, 1, &why)) return 0;
  if (d.layout == DCP_LAYOUT_GQA) return (size_t)2 * d.num_kv_heads * d.block_size * d.head_dim_qk * kv_elem_bytes(d);
  return (size_t)d.block_size * d.head_dim_qk * kv_elem_bytes(d);
}

dcp_status dcp_place_kv(const dcp_attn_desc* desc, int32_t D, const void* kv_src, const int64_t* cu_seqlens,
                        const int32_t* seq_lens, const int32_t* const* tables, void* const* kv_pools,
                        const int32_t* pool_pages, int32_t* device_error, void* stream) {
  if (desc == nullptr || kv_src == nullptr || cu_seqlens == nullptr || seq_lens == nullptr || tables == nullptr ||
      kv_pools == nullptr || pool_pages == nullptr)
    return DCP_ERR_INVALID_ARG;
  dcp_status why;
  if (!desc_supported(*desc, D, &why)) return why;
  for (int s = 0; s < D; ++s) {
    if (tables[s] == nullptr || pool_pages[s] < 0 || (pool_pages[s] > 0 && kv_pools[s] == nullptr))
      return DCP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv_pools[s]) & 15u) != 0) return DCP_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(kv_src) & 15u) != 0) return DCP_ERR_INVALID_ARG;
  return launch_place_kv(*desc, D, kv_src, cu_seqlens, nullptr, seq_lens, tables, kv_pools, pool_pages, device_error,
                         false, static_cast<cudaStream_t>(stream));
}

dcp_status dcp_grow_block_table(const int32_t* old_seq_lens, const int32_t* new_seq_lens, int32_t batch,
                                int32_t block_size, int32_t D, int32_t max_local_blocks, int32_t* tables,
                                int32_t* local_len, int32_t* next_page, const int32_t* pool_pages) {
  if (old_seq_lens == nullptr || new_seq_lens == nullptr || tables == nullptr || next_page == nullptr ||
      pool_pages == nullptr || batch < 0 || block_size <= 0 || D < 1 || D > kMaxShardsHost || max_local_blocks < 0)
    return DCP_ERR_INVALID_ARG;
  std::vector<int64_t> need(D, 0);
  for (int b = 0; b < batch; ++b) {
    if (old_seq_lens[b] < 0 || new_seq_lens[b] < old_seq_lens[b]) return DCP_ERR_INVALID_ARG;
    const int64_t g0 = (old_seq_lens[b] + block_size - 1) / block_size;  // first block without a page
    const int64_t g1 = ((int64_t)new_seq_lens[b] + block_size - 1) / block_size;
    for (int64_t g = g0; g < g1; ++g) {
      if (g / D >= max_local_blocks) return DCP_ERR_CAPACITY;
      ++need[g % D];
    }
  }
  for (int s = 0; s < D; ++s)
    if (next_page[s] < 0 || (int64_t)next_page[s] + need[s] > pool_pages[s]) return DCP_ERR_CAPACITY;
  // checks passed: apply (new blocks take their shard's next free page, requests in order)
  for (int b = 0; b < batch; ++b) {
    const int64_t old_len = old_seq_lens[b], new_len = new_seq_lens[b];
    const int64_t g0 = (old_len + block_size - 1) / block_size;
    const int64_t g1 = (new_len + block_size - 1) / block_size;
    for (int64_t g = g0; g < g1; ++g)
      tables[((size_t)(g % D) * batch + b) * max_local_blocks + g / D] = next_page[g % D]++;
    if (local_len != nullptr)
      for (int64_t g = old_len / block_size; g < g1; ++g) {
        const int64_t lo = g * block_size > old_len ? g * block_size : old_len;
        const int64_t hi = (g + 1) * block_size < new_len ? (g + 1) * block_size : new_len;
        if (hi > lo) local_len[(size_t)(g % D) * batch + b] += (int32_t)(hi - lo);
      }
  }
  return DCP_OK;
}

dcp_status dcp_append_kv(const dcp_attn_desc* desc, int32_t D, const void* kv_new, const int64_t* cu_rows,
                         const int32_t* first_pos, const int32_t* const* tables, void* const* kv_pools,
                         const int32_t* pool_pages, int32_t* device_error, void* stream) {
  if (desc == nullptr || kv_new == nullptr || cu_rows == nullptr || first_pos == nullptr || tables == nullptr ||
      kv_pools == nullptr || pool_pages == nullptr)
    return DCP_ERR_INVALID_ARG;
  dcp_status why;
  if (!desc_supported(*desc, D, &why)) return why;
  // under the contiguous rule a token's shard depends on the request's final length
  if (desc->shard_rule != DCP_SHARD_INTERLEAVED) return DCP_ERR_UNSUPPORTED;
  for (int s = 0; s < D; ++s) {
    if (tables[s] == nullptr || pool_pages[s] < 0 || (pool_pages[s] > 0 && kv_pools[s] == nullptr))
      return DCP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv_pools[s]) & 15u) != 0) return DCP_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(kv_new) & 15u) != 0) return DCP_ERR_INVALID_ARG;
  return launch_place_kv(*desc, D, kv_new, cu_rows, first_pos, nullptr, tables, kv_pools, pool_pages, device_error,
                         true, static_cast<cudaStream_t>(stream));
}

size_t dcp_decode_workspace_bytes(const dcp_attn_desc* desc, int32_t D) {
  if (desc == nullptr) return 0;
  WorkspaceLayout L;
  if (!workspace_layout(*desc, D, &L)) return 0;
  return L.total;
}

dcp_status dcp_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DCP_ERR_INVALID_ARG;
  const size_t words = workspace_bytes / 4;
  if (words == 0) return DCP_OK;
  size_t blocks = (words + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  zero_words_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t*>(workspace), words);
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

static dcp_status check_decode_args(const dcp_attn_desc* desc, int D, const void* q, const int32_t* seq_lens,
                                    void* workspace, size_t workspace_bytes) {
  if (desc == nullptr || q == nullptr || seq_lens == nullptr || workspace == nullptr) return DCP_ERR_INVALID_ARG;
  dcp_status why;
  if (!desc_supported(*desc, D, &why)) return why;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || (reinterpret_cast<uintptr_t>(q) & 15u) != 0)
    return DCP_ERR_INVALID_ARG;
  WorkspaceLayout L;
  workspace_layout(*desc, D, &L);
  if (workspace_bytes < L.total) return DCP_ERR_CAPACITY;
  return DCP_OK;
}

static dcp_status run_decode(const dcp_attn_desc* desc, int D, const ShardSet& set, const void* q,
                             const int32_t* seq_lens, void* workspace, size_t ws_bytes, void* stream) {
  for (int i = 0; i < set.n; ++i) {
    if (set.table[i] == nullptr || set.O[i] == nullptr || set.LSE[i] == nullptr || set.pool_pages[i] < 0 ||
        (set.pool_pages[i] > 0 && set.pool[i] == nullptr))
      return DCP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(set.pool[i]) & 15u) != 0 || (reinterpret_cast<uintptr_t>(set.O[i]) & 15u) != 0)
      return DCP_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (desc->layout == DCP_LAYOUT_GQA) return launch_gqa_decode(*desc, D, set, q, seq_lens, workspace, ws_bytes, st);
  return launch_mla_decode(*desc, D, set, q, seq_lens, workspace, ws_bytes, st);
}

dcp_status dcp_decode_partial(const dcp_attn_desc* desc, const void* q, const void* kv_pool, int32_t pool_pages,
                              const int32_t* table, const int32_t* seq_lens, int32_t shard, int32_t D, float* O_i,
                              float* LSE_i, void* workspace, size_t workspace_bytes, void* stream) {
  dcp_status st = check_decode_args(desc, D, q, seq_lens, workspace, workspace_bytes);
  if (st != DCP_OK) return st;
  if (shard < 0 || shard >= D) return DCP_ERR_INVALID_ARG;
  ShardSet set;
  set.n = 1;
  set.shard[0] = shard;
  set.pool[0] = kv_pool;
  set.pool_pages[0] = pool_pages;
  set.table[0] = table;
  set.O[0] = O_i;
  set.LSE[0] = LSE_i;
  return run_decode(desc, D, set, q, seq_lens, workspace, workspace_bytes, stream);
}

size_t dcp_owner_chunk_floats(const dcp_attn_desc* desc, int32_t n_owners) {
  if (desc == nullptr || n_owners < 1 || desc->num_q_heads % n_owners != 0 || desc->batch < 1 || desc->q_len < 1)
    return 0;
  const size_t rows = (size_t)desc->batch * desc->q_len * (desc->num_q_heads / n_owners);
  return rows * desc->head_dim_v + ((rows + 63) / 64) * 64;  // O rows, then LSE rows padded to 256 B
}

dcp_status dcp_decode_partial_owner_major(const dcp_attn_desc* desc, const void* q, const void* kv_pool,
                                          int32_t pool_pages, const int32_t* table, const int32_t* seq_lens,
                                          int32_t shard, int32_t D, int32_t n_owners, float* send,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  dcp_status st = check_decode_args(desc, D, q, seq_lens, workspace, workspace_bytes);
  if (st != DCP_OK) return st;
  if (shard < 0 || shard >= D || send == nullptr || n_owners > kMaxShardsHost) return DCP_ERR_INVALID_ARG;
  const size_t chunk = dcp_owner_chunk_floats(desc, n_owners);
  if (chunk == 0) return DCP_ERR_INVALID_ARG;  // n_owners must divide the query heads
  const size_t rows = (size_t)desc->batch * desc->q_len * (desc->num_q_heads / n_owners);
  ShardSet set;
  set.n = 1;
  set.shard[0] = shard;
  set.pool[0] = kv_pool;
  set.pool_pages[0] = pool_pages;
  set.table[0] = table;
  set.O[0] = send;
  set.LSE[0] = send + rows * desc->head_dim_v;
  set.owner_heads = desc->num_q_heads / n_owners;
  for (int k = 1; k < n_owners; ++k) {
    set.owner_O[k] = send + k * chunk;
    set.owner_L[k] = send + k * chunk + rows * desc->head_dim_v;
  }
  return run_decode(desc, D, set, q, seq_lens, workspace, workspace_bytes, stream);
}

dcp_status dcp_decode_partial_to_owners(const dcp_attn_desc* desc, const void* q, const void* kv_pool,
                                        int32_t pool_pages, const int32_t* table, const int32_t* seq_lens,
                                        int32_t shard, int32_t D, int32_t n_owners, float* const* owner_chunks,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  dcp_status st = check_decode_args(desc, D, q, seq_lens, workspace, workspace_bytes);
  if (st != DCP_OK) return st;
  if (shard < 0 || shard >= D || owner_chunks == nullptr || n_owners > kMaxShardsHost) return DCP_ERR_INVALID_ARG;
  const size_t chunk = dcp_owner_chunk_floats(desc, n_owners);
  if (chunk == 0) return DCP_ERR_INVALID_ARG;  // n_owners must divide the query heads
  const size_t rows = (size_t)desc->batch * desc->q_len * (desc->num_q_heads / n_owners);
  for (int k = 0; k < n_owners; ++k)
    if (owner_chunks[k] == nullptr || (reinterpret_cast<uintptr_t>(owner_chunks[k]) & 15u) != 0)
      return DCP_ERR_INVALID_ARG;
  ShardSet set;
  set.n = 1;
  set.shard[0] = shard;
  set.pool[0] = kv_pool;
  set.pool_pages[0] = pool_pages;
  set.table[0] = table;
  set.O[0] = owner_chunks[0];
  set.LSE[0] = owner_chunks[0] + rows * desc->head_dim_v;
  set.owner_heads = desc->num_q_heads / n_owners;
  for (int k = 1; k < n_owners; ++k) {
    set.owner_O[k] = owner_chunks[k];
    set.owner_L[k] = owner_chunks[k] + rows * desc->head_dim_v;
  }
  return run_decode(desc, D, set, q, seq_lens, workspace, workspace_bytes, stream);
}

dcp_status dcp_decode_partial_all(const dcp_attn_desc* desc, const void* q, const void* const* kv_pools,
                                  const int32_t* pool_pages, const int32_t* const* tables, const int32_t* seq_lens,
                                  int32_t D, float* const* O_parts, float* const* LSE_parts, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  dcp_status st = check_decode_args(desc, D, q, seq_lens, workspace, workspace_bytes);
  if (st != DCP_OK) return st;
  if (kv_pools == nullptr || pool_pages == nullptr || tables == nullptr || O_parts == nullptr || LSE_parts == nullptr)
    return DCP_ERR_INVALID_ARG;
  ShardSet set;
  set.n = D;
  for (int s = 0; s < D; ++s) {
    set.shard[s] = s;
    set.pool[s] = kv_pools[s];
    set.pool_pages[s] = pool_pages[s];
    set.table[s] = tables[s];
    set.O[s] = O_parts[s];
    set.LSE[s] = LSE_parts[s];
  }
  return run_decode(desc, D, set, q, seq_lens, workspace, workspace_bytes, stream);
}

dcp_status dcp_lse_merge(const float* const* O_parts, const float* const* LSE_parts, int32_t D, int32_t rows,
                         int32_t d_v, float* O, float* LSE_out, void* stream) {
  if (O_parts == nullptr || LSE_parts == nullptr || O == nullptr || D < 1 || D > kMaxShardsHost || rows < 0 ||
      d_v < 4 || d_v % 4 != 0)
    return DCP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(O) & 15u) != 0) return DCP_ERR_INVALID_ARG;
  for (int i = 0; i < D; ++i)
    if (O_parts[i] == nullptr || LSE_parts[i] == nullptr || (reinterpret_cast<uintptr_t>(O_parts[i]) & 15u) != 0)
      return DCP_ERR_INVALID_ARG;
  return launch_lse_merge(O_parts, LSE_parts, D, rows, d_v, O, LSE_out, static_cast<cudaStream_t>(stream));
}

dcp_status dcp_read_device_error(void* workspace, int32_t* error_out, void* stream) {
  if (workspace == nullptr || error_out == nullptr) return DCP_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DCP_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DCP_ERR_CUDA;
  zero_words_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(workspace), 1);
  if (cudaGetLastError() != cudaSuccess) return DCP_ERR_CUDA;
  *error_out = v;
  return DCP_OK;
}

dcp_status dcp_validate_config(int32_t tp, int32_t dcp, int32_t num_kv_heads, int32_t layout) {
  if (tp <= 0 || dcp <= 0) return DCP_ERR_INVALID_ARG;
  if (dcp == 1) return DCP_OK;
  if (layout == DCP_LAYOUT_MLA) return (tp >= dcp && tp % dcp == 0) ? DCP_OK : DCP_ERR_UNSUPPORTED;
  if (layout != DCP_LAYOUT_GQA || num_kv_heads <= 0) return DCP_ERR_INVALID_ARG;
  const int rep = tp / num_kv_heads;
  return (rep >= dcp && rep % dcp == 0) ? DCP_OK : DCP_ERR_UNSUPPORTED;
}

}  // extern "C"
