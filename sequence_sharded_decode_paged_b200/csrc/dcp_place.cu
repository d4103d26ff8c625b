// dcp_place.cu -- cache placement: scatter unsharded KV rows into the D shard pools.
//
// "vLLM长序列推理优化：DCP切分KV Cache原理与实战" §2.2/§3.2: logical block
// g = t / block_size of a request belongs to shard g % D, where it is local
// block g / D and lives in the physical page that the shard's block table
// names.  This is the cache write that precedes decoding; it is a pure copy.
//
// One warp per source row (token): the warp finds its request by binary
// search over cu_seqlens, then copies the row with 16-byte loads and stores.
// The same kernel appends new tokens (the decode step's cache write): the rows
// of request b then start at token position token_begin[b] instead of 0.
//   GQA: source row [2][Hkv][d] -> pool page [2][Hkv][bs][d], slot t % bs.
//   MLA: source row [576]       -> pool page [bs][576],        slot t % bs.
#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {

struct PlaceParams {
  const int32_t* table[kMaxShards];
  uint8_t* pool[kMaxShards];
  int pool_pages[kMaxShards];
  const uint8_t* src;
  const int64_t* cu_seqlens;
  const int32_t* token_begin;  // position of each request's first source row (nullptr: 0)
  int32_t* err;
  int layout, B, Hkv, d, bs, D, mlb;
};

__global__ void __launch_bounds__(256) place_kv_kernel(const __grid_constant__ PlaceParams p) {
  const long total = p.cu_seqlens[p.B];
  const int lane = threadIdx.x & 31;
  const long warps = (long)gridDim.x * (blockDim.x >> 5);
  const int row_bytes = p.layout == DCP_LAYOUT_GQA ? 2 * p.Hkv * p.d * 2 : p.d * 2;
  const int row_vecs = row_bytes / 16;
  for (long r = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < total; r += warps) {
    // request b with cu_seqlens[b] <= r < cu_seqlens[b+1]
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cu_seqlens[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const long t = r - p.cu_seqlens[b] + (p.token_begin != nullptr ? p.token_begin[b] : 0);
    if (t < 0) {  // a negative start position names no slot
      if (lane == 0 && p.err != nullptr) atomicOr(p.err, kDevBadPage);
      continue;
    }
    const long g = t / p.bs;
    const int s = (int)(g % p.D);
    const long j = g / p.D;
    const int slot = (int)(t % p.bs);
    const int page = (j < p.mlb) ? p.table[s][(size_t)b * p.mlb + j] : -1;
    if (page < 0 || page >= p.pool_pages[s]) {
      if (lane == 0 && p.err != nullptr) atomicOr(p.err, kDevBadPage);
      continue;
    }
    const uint4* srow = reinterpret_cast<const uint4*>(p.src + (size_t)r * row_bytes);
    if (p.layout == DCP_LAYOUT_GQA) {
      const int head_vecs = p.d * 2 / 16;  // 16-byte vectors per head row
      for (int v = lane; v < row_vecs; v += 32) {
        const int kvh = v / head_vecs;  // (kv, h) pair index = kv * Hkv + h
        const int w = v - kvh * head_vecs;
        const size_t dst = (((size_t)page * 2 * p.Hkv + kvh) * p.bs + slot) * (size_t)p.d * 2 + (size_t)w * 16;
        *reinterpret_cast<uint4*>(p.pool[s] + dst) = __ldg(srow + v);
      }
    } else {
      for (int v = lane; v < row_vecs; v += 32) {
        const size_t dst = ((size_t)page * p.bs + slot) * (size_t)p.d * 2 + (size_t)v * 16;
        *reinterpret_cast<uint4*>(p.pool[s] + dst) = __ldg(srow + v);
      }
    }
  }
}

dcp_status launch_place_kv(const dcp_attn_desc& d, int D, const void* kv_src, const int64_t* cu_seqlens,
                           const int32_t* token_begin, const int32_t* const* tables, void* const* pools,
                           const int32_t* pool_pages, int32_t* device_error, cudaStream_t st) {
  PlaceParams p;
  memset(&p, 0, sizeof(p));
  for (int s = 0; s < D; ++s) {
    p.table[s] = tables[s];
    p.pool[s] = static_cast<uint8_t*>(pools[s]);
    p.pool_pages[s] = pool_pages[s];
  }
  p.src = static_cast<const uint8_t*>(kv_src);
  p.cu_seqlens = cu_seqlens;
  p.token_begin = token_begin;
  p.err = device_error;
  p.layout = d.layout;
  p.B = d.batch;
  p.Hkv = d.layout == DCP_LAYOUT_GQA ? d.num_kv_heads : 1;
  p.d = d.head_dim_qk;
  p.bs = d.block_size;
  p.D = D;
  p.mlb = d.max_local_blocks;
  const int blocks = device_sm_count() * 8;
  place_kv_kernel<<<blocks, 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

}  // namespace dcp
