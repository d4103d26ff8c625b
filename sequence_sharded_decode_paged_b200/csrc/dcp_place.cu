// dcp_place.cu -- cache placement: scatter unsharded KV rows into the D shard pools.
//
// "vLLM长序列推理优化：DCP切分KV Cache原理与实战" §2.2/§3.2: logical block
// g = t / block_size of a request belongs to shard g % D, where it is local
// block g / D and lives in the physical page that the shard's block table
// names.  This is the cache write that precedes decoding; it is a pure copy.
//
// Under the contiguous shard rule a token's shard and local block follow from
// its request's length (seq_lens): shard s holds the blocks
// [floor(s * nblk / D), floor((s + 1) * nblk / D)).
// Bulk placement (place_kv_kernel): one warp per source row (token); the warp
// finds its request by binary search over cu_seqlens, then copies the row with
// 16-byte loads and stores.
// Append (append_kv_kernel, the decode step's cache write of a few new tokens
// per request, whose rows start at token position token_begin[b]): one thread
// per 16-byte piece, so the handful of rows is spread over the whole grid and
// the copy takes one dependent chain of loads instead of one per piece.
//   GQA: source row [2][Hkv][d] -> pool page [2][Hkv][bs][d], slot t % bs.
//   MLA: source row [576]       -> pool page [bs][576],        slot t % bs.
// An FP8 pool (GQA) stores E4M3 codes: each bf16 value x becomes
// e4m3_rn_satfinite(float32(x) * inv), inv = float32(1 / k_scale) for K and
// float32(1 / v_scale) for V (one byte per value, same page layout).
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
  int eb;            // bytes per pool element: 2 (bf16) or 1 (FP8 code)
  int rule;          // shard rule: 0 interleaved, 1 contiguous chunks (needs seq_lens)
  const int32_t* seq_lens;
  float inv_k, inv_v;  // FP8: multipliers applied before rounding to E4M3
};

// Destination of source row r: its request b, and the byte offset of the row's
// slot in shard *s's pool (GQA: offset of head 0's K row).  False (and the error
// flag set once, by `report`) when the position names no page.
__device__ __forceinline__ bool row_slot(const PlaceParams& p, long r, bool report, int* s_out, size_t* base_out) {
  int lo = 0, hi = p.B - 1;  // request b with cu_seqlens[b] <= r < cu_seqlens[b+1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.cu_seqlens[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const long t = r - p.cu_seqlens[b] + (p.token_begin != nullptr ? p.token_begin[b] : 0);
  if (t < 0) {  // a negative start position names no slot
    if (report && p.err != nullptr) atomicOr(p.err, kDevBadPage);
    return false;
  }
  const long g = t / p.bs;
  int s;
  long j;
  if (p.rule == 0) {
    s = (int)(g % p.D);
    j = g / p.D;
  } else {  // the chunk of the request's blocks that holds g
    const int nblk = (p.seq_lens[b] + p.bs - 1) / p.bs;
    s = 0;
    while (s < p.D - 1 && g >= chunk_begin(nblk, p.D, s + 1)) ++s;
    j = g - chunk_begin(nblk, p.D, s);
  }
  const int slot = (int)(t % p.bs);
  const int page = (j < p.mlb) ? p.table[s][(size_t)b * p.mlb + j] : -1;
  if (page < 0 || page >= p.pool_pages[s]) {
    if (report && p.err != nullptr) atomicOr(p.err, kDevBadPage);
    return false;
  }
  *s_out = s;
  *base_out = p.layout == DCP_LAYOUT_GQA ? ((size_t)page * 2 * p.Hkv * p.bs + slot) * (size_t)p.d * p.eb
                                         : ((size_t)page * p.bs + slot) * (size_t)p.d * p.eb;
  return true;
}

// Byte offset of piece v (source elements 8v .. 8v+7 of a row) relative to the
// row's slot offset.
__device__ __forceinline__ size_t piece_offset(const PlaceParams& p, int v) {
  if (p.layout != DCP_LAYOUT_GQA) return (size_t)v * 8 * p.eb;
  const int head_vecs = p.d / 8;  // pieces per head row
  const int kvh = v / head_vecs;  // (kv, h) pair index = kv * Hkv + h
  return ((size_t)kvh * p.bs * p.d + (size_t)(v - kvh * head_vecs) * 8) * p.eb;
}

// Store piece v (eight bf16 values `x`) of a row at `dst`: as is, or as E4M3 codes.
__device__ __forceinline__ void store_piece(const PlaceParams& p, int v, uint8_t* dst, uint4 x) {
  if (p.eb == 2) {
    *reinterpret_cast<uint4*>(dst) = x;
    return;
  }
  const float inv = (v / (p.d / 8)) < p.Hkv ? p.inv_k : p.inv_v;  // K half of the row, then V
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    c[i] = f32x2_to_e4m3x2(__fmul_rn(__uint_as_float(w[i] << 16), inv),
                           __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv));
  *reinterpret_cast<uint2*>(dst) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__global__ void __launch_bounds__(256) append_kv_kernel(const __grid_constant__ PlaceParams p) {
  const long rows = p.cu_seqlens[p.B];
  const int row_vecs = (p.layout == DCP_LAYOUT_GQA ? 2 * p.Hkv * p.d * 2 : p.d * 2) / 16;
  const long total = rows * row_vecs;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long r = i / row_vecs;
    const int v = (int)(i - r * row_vecs);
    int s;
    size_t base;
    if (!row_slot(p, r, v == 0, &s, &base)) continue;
    const uint4* srow = reinterpret_cast<const uint4*>(p.src + (size_t)r * row_vecs * 16);
    store_piece(p, v, p.pool[s] + base + piece_offset(p, v), __ldg(srow + v));
  }
}

__global__ void __launch_bounds__(256) place_kv_kernel(const __grid_constant__ PlaceParams p) {
  const long total = p.cu_seqlens[p.B];
  const int lane = threadIdx.x & 31;
  const long warps = (long)gridDim.x * (blockDim.x >> 5);
  const int row_bytes = p.layout == DCP_LAYOUT_GQA ? 2 * p.Hkv * p.d * 2 : p.d * 2;
  const int row_vecs = row_bytes / 16;
  for (long r = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < total; r += warps) {
    int s;
    size_t base;
    if (!row_slot(p, r, lane == 0, &s, &base)) continue;
    const uint4* srow = reinterpret_cast<const uint4*>(p.src + (size_t)r * row_bytes);
    for (int v = lane; v < row_vecs; v += 32) store_piece(p, v, p.pool[s] + base + piece_offset(p, v), __ldg(srow + v));
  }
}

dcp_status launch_place_kv(const dcp_attn_desc& d, int D, const void* kv_src, const int64_t* cu_seqlens,
                           const int32_t* token_begin, const int32_t* seq_lens, const int32_t* const* tables,
                           void* const* pools, const int32_t* pool_pages, int32_t* device_error, bool few_rows,
                           cudaStream_t st) {
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
  p.eb = kv_elem_bytes(d);
  p.rule = d.shard_rule;
  p.seq_lens = seq_lens;
  if (p.rule != 0 && seq_lens == nullptr) return DCP_ERR_INVALID_ARG;
  p.inv_k = p.eb == 1 ? 1.0f / d.k_scale : 1.f;
  p.inv_v = p.eb == 1 ? 1.0f / d.v_scale : 1.f;
  if (few_rows) {
    // sized for about four rows per request; the grid-stride loop covers any more
    const long pieces = (long)p.B * 4 * ((p.layout == DCP_LAYOUT_GQA ? 2 * p.Hkv * p.d * 2 : p.d * 2) / 16);
    const long want = (pieces + 255) / 256;
    const int blocks = (int)(want < device_sm_count() * 8 ? (want > 0 ? want : 1) : device_sm_count() * 8);
    append_kv_kernel<<<blocks, 256, 0, st>>>(p);
  } else {
    place_kv_kernel<<<device_sm_count() * 8, 256, 0, st>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

}  // namespace dcp
