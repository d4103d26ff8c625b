// dcp_device.cuh -- device-side building blocks shared by the DCP kernels
// (sm_100a): mbarrier / TMA / ldmatrix / mma.sync wrappers with bounded
// waits, the status word, and the balanced work planner that cuts the
// concatenated local page lists of all (shard, request) segments into equal
// contiguous ranges, one per CTA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace dcp {

constexpr int kMaxShards = 16;

// Device status bits (workspace word 0).
constexpr int kDevBadPage = 1;  // a table entry pointed outside its pool
constexpr int kDevTimeout = 2;  // a pipeline wait exceeded its time limit (never expected)

// A wait that has not completed after this many nanoseconds is abandoned.
constexpr unsigned long long kWaitLimitNs = 4000000000ull;

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity` of `bar`.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; false if the time limit passed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u && global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled load of box (x, y) of tensor map `m` into shared memory; completion
// is signalled on `bar` as transaction bytes.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* m, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------- ldmatrix / mma.sync
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col)
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two f32 -> packed f16x2 (round to nearest even): `lo` in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes (bits 0-7 and 8-15 of `x`) -> f16x2 (exact: every E4M3 value is an f16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t x) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(x));
  return r;
}

// Four E4M3 codes (bytes of w) -> two f16x2: bytes 0-1 -> lo, bytes 2-3 -> hi (exact).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Two f32 -> two E4M3 codes, nearest even, magnitudes past 448 saturated: `lo` in bits 0-7.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// bf16x2 -> f16x2 (round to nearest even; exact for f16's normal range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  return pack_f16x2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^k for an integer-valued k <= 0 (or -inf), exactly: the running maxima of the
// online softmax are kept integral (in log2 units), so every rescale factor is
// an exact power of two and P values computed against different maxima differ
// only by powers of two -- which bf16 rounding preserves, so results do not
// depend on how a sequence was split (across shards or across CTAs).
__device__ __forceinline__ float exp2_int(float k) {
  if (!(k >= -126.f)) return 0.f;  // -inf and tiny factors
  return __int_as_float(((int)k + 127) << 23);
}

__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// 2^x by the PTX ex2.approx instruction (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk `chunk` of row `row` inside a 128-byte-swizzled
// tile (TMA CU_TENSOR_MAP_SWIZZLE_128B: rows of 128 B, chunk index XOR row % 8;
// the tile base must be 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Byte offset of 16-byte chunk `chunk` (0-3) of row `row` inside a 64-byte-swizzled tile of
// 64-byte rows (TMA CU_TENSOR_MAP_SWIZZLE_64B: the chunk index XOR bits 7-8 of the byte offset,
// i.e. row / 2 % 4; the tile base must be 512-byte aligned).
__device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t chunk) {
  return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// ---------------------------------------------------------------- work planning
// Segments are (shard slot si, request b) pairs, sid = si * B + b, laid out in
// that order; segment sid holds n(sid) local pages (the blocks g < ceil(len/bs)
// with g % D == shard).  The concatenation of all segments' pages is cut into
// ranges of P = ceil(T / nctas) pages; CTA c owns pages [c*P, (c+1)*P).
struct SegmentInfo {
  int sid;     // segment id
  int pre;     // first page of the segment in the concatenation
  int n;       // pages of the segment
};

// Shard rules (the descriptor's shard_rule): 0 = interleaved, block g -> shard g % D as local
// block g / D; 1 = contiguous chunks, shard s holds the blocks [chunk_begin(s), chunk_begin(s+1))
// with chunk_begin(s) = floor(s * nblk / D), local block g - chunk_begin(s).
__device__ __forceinline__ int chunk_begin(int nblk, int D, int s) { return (int)(((long long)s * nblk) / D); }

// Local pages of `shard` in a request of seq_len tokens (kernels are instantiated per rule).
template <int RULE>
__device__ __forceinline__ int local_pages_r(int seq_len, int bs, int D, int shard) {
  const int nblk = (seq_len + bs - 1) / bs;
  if constexpr (RULE != 0) return chunk_begin(nblk, D, shard + 1) - chunk_begin(nblk, D, shard);
  else return nblk > shard ? (nblk - 1 - shard) / D + 1 : 0;
}

// Logical block of local page j of `shard` in a request of seq_len tokens.
__device__ __forceinline__ int global_block(int j, int seq_len, int bs, int D, int shard, int rule) {
  if (rule != 0) return chunk_begin((seq_len + bs - 1) / bs, D, shard) + j;
  return j * D + shard;
}

// First CTA that works on a segment, and the last one.  An empty segment
// (n == 0) belongs to exactly one CTA: the owner of page min(pre, T-1).
__device__ __forceinline__ int seg_first_cta(int pre, int n, int T, int P) {
  if (n > 0) return pre / P;
  return T > 0 ? min(pre, T - 1) / P : 0;
}
__device__ __forceinline__ int seg_last_cta(int pre, int n, int T, int P) {
  if (n > 0) return (pre + n - 1) / P;
  return seg_first_cta(pre, n, T, P);
}

// Plan shared by the whole CTA (computed by all threads of the block).
struct CtaPlan {
  int T;        // total pages of the launch
  int P;        // pages per CTA
  int sid0;     // first segment this CTA touches (S if none)
  int pre0;     // its first page in the concatenation
};

// Block-wide planner for shard rule RULE.  Every thread of the block must call it.  `scratch`
// holds at least (blockDim.x / 32 + 4) ints of shared memory.
// seg_cost: units charged to every non-empty segment ahead of its pages (its fixed work: query
// load, epilogue), so that the equal ranges balance work rather than pages.  The kernel loops
// then advance `pre` by seg_cost before each non-empty segment's pages (0: pages only).
template <int RULE>
__device__ __forceinline__ CtaPlan plan_cta_r(const int32_t* __restrict__ seq_lens, int B, int n_si,
                                              const int* shard_of_si, int bs, int D, int cta, int nctas,
                                              int* scratch, int seg_cost = 0) {
  const int S = n_si * B;
  const int nt = blockDim.x;
  const int tid = threadIdx.x;
  const int per = (S + nt - 1) / nt;
  const int s_begin = min(S, tid * per);
  const int s_end = min(S, s_begin + per);
  int local = 0;
  for (int sid = s_begin; sid < s_end; ++sid) {
    const int si = sid / B, b = sid - si * B;
    const int n = local_pages_r<RULE>(seq_lens[b], bs, D, shard_of_si[si]);
    local += n + (n > 0 ? seg_cost : 0);
  }
  // block exclusive scan of `local`
  const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    if (lane < nw) scratch[lane] = wi - w;  // exclusive warp offsets
    if (lane == nw - 1) scratch[nw] = wi;   // total
  }
  __syncthreads();
  const int T = scratch[nw];
  const int P = T > 0 ? (T + nctas - 1) / nctas : 1;
  int pre = scratch[warp] + incl - local;  // exclusive prefix of this thread's first segment
  if (tid == 0) {
    scratch[nw + 1] = S;
    scratch[nw + 2] = T;
  }
  __syncthreads();
  // first segment whose last CTA is >= cta (monotone in sid)
  for (int sid = s_begin; sid < s_end; ++sid) {
    const int si = sid / B, b = sid - si * B;
    const int n = local_pages_r<RULE>(seq_lens[b], bs, D, shard_of_si[si]);
    if (n > 0) pre += seg_cost;
    if (seg_last_cta(pre, n, T, P) >= cta) {
      atomicMin(&scratch[nw + 1], sid);
      break;
    }
    pre += n;
  }
  __syncthreads();
  CtaPlan plan;
  plan.T = T;
  plan.P = P;
  plan.sid0 = scratch[nw + 1];
  plan.pre0 = 0;
  // the thread whose range contains sid0 publishes its prefix
  if (plan.sid0 >= s_begin && plan.sid0 < s_end) {
    int p2 = scratch[warp] + incl - local;
    for (int sid = s_begin; sid < plan.sid0; ++sid) {
      const int si = sid / B, b = sid - si * B;
      const int n = local_pages_r<RULE>(seq_lens[b], bs, D, shard_of_si[si]);
      p2 += n + (n > 0 ? seg_cost : 0);
    }
    scratch[nw + 2] = p2;
  }
  __syncthreads();
  plan.pre0 = plan.sid0 < S ? scratch[nw + 2] : T;
  __syncthreads();  // scratch may be reused by the caller
  return plan;
}

}  // namespace dcp
