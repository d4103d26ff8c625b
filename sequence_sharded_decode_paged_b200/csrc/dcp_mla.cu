// dcp_mla.cu -- MLA partial decode attention (absorbed form) over D interleaved paged shards.
//
// What it computes ("Efficient Decode Context Parallelism with vLLM for Long
// Context Workloads", A2 方法细节: MLA keeps one latent vector per token shared
// by every query head, and DCP splits that latent cache along the sequence;
// "vLLM长序列推理优化：DCP切分KV Cache原理与实战" §2.2/§3.2 for the shard layout):
// for every shard s, request b and query head h (64 heads),
//   s_t = scale * q[b][h] . C_t          (C_t: the 576-wide latent row of token t)
//   O_s[b][h] = sum_t softmax(s)_t * C_t[0:512],  LSE_s[b][h] = log-sum-exp of s,
// over the tokens of b that shard s stores.
//
// Design (121 flop per KV byte, about half the B200 bf16 ridge; with 64 heads
// the products are narrow, so tensor-pipe issue matters as much as HBM):
//  * Persistent CTAs (one per SM), each owning an equal contiguous range of the
//    concatenated local page lists of all (shard, request) segments; pieces of
//    a segment cut by a range boundary are merged by the last CTA to arrive.
//  * Pages are taken two at a time.  The pair stage holds both pages box by
//    box (box cb of page a in rows 0-63, of page b in rows 64-127 of a 16 KB
//    box), so the two pages form one 128-row operand:
//      S^T  = K Q^T   : tcgen05.mma M=128 (the pair's tokens) N=64 (heads)
//                       K=576 into one of two 64-column TMEM buffers -- half the
//                       instructions of a per-page M=64 product;
//      O^T += V^T P^T : M=128 (value dims, four tiles) N=64 (heads) K=128
//                       tokens; V^T is read straight from the pair stage as an
//                       MN-major operand, P^T from an MN-major tile (row =
//                       token) that the softmax writes into the pair's rope
//                       boxes (dead once S^T is done).
//  * Warp 0 (one thread): TMA producer.  Per segment piece the query tile
//    (64 x 576, 72 KB) and per pair the stage, in five load groups (value boxes
//    {0,1}, {2,3}, {4,5}, {6,7}, then the rope box): each group is reloaded
//    for the next pair as soon as the PV tile that reads it (or, for the rope
//    boxes, the whole PV) completes, and S^T of the next pair starts on the
//    groups that have landed.  Query + pair stage fill the shared memory.
//  * Warp 1: TMEM allocator; one thread issues S^T.  Each issue loop is fully
//    unrolled with constant descriptor steps: a lone issuing thread feeds the
//    tensor pipe only as fast as its own instruction latency allows.
//  * Warps 2-9: softmax in the transposed layout: thread t of warp w holds
//    token 32*(w%4) + t of the pair and heads 32*((w-2)/4) .. +31.  The
//    reference maximum of each head is an integer (log2 units), raised only
//    when a score exceeds it by more than 8 (then O^T is rescaled in TMEM by
//    an exact power of two); the common pair therefore needs no reduction
//    across threads, only one block-wide OR of "some score exceeds its
//    reference".  Each thread keeps running sums of its token slot; they are
//    reduced over the 128 slots once per segment.  Tokens past the sequence
//    end are masked in S and their value rows zeroed in shared memory before
//    the PV product, so stale cache contents never leak in.  Once the group
//    has written P^T (a hardware barrier), one of its threads issues the PV
//    product itself -- no mbarrier hand-off to another warp.  One warp waits on
//    each mbarrier for the group; the others sleep on a hardware barrier.
//    Epilogue: O^T rows (value dims) are read from TMEM, normalised per head
//    and stored with coalesced 128-byte writes.
//  * Multi-token decode (q_len > 1): blockIdx.y is the query token j; the
//    q_len CTAs of one page range run side by side (the grid keeps q_len x
//    ranges within one wave), so each latent page is fetched from HBM about
//    once and the other reads hit L2.  Token j masks the scores of tokens at
//    or past seq_len - (q_len - 1 - j).
//  * FP8 latent cache (KV8): pages hold E4M3 codes, 576 bytes per token, one
//    per-tensor scale.  The codes land inside the 16-bit pair stage itself and
//    are widened there, so the stage, the products and the softmax keep their
//    shapes: a value group's codes (dims 128g .. 128g+127, one 128-byte row per
//    token) land in the group's second box, the rope codes (dims 512-575, a
//    128-byte box half past the row end, which TMA fills with zeros and does
//    not read) in the rope box.  Two more warps (10-11, one per page of the
//    pair) widen each row to f16 in place -- every E4M3 value is an f16, so
//    exactly -- each thread rewriting only the rows it read, and convert the
//    query tile from bf16 to f16 (exact within f16's normal range) when it
//    lands.  Products run as kind::f16 with f16 operands; P^T is written as
//    f16; the scale multiplies the scores (folded into the exponent's FMA) and
//    the normalisation of O.
#include <float.h>
#include <stddef.h>

#include "dcp_device.cuh"
#include "dcp_internal.h"
#include "dcp_tcgen05.cuh"

namespace dcp {

namespace {

constexpr int kMlaThreads = 320;                      // producer warp, MMA warp, 8 softmax warps
constexpr int kMlaHeads = 64;
constexpr int kMlaDqk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaBs = 64;
constexpr uint32_t kBlockBytes = 8192;                // one page's box: 64 rows x 64 bf16, 128-byte swizzled
constexpr uint32_t kTileBytes = 9 * kBlockBytes;      // 64 rows x 576 bf16 (a page, or the query)
constexpr uint32_t kPairBox = 2 * kBlockBytes;        // a pair-stage box: page a rows 0-63, page b rows 64-127
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kTileBytes;               // the pair stage: 9 boxes of 16 KB
constexpr uint32_t kOffPT = kOffKV + 8 * kPairBox;    // P^T (128 tokens x 64 heads bf16) in the rope boxes
constexpr uint32_t kOffMisc = kOffKV + 9 * kPairBox;  // 221,184
constexpr uint32_t kMiscBytes = 4096;
// Split combine: per-piece softmax weights of the 64 rows, up to kCombineMax pieces at once.
constexpr int kCombineMax = 16;
constexpr uint32_t kOffW = kOffMisc + kMiscBytes;
constexpr uint32_t kMlaSmem = kOffW + kCombineMax * 64 * 4;  // 229,376 bytes
constexpr int kGroups = 5;
// Fixed work of a segment piece (query load, epilogue), in pages, charged ahead of every
// non-empty segment when the page ranges are cut: measured ~8.8 K cycles per piece against
// ~3.4 K per page of pair work.
constexpr int kMlaSegCost = 3;                            // load groups: boxes {0,1},{2,3},{4,5},{6,7},{8}
// Pairs whose pages are prefetched into L2 ahead of the pair being loaded (0: none).
#ifndef DCP_MLA_L2_PAIRS_AHEAD
#define DCP_MLA_L2_PAIRS_AHEAD 0
#endif
constexpr int kL2PairsAhead = DCP_MLA_L2_PAIRS_AHEAD;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;                         // O^T: 4 tiles x 64 columns
constexpr uint32_t kColS = 256;                       // S^T: 2 buffers x 64 columns
constexpr float kRescaleThreshold = 8.0f;             // log2 units
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = 8;
// FP8 cache: warps 10-11 widen the codes (warp 10: page a of a pair, warp 11: page b).
constexpr int kConvWarp0 = 10;
constexpr int kConvThreads = 64;
template <bool KV8>
__host__ __device__ constexpr int mla_threads() { return KV8 ? kMlaThreads + kConvThreads : kMlaThreads; }

struct MlaMisc {
  uint64_t q_full, q_empty, kv_full[kGroups], kv_empty[kGroups], s_full[2], s_empty[2], mma_done, pv_done;
  uint64_t cv_full[kGroups], qc_full;  // FP8: a group's codes / the query tile converted to f16
  uint32_t tmem_base;
  int bcast;
  alignas(16) float mref[kMlaHeads];  // integral reference maxima (log2 units); read as float4
  alignas(16) float msub[kMlaHeads];  // what the weights subtract: mref, or 0 while it is -inf
  alignas(16) float thr[kMlaHeads];   // raise when s*scale - msub passes it: the threshold, or -inf
  float alpha[kMlaHeads];     // factors of the latest raise (exact powers of two)
  float inv_l[kMlaHeads];
  float lse2[kMlaHeads];
  float part[4][kMlaHeads];   // per-sub-partition partial maxima or sums
  float* rowptr[kMlaHeads];   // epilogue / combine: head h's output row
  int scratch[32];
};
static_assert(sizeof(MlaMisc) <= kMiscBytes, "misc block");
static_assert(offsetof(MlaMisc, mref) % 16 == 0, "float4 reads of the reference maxima");
static_assert(offsetof(MlaMisc, msub) % 16 == 0 && offsetof(MlaMisc, thr) % 16 == 0, "float4 reads");
static_assert(kOffMisc % 16 == 0, "misc block alignment");

// Load group g: its first box and box count.
__host__ __device__ constexpr int group_box0(int g) { return g < 4 ? 2 * g : 8; }
__host__ __device__ constexpr int group_boxes(int g) { return g < 4 ? 2 : 1; }

}  // namespace

struct MlaParams {
  CUtensorMap kvmap[kMaxShards];
  CUtensorMap qmap;
  const uint8_t* pool[kMaxShards];
  const int32_t* table[kMaxShards];
  float* O[kMaxShards];
  float* LSE[kMaxShards];
  int pool_pages[kMaxShards];
  int shard_of_si[kMaxShards];
  const int32_t* seq_lens;
  int* status;
  int* counters;
  float* slots;
  float scale_log2;
  float v_scale;  // multiplies the normalised O (the FP8 latent's scale; 1 for bf16)
  int n_si, B, D, mlb, slot_floats, q_len;
  // Output layout: query heads are owned in consecutive slices of Hk heads; owner 0's O and
  // LSE rows start at O[si] / LSE[si], owner k's (k >= 1) at own_O[k] / own_L[k] (any address
  // this GPU can store to, a peer GPU's memory included).  The standard layout is Hk = 64 (a
  // single owner).
  int Hk;
  float* own_O[kMaxShards];
  float* own_L[kMaxShards];
};

namespace {

__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// tcgen05.mma with the descriptors passed as 32-bit halves: the issue loops add constant
// (byte offset >> 4) steps to the low words only, which hold the start-address field (a
// shared-memory offset below 256 KB never carries out of its 14 bits).  One thread issues
// back to back, so its own instruction latency sets how fast the tensor pipe is fed.
__device__ __forceinline__ void umma_bf16_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                             uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tmov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One lane of a converged warp (the lowest): the warp that issues tcgen05.mma stays
// converged around the issue, which lets the issue run at the tensor pipe's pace (a lone lane
// of a diverged warp issued the same products ~20 % slower in a microbenchmark).  Products and
// the commits that track them are issued from the same elected lane.
__device__ __forceinline__ bool elect_one() {
  uint32_t is;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(is));
  return is != 0;
}

// O^T += V^T P^T for one pair: 4 tiles of 128 value dims x KST 16-token steps, each tile
// releasing the two value boxes it read, then the rope boxes (P^T) and the pair's O^T.
// V^T: MN-major, 64-dim atoms one pair box apart; P^T: MN-major, one 64-head atom.
template <int KST>
__device__ __forceinline__ void issue_pv(uint32_t t_o, uint32_t v_lo, uint32_t v_hi, uint32_t p_lo, uint32_t p_hi,
                                         uint32_t idO, uint32_t acc0, MlaMisc* misc) {
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
    for (int ks = 0; ks < KST; ++ks)
      umma_bf16_lo(t_o + mt * 64, v_lo + ((2 * mt * kPairBox + ks * 2048) >> 4), v_hi, p_lo + ((ks * 2048) >> 4),
                   p_hi, idO, ks > 0 ? 1u : acc0);
    umma_commit(&misc->kv_empty[mt]);  // value boxes 2mt, 2mt+1 are free
  }
  umma_commit(&misc->kv_empty[4]);  // the rope boxes (P^T) are free, and the pair's O^T is complete
}

// This thread's P^T row: its token's weights for heads 32*hf .. +31 as bf16 (f16 for the FP8
// cache, whose products take f16 operands), four 16-byte chunks of the 128-byte-swizzled row.
template <bool F16>
__device__ __forceinline__ void write_pt(uint8_t* prow, const float (&w)[32], int hf, int tok) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 w4;
    if constexpr (F16)
      w4 = make_uint4(pack_f16x2(w[8 * c + 0], w[8 * c + 1]), pack_f16x2(w[8 * c + 2], w[8 * c + 3]),
                      pack_f16x2(w[8 * c + 4], w[8 * c + 5]), pack_f16x2(w[8 * c + 6], w[8 * c + 7]));
    else
      w4 = make_uint4(pack_bf16x2(w[8 * c + 0], w[8 * c + 1]), pack_bf16x2(w[8 * c + 2], w[8 * c + 3]),
                      pack_bf16x2(w[8 * c + 4], w[8 * c + 5]), pack_bf16x2(w[8 * c + 6], w[8 * c + 7]));
    *reinterpret_cast<uint4*>(prow + ((((uint32_t)(4 * hf + c)) ^ (uint32_t)(tok & 7)) << 4)) = w4;
  }
}

// FP8 cache: widen page slot x of load group g in place.  The group's codes sit in its landing
// box (value group g: box 2g+1, rope group: box 8), one 128-byte row per token (128-byte
// swizzled, as TMA wrote them): codes of dims 16k .. 16k+15 of the group in chunk k.  Chunks
// 0-3 become the f16 row of the group's first box (value: box 2g; rope: box 8 itself), chunks
// 4-7 the f16 row of box 2g+1 (value groups only).  A thread handles rows lane and lane + 32
// and reads a whole row before writing it: the only code bytes its stores overwrite are those
// of its own rows, so no other thread's input is touched.
__device__ __forceinline__ void widen_group(uint8_t* kv, int g, int x, int lane) {
  uint8_t* land = kv + (g < 4 ? 2 * g + 1 : 8) * kPairBox + x * kBlockBytes;
  uint8_t* first = kv + (g < 4 ? 2 * g : 8) * kPairBox + x * kBlockBytes;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const uint32_t r = (uint32_t)(lane + 32 * rr), sw = r & 7u;
    uint4 c[8];
    if (g < 4) {
#pragma unroll
      for (int k = 0; k < 8; ++k) c[k] = *reinterpret_cast<const uint4*>(land + r * 128 + (((uint32_t)k ^ sw) << 4));
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) c[k] = *reinterpret_cast<const uint4*>(land + r * 128 + (((uint32_t)k ^ sw) << 4));
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (g == 4 && k >= 4) break;
      uint4 lo, hi;  // f16 of codes 16k .. 16k+7, 16k+8 .. 16k+15
      e4m3x4_to_f16x2x2(c[k].x, lo.x, lo.y);
      e4m3x4_to_f16x2x2(c[k].y, lo.z, lo.w);
      e4m3x4_to_f16x2x2(c[k].z, hi.x, hi.y);
      e4m3x4_to_f16x2x2(c[k].w, hi.z, hi.w);
      uint8_t* row = (k < 4 ? first : land) + r * 128;
      const uint32_t m = (uint32_t)(2 * (k & 3));
      *reinterpret_cast<uint4*>(row + ((m ^ sw) << 4)) = lo;
      *reinterpret_cast<uint4*>(row + (((m + 1) ^ sw) << 4)) = hi;
    }
  }
}

// Wait unless the caller has already given up; a failed wait marks it dead.
__device__ __forceinline__ void wait_or_die(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  if (dead) return;
  if (!mbar_wait(bar, parity)) {
    atomicOr(status, kDevTimeout);
    dead = true;
  }
}

// Warp-wide variant: the verdict is made uniform across the warp.
__device__ __forceinline__ void wait_or_die_warp(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  wait_or_die(bar, parity, dead, status);
  dead = __any_sync(0xffffffffu, dead);
}

// Softmax-group variant: one warp (the group's first) waits on the mbarrier while the
// others sleep on hardware barrier `id`, which releases them with the verdict made uniform
// across the group (the tcgen05.ld / st that follow are warp-collective).  A whole group
// polling the mbarrier would keep the shared-memory port busy while the tensor core reads
// its operands from there.
__device__ __forceinline__ void wait_or_die_group(uint64_t* bar, uint32_t parity, bool& dead, int* status,
                                                  bool waiter, int id, int nthreads) {
  if (waiter) wait_or_die(bar, parity, dead, status);
  dead = bar_red_or(id, nthreads, dead);
}

__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool page_ok(const MlaParams& p, int si, int b, int j, int* page_out) {
  // a local block past the table row (lengths grown beyond max_local_blocks) is
  // treated like an out-of-pool page: never read, flagged in the status word
  const int page = j < p.mlb ? p.table[si][(size_t)b * p.mlb + j] : -1;
  *page_out = page;
  return page >= 0 && page < p.pool_pages[si];
}


// Reduces v[i] over the 32 lanes of the warp for every i = 0..31, transposed:
// lane l returns the result for index l.  At the step of width k each lane
// keeps one half of its remaining indices (the upper half if lane bit k is
// set) and exchanges the other half with lane l ^ k: 31 shuffles in all.
template <bool MAX>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = upper ? v[i] : v[i + k];
      const float keep = upper ? v[i + k] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, k);
      v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

}  // namespace

// RULE: the shard rule (0 interleaved, 1 contiguous chunks), fixed at compile time.
// KV8: the pools hold FP8 E4M3 codes (warps 10-11 widen them in shared memory).
template <int RULE, bool KV8>
__global__ void __launch_bounds__(mla_threads<KV8>(), 1) mla_decode_kernel(const __grid_constant__ MlaParams p) {
  constexpr int kThreads = mla_threads<KV8>();
  extern __shared__ __align__(1024) uint8_t smem[];
  MlaMisc* misc = reinterpret_cast<MlaMisc*>(smem + kOffMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, nctas = gridDim.x;
  const int jq = blockIdx.y, ql = p.q_len;  // query token of this CTA
  const int B = p.B, D = p.D;

  if ((smem_u32(smem) & 1023u) != 0u) {  // swizzled tiles need 1024-byte alignment
    if (tid == 0) atomicOr(p.status, kDevTimeout);
    return;
  }
  if (tid == 0) {
    mbar_init(&misc->q_full, 1);
    mbar_init(&misc->q_empty, 1);
    for (int g = 0; g < kGroups; ++g) {
      mbar_init(&misc->kv_full[g], 1);
      mbar_init(&misc->kv_empty[g], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&misc->s_full[i], 1);
      mbar_init(&misc->s_empty[i], kSoftmaxWarps);
    }
    mbar_init(&misc->mma_done, 1);
    mbar_init(&misc->pv_done, 1);
    if (KV8) {
      for (int g = 0; g < kGroups; ++g) mbar_init(&misc->cv_full[g], kConvThreads);
      mbar_init(&misc->qc_full, kConvThreads);
    }
    fence_barrier_init();
  }
  // The products read every row of the pair stage, also rows no page fills (a pair's
  // missing second page, a skipped page): their scores are masked and their weights are
  // zero, so they only need to be finite -- zero the stage once.
  for (uint32_t i = tid; i < 9 * kPairBox / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + kOffKV)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.qmap);
    for (int si = 0; si < p.n_si; ++si)
      if (p.pool_pages[si] > 0) prefetch_tmap(&p.kvmap[si]);
  }
  if (warp == 1) {
    tmem_alloc(&misc->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc->tmem_base;

  const CtaPlan plan =
      plan_cta_r<RULE>(p.seq_lens, B, p.n_si, p.shard_of_si, kMlaBs, D, cta, nctas, misc->scratch, kMlaSegCost);
  const int T = plan.T, P = plan.P;
  const int lo = cta * P, hi = min(lo + P, T);
  const int S = p.n_si * B;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t q_ph = 0;
      long pc = 0;                 // pairs started
      long last[kGroups];          // last pair each group was loaded for (-1: none)
      for (int g = 0; g < kGroups; ++g) last[g] = -1;
      bool dead = false, q_issued = false;
      int pre = plan.pre0;
      for (int sid = plan.sid0; sid < S && !dead; ++sid) {
        const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
        const int n = local_pages_r<RULE>(p.seq_lens[b], kMlaBs, D, shard);
        if (n > 0) pre += kMlaSegCost;  // the segment's fixed-work units precede its pages
        if (seg_first_cta(pre, n, T, P) > cta) break;
        const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
        pre += n;
        if (n == 0) continue;
        wait_or_die(&misc->q_empty, q_ph ^ 1u, dead, p.status);
        q_ph ^= 1u;
        if (dead) break;
        mbar_arrive_expect_tx(&misc->q_full, kTileBytes);
        for (int cb = 0; cb < 9; ++cb)
          tma_load_2d(smem + kOffQ + cb * kBlockBytes, &p.qmap, cb * 64, (b * ql + jq) * kMlaHeads, &misc->q_full);
        q_issued = true;
        for (int j = a; j < e && !dead; j += 2) {
          int pa = -1, pb = -1;
          const bool oka = page_ok(p, si, b, j, &pa);
          const bool two = j + 1 < e;
          const bool okb = two && page_ok(p, si, b, j + 1, &pb);
          if (!oka || (two && !okb)) atomicOr(p.status, kDevBadPage);
          if (kL2PairsAhead > 0) {
            for (int jj = j + 2 * kL2PairsAhead; jj < min(e, j + 2 * kL2PairsAhead + 2); ++jj) {
              int pp;
              if (page_ok(p, si, b, jj, &pp)) prefetch_l2_bulk(p.pool[si] + (size_t)pp * kTileBytes, kTileBytes);
            }
          }
          const uint32_t par = (uint32_t)(pc & 1);
          for (int g = 0; g < kGroups; ++g) {
            wait_or_die(&misc->kv_empty[g], par ^ 1u, dead, p.status);
            if (dead) break;
            const int nb = group_boxes(g), cb0 = group_box0(g);
            // FP8: one 128-byte box of codes per page (the rope box reads 64 bytes, the rest is fill)
            const uint32_t bytes = (KV8 ? kBlockBytes : nb * kBlockBytes) * ((oka ? 1u : 0u) + (okb ? 1u : 0u));
            last[g] = pc;
            if (bytes == 0) {
              mbar_arrive(&misc->kv_full[g]);
              continue;
            }
            mbar_arrive_expect_tx(&misc->kv_full[g], bytes);
            if (KV8) {
              uint8_t* dst = smem + kOffKV + (g < 4 ? 2 * g + 1 : 8) * kPairBox;  // the group's landing box
              if (oka) tma_load_2d(dst, &p.kvmap[si], 128 * g, pa * kMlaBs, &misc->kv_full[g]);
              if (okb) tma_load_2d(dst + kBlockBytes, &p.kvmap[si], 128 * g, pb * kMlaBs, &misc->kv_full[g]);
            } else {
              for (int cb = cb0; cb < cb0 + nb; ++cb) {
                uint8_t* dst = smem + kOffKV + cb * kPairBox;
                if (oka) tma_load_2d(dst, &p.kvmap[si], cb * 64, pa * kMlaBs, &misc->kv_full[g]);
                if (okb) tma_load_2d(dst + kBlockBytes, &p.kvmap[si], cb * 64, pb * kMlaBs, &misc->kv_full[g]);
              }
            }
          }
          ++pc;
        }
      }
      // never leave with a copy into shared memory in flight
      for (int g = 0; g < kGroups; ++g)
        if (last[g] >= 0) {
          bool d2 = false;
          wait_or_die(&misc->kv_full[g], (uint32_t)(last[g] & 1), d2, p.status);
        }
      if (q_issued) {
        bool d2 = false;
        wait_or_die(&misc->q_full, q_ph ^ 1u, d2, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S^T issuer
    {  // the whole warp walks the pairs and waits; an elected lane issues
      const uint32_t idS = KV8 ? idesc_f16_f32(128, 64, false, false) : idesc_bf16_f32(128, 64, false, false);
      // K rows (A) and the query (B): K-major, one 8-row group per 1,024 bytes
      const uint64_t k_desc = sw128_desc(smem_u32(smem + kOffKV), 16, 1024);
      const uint64_t q_desc = sw128_desc(smem_u32(smem + kOffQ), 16, 1024);
      const uint32_t k_lo = (uint32_t)k_desc, k_hi = (uint32_t)(k_desc >> 32);
      const uint32_t q_lo = (uint32_t)q_desc, q_hi = (uint32_t)(q_desc >> 32);
      uint32_t q_ph = 0;
      long pc = 0;
      bool dead = false;
      int pre = plan.pre0;
      for (int sid = plan.sid0; sid < S && !dead; ++sid) {
        const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
        const int n = local_pages_r<RULE>(p.seq_lens[b], kMlaBs, D, shard);
        if (n > 0) pre += kMlaSegCost;  // the segment's fixed-work units precede its pages
        if (seg_first_cta(pre, n, T, P) > cta) break;
        const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
        pre += n;
        if (n == 0) continue;
        wait_or_die_warp(KV8 ? &misc->qc_full : &misc->q_full, q_ph, dead, p.status);
        q_ph ^= 1u;
        for (int j = a; j < e && !dead; j += 2) {
          // Per pair: S^T = K Q^T group by group as the groups land.  (The softmax group
          // issues the pair's PV product itself once P^T is written.)
          const uint32_t sb = (uint32_t)(pc & 1), par = (uint32_t)(pc & 1);
          wait_or_die_warp(&misc->s_empty[sb], (uint32_t)((pc >> 1) & 1) ^ 1u, dead, p.status);
          const uint32_t dS = tbase + kColS + sb * 64;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) {
            wait_or_die_warp(KV8 ? &misc->cv_full[g] : &misc->kv_full[g], par, dead, p.status);
            if (dead) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
              for (int cb = group_box0(g); cb < group_box0(g) + group_boxes(g); ++cb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                  umma_bf16_lo(dS, k_lo + ((cb * kPairBox + ks * 32) >> 4), k_hi,
                               q_lo + ((cb * kBlockBytes + ks * 32) >> 4), q_hi, idS, (cb > 0 || ks > 0) ? 1u : 0u);
            }
            __syncwarp();
          }
          if (dead) break;
          if (elect_one()) {
            umma_commit(&misc->s_full[sb]);
            if (j + 2 >= e) umma_commit(&misc->q_empty);  // Q is free once these products are done
          }
          __syncwarp();
          ++pc;
        }
      }
      if (elect_one()) umma_commit(&misc->mma_done);  // everything issued has completed before TMEM is released
      __syncwarp();
      bool d2 = false;
      wait_or_die(&misc->mma_done, 0, d2, p.status);
    }
  } else if (warp < kConvWarp0) {
    // ------------------------------------------------------------ softmax + epilogue (warps 2-9)
    // Warp w reads TMEM sub-partition q4 = w % 4: lanes 32*q4 .. +31 hold the pair's tokens
    // 32*q4 .. +31 (page a below 64, page b from 64); half hf = (w - 2) / 4 takes the heads
    // 32*hf .. +31 (columns of S^T).
    const int q4 = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int ts = tid - 64;                       // 0..255
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const int tok = 32 * q4 + lane;                // token of the pair this thread holds
    const bool waiter = warp == 2;                 // the warp that waits on the group's mbarriers
    const uint32_t idO = KV8 ? idesc_f16_f32(128, 64, true, true) : idesc_bf16_f32(128, 64, true, true);
    const uint64_t v_desc = sw128_desc(smem_u32(smem + kOffKV), kPairBox, 1024);
    const uint64_t p_desc = sw128_desc(smem_u32(smem + kOffPT), kPairBox, 1024);
    const uint32_t v_lo = (uint32_t)v_desc, v_hi = (uint32_t)(v_desc >> 32);
    const uint32_t p_lo = (uint32_t)p_desc, p_hi = (uint32_t)(p_desc >> 32);
    const int slot = tok >> 6, trow = tok & 63;    // its page (0: a, 1: b) and row in that page
    long pc = 0;
    bool dead = false;
    int pre = plan.pre0;
    for (int sid = plan.sid0; sid < S; ++sid) {
      const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
      const int seq_len = p.seq_lens[b];
      const int n = local_pages_r<RULE>(seq_len, kMlaBs, D, shard);
      if (n > 0) pre += kMlaSegCost;  // the segment's fixed-work units precede its pages
      const int c0 = seg_first_cta(pre, n, T, P);
      if (c0 > cta) break;
      const int c1 = seg_last_cta(pre, n, T, P);
      // output row of head h: owner h / Hk, row (b * ql + jq) * Hk + h % Hk of that owner's block
      const size_t row0 = ((size_t)b * ql + jq) * p.Hk;
      auto o_row = [&](int h) -> float* {
        const int own = h / p.Hk;
        return (own == 0 ? p.O[si] : p.own_O[own]) + (row0 + (h - own * p.Hk)) * kMlaDv;
      };
      auto l_ptr = [&](int h) -> float* {
        const int own = h / p.Hk;
        return (own == 0 ? p.LSE[si] : p.own_L[own]) + row0 + (h - own * p.Hk);
      };
      const int lim = seq_len - (ql - 1 - jq);  // tokens this query token sees
      // logical block of local page j: g0 + j * gstride (computed once per segment)
      const int g0 = global_block(0, seq_len, kMlaBs, D, shard, RULE);
      const int gstride = RULE != 0 ? 1 : D;
      if (n == 0) {
        for (int i = ts; i < kMlaHeads * kMlaDv / 4; i += kSoftmaxThreads)
          reinterpret_cast<float4*>(o_row(i / (kMlaDv / 4)))[i % (kMlaDv / 4)] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ts < kMlaHeads) *l_ptr(ts) = -INFINITY;
        pre += n;
        continue;
      }
      const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
      // One sum of the fp32 weights normalises O and gives the LSE, so pieces of a
      // split sequence merge back to the unsplit result (up to fp32 order); the PV
      // product uses the same weights rounded to bf16.  l: the running sums of this
      // thread's token slot for its 32 heads; the reference maxima live in misc->mref.
      float l[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) l[i] = 0.f;
      if (ts < kMlaHeads) {
        misc->mref[ts] = -INFINITY;
        misc->msub[ts] = 0.f;
        misc->thr[ts] = -INFINITY;
      }
      named_bar_sync(2, kSoftmaxThreads);  // the references are reset before any thread reads them
      const float4* msub4 = reinterpret_cast<const float4*>(misc->msub + 32 * hf);
      const float4* thr4 = reinterpret_cast<const float4*>(misc->thr + 32 * hf);
      for (int j = a; j < e; j += 2) {
        const bool two = j + 1 < e;
        int pa = -1, pb = -1;
        const bool oka = page_ok(p, si, b, j, &pa);
        const bool okb = two && page_ok(p, si, b, j + 1, &pb);
        const int tok0a = (g0 + j * gstride) * kMlaBs, tok0b = (g0 + (j + 1) * gstride) * kMlaBs;
        const bool mine_ok = slot == 0 ? oka : okb;
        const bool visible = mine_ok && trow < lim - (slot == 0 ? tok0a : tok0b);
        const uint32_t sb = (uint32_t)(pc & 1);
        wait_or_die_group(&misc->s_full[sb], (uint32_t)((pc >> 1) & 1), dead, p.status, waiter, 2, kSoftmaxThreads);
        tc_fence_after();
        float s[32];
        if (!dead) {
          tmem_ld32(tbase + lane_off + kColS + sb * 64 + 32 * hf, s);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->s_empty[sb]);
        // zero the value rows past the sequence end (dims 0..511) of the pair's pages:
        // they may hold stale values, which the zero weights must not multiply
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          const bool okx = x == 0 ? oka : okb;
          const int valid = min(kMlaBs, seq_len - (x == 0 ? tok0a : tok0b));
          if (!okx || dead || valid >= kMlaBs) continue;
          const int nchunks = (kMlaBs - valid) * 64;
          for (int i = ts; i < nchunks; i += kSoftmaxThreads) {
            const int row = valid + (i >> 6), cb = (i >> 3) & 7, ch = i & 7;
            *reinterpret_cast<uint4*>(smem + kOffKV + cb * kPairBox + x * kBlockBytes + row * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        const bool see = visible && !dead;
        // Weights against the current references, optimistically: w = 2^(s*scale - m) in one FMA
        // (m: the head's reference, 0 while it has none).  A score past its reference by more
        // than the threshold -- or any visible score of a head without a reference -- makes the
        // whole group redo the pair below after raising references; a piece's first pair
        // (references just reset) goes there directly.  The OR barrier that takes that
        // decision also tells the issuing thread that every P^T row is written.
        bool raise = j == a;
        if (!raise) {
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 m4 = msub4[i4], t4 = thr4[i4];
            const float mm[4] = {m4.x, m4.y, m4.z, m4.w}, th[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = 4 * i4 + k;
              const float t = see ? fmaf(s[i], p.scale_log2, -mm[k]) : -INFINITY;
              raise = raise || t > th[k];
              s[i] = ex2_approx(t);
            }
          }
          if (!dead) write_pt<KV8>(smem + kOffPT + tok * 128, s, hf, tok);
        }
        fence_proxy_async_smem();  // P^T rows and zeroed value rows -> the async proxy
        tc_fence_before();
        if (bar_red_or(2, kSoftmaxThreads, raise)) {
          // ---- references move (rare): the pair's scores again (S^T buffer sb is rewritten
          // only for a pair whose groups this pair's PV releases), exact maxima per head: over
          // the warp's 32 tokens (transposed: lane i gets head 32*hf + i), then over the four
          // sub-partitions; heads whose maximum passes their reference by more than the
          // threshold get a new integral reference
          tc_fence_after();
          if (!dead && j != a) {  // (a piece's first pair skipped the weights: s still holds the scores)
            tmem_ld32(tbase + lane_off + kColS + sb * 64 + 32 * hf, s);
            tmem_ld_wait();
          }
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = see ? s[i] * p.scale_log2 : -INFINITY;
          misc->part[q4][32 * hf + lane] = warp_transpose_reduce<true>(v, lane);
          named_bar_sync(2, kSoftmaxThreads);
          bool changed = false;
          if (ts < kMlaHeads) {
            const float pm = fmaxf(fmaxf(misc->part[0][ts], misc->part[1][ts]),
                                   fmaxf(misc->part[2][ts], misc->part[3][ts]));
            const float mo = misc->mref[ts];
            float mn = mo;
            if (mo == -INFINITY || pm > mo + kRescaleThreshold) mn = ceilf(pm);
            const float al = mn == mo ? 1.f : exp2_int(mo - mn);
            misc->alpha[ts] = al;
            misc->mref[ts] = mn;
            misc->msub[ts] = mn == -INFINITY ? 0.f : mn;
            misc->thr[ts] = mn == -INFINITY ? -INFINITY : kRescaleThreshold;
            changed = al != 1.f;
          }
          const bool resc = bar_red_or(2, kSoftmaxThreads, changed) && j > a;  // O^T holds earlier pairs
#pragma unroll
          for (int i = 0; i < 32; ++i) l[i] *= misc->alpha[32 * hf + i];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 m4 = msub4[i4];
            const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = 4 * i4 + k;
              s[i] = ex2_approx(see ? fmaf(s[i], p.scale_log2, -mm[k]) : -INFINITY);
            }
          }
          if (!dead) write_pt<KV8>(smem + kOffPT + tok * 128, s, hf, tok);
          if (resc) {
            // O^T holds the earlier pairs: observe the previous pair's PV completion before
            // rescaling it.  (That PV has finished by now -- it released the groups this pair's
            // S^T needed -- so pairs without a rescale skip the wait.  The barrier completes
            // once per pair and cannot pass this phase before this pair's PV is issued, so the
            // phase parity is the previous pair's index.)
            wait_or_die_group(&misc->kv_empty[4], (uint32_t)((pc - 1) & 1), dead, p.status, waiter, 2, kSoftmaxThreads);
            tc_fence_after();
            if (!dead) {
#pragma unroll 1
              for (int mt = 2 * hf; mt < 2 * hf + 2; ++mt)
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                  const uint32_t ta = tbase + lane_off + kColO + mt * 64 + c;
                  tmem_ld32(ta, v);
                  tmem_ld_wait();
#pragma unroll
                  for (int i = 0; i < 32; ++i) v[i] *= misc->alpha[c + i];
                  tmem_st32(ta, v);
                }
              tmem_st_wait();
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          named_bar_sync(2, kSoftmaxThreads);  // P^T rewritten, O^T rescaled
        }
        // one thread issues the pair's PV product.  (The previous piece's epilogue read O^T
        // before the barriers above, so a fresh accumulation may begin.)
        if (waiter && !dead) {  // (dead is uniform across the group)
          tc_fence_after();
          const uint32_t acc0 = j > a ? 1u : 0u;  // O^T holds earlier pairs of this piece
          if (elect_one()) {
            if (two) issue_pv<8>(tbase + kColO, v_lo, v_hi, p_lo, p_hi, idO, acc0, misc);
            else issue_pv<4>(tbase + kColO, v_lo, v_hi, p_lo, p_hi, idO, acc0, misc);  // no second page
          }
          __syncwarp();
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) l[i] += s[i];  // (off the path to the PV issue)
        ++pc;
      }
      // ---------------------------------------------------------- epilogue
      // the piece's last PV: its final commit (the rope group's release) marks O^T complete
      wait_or_die_group(&misc->kv_empty[4], (uint32_t)((pc - 1) & 1), dead, p.status, waiter, 2, kSoftmaxThreads);
      tc_fence_after();
      // row sums over the 128 token slots: over the warp's 32 (transposed), then the sub-partitions
      misc->part[q4][32 * hf + lane] = warp_transpose_reduce<false>(l, lane);
      const bool complete = (c0 == c1);
      const int slot_i = complete ? 0 : 2 * cta + ((cta == c0 && pre != c0 * P) ? 1 : 0);
      float* slot_base = p.slots + ((size_t)slot_i * ql + jq) * p.slot_floats;
      named_bar_sync(2, kSoftmaxThreads);
      if (ts < kMlaHeads) {
        const float lt = (misc->part[0][ts] + misc->part[1][ts]) + (misc->part[2][ts] + misc->part[3][ts]);
        const float mh = misc->mref[ts];
        misc->inv_l[ts] = lt > 0.f ? (KV8 ? p.v_scale / lt : 1.f / lt) : 0.f;
        misc->lse2[ts] = lt > 0.f ? mh + __log2f(lt) : -INFINITY;
        // row pointers once per piece, so that the stores below need no owner arithmetic
        misc->rowptr[ts] = complete ? o_row(ts) : slot_base + (size_t)ts * kMlaDv;
      }
      named_bar_sync(2, kSoftmaxThreads);
#pragma unroll 1
      for (int mt = 2 * hf; mt < 2 * hf + 2; ++mt)
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          float v[32];
          if (!dead) {
            tmem_ld32(tbase + lane_off + kColO + mt * 64 + c, v);
            tmem_ld_wait();
          }
          const int col = mt * 128 + 32 * q4 + lane;  // this thread's value dim
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float inv = misc->inv_l[c + i];
            misc->rowptr[c + i][col] = (inv == 0.f || dead) ? 0.f : v[i] * inv;
          }
        }
      if (ts < kMlaHeads) {
        if (complete) *l_ptr(ts) = misc->lse2[ts] * kLn2;
        else slot_base[kMlaHeads * kMlaDv + ts] = misc->lse2[ts];
      }
      tc_fence_before();  // O^T reads complete before the next piece's first PV (ordered by its barrier)
      if (!complete) {
        __threadfence();
        named_bar_sync(2, kSoftmaxThreads);
        int* ctr = p.counters + (size_t)sid * ql + jq;
        if (ts == 0) misc->bcast = (atomicAdd(ctr, 1) == c1 - c0) ? 1 : 0;
        named_bar_sync(2, kSoftmaxThreads);
        if (misc->bcast) {
          __threadfence();
          const int np = c1 - c0 + 1;
          // every piece's slot into L2 with one bulk prefetch each (pieces finished long ago may
          // have left L2 under the cache stream): the loads below then wait on L2, not HBM
          if (ts < np) {
            const int c = c0 + ts, k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
            prefetch_l2_bulk(p.slots + ((size_t)k * ql + jq) * p.slot_floats, (uint32_t)p.slot_floats * 4u);
          }
          if (np <= kCombineMax) {
            // Weights of every (piece, row) first, one thread per row, into shared memory;
            // then every thread merges 16-byte chunks of the rows with all of its loads
            // independent of one another (8 rows at a time, every piece), so the pieces
            // stream from L2 with many requests in flight instead of one row at a time.
            float* wt = reinterpret_cast<float*>(smem + kOffW);  // [piece][row]
            if (ts < kMlaHeads) {
              // every piece's LSE of this row loaded at once (one round trip), then the weights
              float lk[kCombineMax];
#pragma unroll
              for (int i = 0; i < kCombineMax; ++i) {
                lk[i] = -INFINITY;
                if (i < np) {
                  const int c = c0 + i, k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                  lk[i] = __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kMlaHeads * kMlaDv + ts);
                }
              }
              float mx = -INFINITY;
#pragma unroll
              for (int i = 0; i < kCombineMax; ++i) mx = fmaxf(mx, lk[i]);
              float wsum = 0.f;
#pragma unroll
              for (int i = 0; i < kCombineMax; ++i) {
                if (i < np) {
                  const float w = (mx == -INFINITY || lk[i] == -INFINITY) ? 0.f : exp2f(lk[i] - mx);
                  wsum += w;
                  wt[i * kMlaHeads + ts] = w;
                }
              }
              misc->inv_l[ts] = wsum > 0.f ? 1.f / wsum : 0.f;
              *l_ptr(ts) = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
              misc->rowptr[ts] = o_row(ts);
            }
            named_bar_sync(2, kSoftmaxThreads);
            const int ch = ts & 127, rh = ts >> 7;  // chunk of a row; rows 2u + rh
#pragma unroll 1
            for (int u0 = 0; u0 < kMlaHeads / 2; u0 += 8) {
              float4 acc[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
              for (int i = 0; i < np; ++i) {
                const int c = c0 + i, k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                const float4* src = reinterpret_cast<const float4*>(p.slots + ((size_t)k * ql + jq) * p.slot_floats) + ch;
                float4 x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = __ldcg(src + (size_t)(2 * (u0 + u) + rh) * (kMlaDv / 4));
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const float w = wt[i * kMlaHeads + 2 * (u0 + u) + rh];
                  acc[u].x += w * x[u].x;
                  acc[u].y += w * x[u].y;
                  acc[u].z += w * x[u].z;
                  acc[u].w += w * x[u].w;
                }
              }
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int r = 2 * (u0 + u) + rh;
                const float inv = misc->inv_l[r];
                reinterpret_cast<float4*>(misc->rowptr[r])[ch] =
                    make_float4(acc[u].x * inv, acc[u].y * inv, acc[u].z * inv, acc[u].w * inv);
              }
            }
          } else {
            // many pieces (a segment cut across more than kCombineMax CTAs): row by row
            const int w8 = ts >> 5;
            for (int r = w8; r < kMlaHeads; r += kSoftmaxWarps) {
              float mx = -INFINITY;
              for (int c = c0; c <= c1; ++c) {
                const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                mx = fmaxf(mx, __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kMlaHeads * kMlaDv + r));
              }
              float4 acc[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
              float wsum = 0.f;
              if (mx != -INFINITY) {
                for (int c = c0; c <= c1; ++c) {
                  const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                  const float* sl = p.slots + ((size_t)k * ql + jq) * p.slot_floats;
                  const float lk = __ldcg(sl + kMlaHeads * kMlaDv + r);
                  const float w = lk == -INFINITY ? 0.f : exp2f(lk - mx);
                  wsum += w;
                  const float4* src = reinterpret_cast<const float4*>(sl + (size_t)r * kMlaDv) + lane * 4;
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    const float4 x = __ldcg(src + i);
                    acc[i].x += w * x.x;
                    acc[i].y += w * x.y;
                    acc[i].z += w * x.z;
                    acc[i].w += w * x.w;
                  }
                }
              }
              const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
              float4* out = reinterpret_cast<float4*>(o_row(r)) + lane * 4;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                out[i] = make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
              if (lane == 0) *l_ptr(r) = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
            }
          }
          if (ts == 0) *ctr = 0;  // ready for the next call
        }
      }
      pre += n;
    }
    if (waiter) {  // every PV product issued here has completed before TMEM is released
      if (elect_one()) umma_commit(&misc->pv_done);
      __syncwarp();
      bool d2 = false;
      wait_or_die(&misc->pv_done, 0, d2, p.status);
    }
  }

  if (KV8 && warp >= kConvWarp0) {
    // ------------------------------------------------------------ FP8 -> f16 (warps 10-11)
    // The same walk as the producer: per segment piece the query tile, per pair the five load
    // groups.  Warp 10 widens page a of every pair, warp 11 page b; a page that was not loaded
    // (a pair's missing second page, an invalid page id) keeps what its rows held, as in the
    // bf16 stage.  Every converter thread arrives on the group's barrier after its own stores
    // and a proxy fence, so the products see every row.
    const int x = warp - kConvWarp0, ct = tid - kMlaThreads;
    uint32_t q_ph = 0;
    long pc = 0;
    bool dead = false;
    int pre = plan.pre0;
    for (int sid = plan.sid0; sid < S && !dead; ++sid) {
      const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
      const int n = local_pages_r<RULE>(p.seq_lens[b], kMlaBs, D, shard);
      if (n > 0) pre += kMlaSegCost;  // the segment's fixed-work units precede its pages
      if (seg_first_cta(pre, n, T, P) > cta) break;
      const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
      pre += n;
      if (n == 0) continue;
      wait_or_die_warp(&misc->q_full, q_ph, dead, p.status);
      q_ph ^= 1u;
      if (dead) break;
      for (int i = ct; i < (int)(kTileBytes / 16); i += kConvThreads) {  // bf16 -> f16, in place
        uint4* c = reinterpret_cast<uint4*>(smem + kOffQ) + i;
        uint4 v = *c;
        v.x = bf16x2_to_f16x2(v.x);
        v.y = bf16x2_to_f16x2(v.y);
        v.z = bf16x2_to_f16x2(v.z);
        v.w = bf16x2_to_f16x2(v.w);
        *c = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(&misc->qc_full);
      for (int j = a; j < e && !dead; j += 2) {
        int pg = -1;
        const bool ok = x == 0 ? page_ok(p, si, b, j, &pg) : (j + 1 < e && page_ok(p, si, b, j + 1, &pg));
        const uint32_t par = (uint32_t)(pc & 1);
#pragma unroll 1
        for (int g = 0; g < kGroups; ++g) {
          wait_or_die_warp(&misc->kv_full[g], par, dead, p.status);
          if (dead) break;
          if (ok) widen_group(smem + kOffKV, g, x, lane);
          fence_proxy_async_smem();
          mbar_arrive(&misc->cv_full[g]);
        }
        ++pc;
      }
    }
  }

  // ---------------------------------------------------------------- release TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ---------------------------------------------------------------------------- host side
// CTAs per query token: q_len x ranges fill one wave (one CTA per SM).
int mla_ctas(int q_len) {
  const int n = device_sm_count() / q_len;
  return n > 0 ? n : 1;
}

dcp_status launch_mla_decode(const dcp_attn_desc& d, int D, const ShardSet& set, const void* q,
                             const int32_t* seq_lens, void* ws, size_t ws_bytes, cudaStream_t stream) {
  WorkspaceLayout L;
  if (!workspace_layout(d, D, &L)) return DCP_ERR_UNSUPPORTED;
  if (ws_bytes < L.total) return DCP_ERR_CAPACITY;
  MlaParams p;
  memset(&p, 0, sizeof(p));
  p.n_si = set.n;
  p.B = d.batch;
  p.D = D;
  p.mlb = d.max_local_blocks;
  p.slot_floats = L.slot_floats;
  const bool kv8 = d.kv_dtype == DCP_KV_FP8_E4M3;
  // FP8: the latent's scale multiplies every score (folded into the exponent) and the normalised O
  p.scale_log2 = kv8 ? (float)((double)d.softmax_scale * (double)d.k_scale * 1.4426950408889634)
                     : d.softmax_scale * 1.4426950408889634f;
  p.v_scale = kv8 ? d.v_scale : 1.f;
  p.q_len = d.q_len;
  p.Hk = set.owner_heads > 0 ? set.owner_heads : kMlaHeads;
  for (int k = 0; k < kMaxShards; ++k) {
    p.own_O[k] = set.owner_O[k];
    p.own_L[k] = set.owner_L[k];
  }
  p.seq_lens = seq_lens;
  p.status = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.status_off);
  p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.counters_off);
  p.slots = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.slots_off);
  const uint64_t q_rows = (uint64_t)d.batch * d.q_len * kMlaHeads;  // q: [batch][q_len][64][576]
  if (q_rows > (uint64_t)INT32_MAX) return DCP_ERR_UNSUPPORTED;
  if (encode_tiled_2d(&p.qmap, q, kMlaDqk, q_rows, kMlaDqk * 2, 64, 64) != CUDA_SUCCESS) return DCP_ERR_CUDA;
  for (int si = 0; si < set.n; ++si) {
    p.pool[si] = static_cast<const uint8_t*>(set.pool[si]);
    p.table[si] = set.table[si];
    p.O[si] = set.O[si];
    p.LSE[si] = set.LSE[si];
    p.pool_pages[si] = set.pool_pages[si];
    p.shard_of_si[si] = set.shard[si];
    if (set.pool_pages[si] > 0) {
      const uint64_t rows = (uint64_t)set.pool_pages[si] * kMlaBs;
      if (rows > (uint64_t)INT32_MAX) return DCP_ERR_UNSUPPORTED;  // TMA row coordinates are int32
      // FP8: 128-byte boxes of codes (the rope group's box starts at byte 512 and runs past the
      // 576-byte row: TMA fills the missing part and does not read it)
      const CUresult r = kv8 ? encode_tiled_2d(&p.kvmap[si], set.pool[si], kMlaDqk, rows, kMlaDqk, 128, 64, 1)
                             : encode_tiled_2d(&p.kvmap[si], set.pool[si], kMlaDqk, rows, kMlaDqk * 2, 64, 64);
      if (r != CUDA_SUCCESS) return DCP_ERR_CUDA;
    }
  }
  auto kern = d.shard_rule == DCP_SHARD_INTERLEAVED ? (kv8 ? mla_decode_kernel<0, true> : mla_decode_kernel<0, false>)
                                                    : (kv8 ? mla_decode_kernel<1, true> : mla_decode_kernel<1, false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMlaSmem) != cudaSuccess)
    return DCP_ERR_CUDA;
  kern<<<dim3(L.nctas, d.q_len), kv8 ? mla_threads<true>() : mla_threads<false>(), kMlaSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

}  // namespace dcp
