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
// Design (121 flop per KV byte, about half the B200 bf16 ridge, so both the
// HBM stream and the tensor pipe matter):
//  * Persistent CTAs (one per SM), each owning an equal contiguous range of the
//    concatenated local page lists of all (shard, request) segments; pieces of
//    a segment cut by a range boundary are merged by the last CTA to arrive.
//  * Warp 0 (one thread): TMA producer.  Per segment the query tile (64 x 576
//    bf16, 72 KB) and per page the latent tile (64 tokens x 576, 72 KB), both
//    as nine 64 x 64 boxes with 128-byte swizzle, into a 2-stage ring (two
//    72 KB stages and the 72 KB query tile fill the shared memory).
//  * Warp 1: TMEM allocator and the single MMA-issuing thread.
//      S  = Q K^T   : tcgen05.mma M=64 (heads) N=64 (tokens) K=576, into one of
//                     two 64-column TMEM buffers (head h in lane h%16 + 32*(h/16)).
//      O^T += V^T P^T: M=128 (value dims, four tiles) N=64 (heads) K=64 tokens;
//                     V^T is read straight from the latent tile as an MN-major
//                     operand, P^T from a 64 x 64 bf16 tile the softmax writes
//                     into the page's own rope box (dead after QK^T), so the
//                     softmax of a page never waits for the previous PV product.
//    S of page i+1 is issued before O of page i, so the tensor pipe works while
//    the softmax runs.
//  * Warps 2-9: softmax (two warps per TMEM sub-partition of 16 head rows, each
//    on half the page's tokens, four threads per head row), fp32, base-2; the
//    reference maximum is an integer and is only raised (O^T rescaled in TMEM
//    by an exact power of two) when a page's maximum exceeds it by more than 8
//    (a factor of 256); the result is unchanged because the final
//    normalisation uses the same reference.  Tokens
//    past the sequence end are masked in S and their value rows zeroed in
//    shared memory before the PV product, so stale cache contents never leak in.
//    Epilogue: O^T rows (value dims) are read from TMEM, normalised per head
//    and stored with coalesced 128-byte writes.
//  * Multi-token decode (q_len > 1): blockIdx.y is the query token j; the
//    q_len CTAs of one page range run side by side (the grid keeps q_len x
//    ranges within one wave), so each latent page is fetched from HBM about
//    once and the other reads hit L2.  Token j masks the scores of tokens at
//    or past seq_len - (q_len - 1 - j).
#include <float.h>

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
constexpr uint32_t kBlockBytes = 8192;                // 64 rows x 64 bf16, 128-byte swizzled
constexpr uint32_t kTileBytes = 9 * kBlockBytes;      // 64 rows x 576 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kTileBytes;               // two stages
// P^T (64 heads x 64 tokens bf16, 8 KB) of a page lives in its stage's rope box (dims 512-575 of
// the latent tile), which only QK^T reads: no separate buffer.
constexpr uint32_t kOffMisc = 3 * kTileBytes;
// Split combine: per-piece softmax weights of the 64 rows, up to kCombineMax pieces at once.
constexpr int kCombineMax = 16;
constexpr uint32_t kOffW = kOffMisc + 3072;
constexpr uint32_t kMlaSmem = kOffW + kCombineMax * 64 * 4;  // 228,352 bytes
// Pages prefetched into L2 ahead of the page whose tile load is being issued (0: none).
#ifndef DCP_MLA_L2_AHEAD
#define DCP_MLA_L2_AHEAD 0
#endif
constexpr int kL2Ahead = DCP_MLA_L2_AHEAD;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;                         // O^T: 4 tiles x 64 columns
constexpr uint32_t kColS = 256;                       // S: 2 buffers x 64 columns
constexpr float kRescaleThreshold = 8.0f;             // log2 units
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = 8;

struct MlaMisc {
  // kv_empty[st][g]: the groups of a stage that become free at different times --
  // g = 0 the rope box (read by QK^T only), g = 1 value boxes 0-3 (PV tiles 0-1),
  // g = 2 value boxes 4-7 (PV tiles 2-3) -- so the next page streams in early.
  uint64_t q_full, q_empty, kv_full[2], kv_empty[2][3], s_full[2], s_empty[2], p_full, o_done, o_free, mma_done;
  uint32_t tmem_base;
  int bcast;
  float alpha[kMlaHeads];
  float inv_l[kMlaHeads];
  float lse2[kMlaHeads];
  float pmax[2][2][kMlaHeads];  // [page parity][token half][head]: page maxima exchanged between halves
  float lpart[kMlaHeads];       // token-half 1's row sums at the epilogue
  int scratch[32];
};
static_assert(sizeof(MlaMisc) <= 3072, "misc block");

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
  int n_si, B, D, mlb, slot_floats, q_len;
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

// Wait unless the caller has already given up; a failed wait marks it dead.
__device__ __forceinline__ void wait_or_die(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  if (dead) return;
  if (!mbar_wait(bar, parity)) {
    atomicOr(status, kDevTimeout);
    dead = true;
  }
}

// Warp-wide variant: the verdict is made uniform across the warp, because the
// tcgen05.ld / st that follow are warp-collective.
__device__ __forceinline__ void wait_or_die_warp(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  wait_or_die(bar, parity, dead, status);
  dead = __any_sync(0xffffffffu, dead);
}

// Walks the pages of a CTA's range in order (segment by segment), for the L2 prefetch.
template <int RULE>
struct PageCursor {
  int sid, pre, si, b, j, e;
  bool live;
  __device__ __forceinline__ void init(int sid0, int pre0) {
    sid = sid0;
    pre = pre0;
    j = e = si = b = 0;
    live = true;
  }
  // Next page of the range: (slot, request, local block); false at its end.
  __device__ __forceinline__ bool next(const MlaParams& p, int S, int T, int P, int cta, int lo, int hi, int* osi,
                                       int* ob, int* oj) {
    while (live) {
      if (j < e) {
        *osi = si;
        *ob = b;
        *oj = j++;
        return true;
      }
      if (sid >= S) break;
      const int si2 = sid / p.B, b2 = sid - si2 * p.B;
      const int n2 = local_pages_r<RULE>(p.seq_lens[b2], kMlaBs, p.D, p.shard_of_si[si2]);
      if (seg_first_cta(pre, n2, T, P) > cta) break;
      si = si2;
      b = b2;
      j = max(pre, lo) - pre;
      e = n2 > 0 ? min(pre + n2, hi) - pre : 0;
      pre += n2;
      ++sid;
    }
    live = false;
    return false;
  }
};

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

}  // namespace

// RULE: the shard rule (0 interleaved, 1 contiguous chunks), fixed at compile time.
template <int RULE>
__global__ void __launch_bounds__(kMlaThreads, 1) mla_decode_kernel(const __grid_constant__ MlaParams p) {
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&misc->kv_full[i], 1);
      for (int g = 0; g < 3; ++g) mbar_init(&misc->kv_empty[i][g], 1);
      mbar_init(&misc->s_full[i], 1);
      mbar_init(&misc->s_empty[i], kSoftmaxWarps);
    }
    mbar_init(&misc->p_full, kSoftmaxWarps);
    mbar_init(&misc->o_done, 1);
    mbar_init(&misc->o_free, kSoftmaxWarps);
    mbar_init(&misc->mma_done, 1);
    fence_barrier_init();
  }
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

  const CtaPlan plan = plan_cta_r<RULE>(p.seq_lens, B, p.n_si, p.shard_of_si, kMlaBs, D, cta, nctas, misc->scratch);
  const int T = plan.T, P = plan.P;
  const int lo = cta * P, hi = min(lo + P, T);
  const int S = p.n_si * B;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t st = 0, kv_ph = 0, q_ph = 0;
      long issued = 0;
      bool dead = false, q_issued = false;
      int pre = plan.pre0;
      // L2 prefetch kL2Ahead pages ahead of the page whose tile load is issued next
      PageCursor<RULE> ahead;
      ahead.init(plan.sid0, plan.pre0);
      auto prefetch_next = [&]() {
        int asi, ab, aj, apage;
        if (ahead.next(p, S, T, P, cta, lo, hi, &asi, &ab, &aj) && page_ok(p, asi, ab, aj, &apage))
          prefetch_l2_bulk(p.pool[asi] + (size_t)apage * kTileBytes, kTileBytes);
      };
      if (kL2Ahead > 0)
        for (int i = 0; i < kL2Ahead; ++i) prefetch_next();
      for (int sid = plan.sid0; sid < S; ++sid) {
        const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
        const int n = local_pages_r<RULE>(p.seq_lens[b], kMlaBs, D, shard);
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
        for (int j = a; j < e; ++j) {
          int page;
          const bool ok = page_ok(p, si, b, j, &page);
          if (!ok) atomicOr(p.status, kDevBadPage);
          if (kL2Ahead > 0) prefetch_next();
          uint8_t* dst = smem + kOffKV + st * kTileBytes;
          // box groups in the order they are freed: value boxes 0-3, value boxes 4-7, rope box
          // (the rope box holds the page's P^T tile until its PV product is done)
          for (int gi = 0; gi < 3 && !dead; ++gi) {
            const int g = gi == 2 ? 0 : gi + 1;
            wait_or_die(&misc->kv_empty[st][g], kv_ph ^ 1u, dead, p.status);
            if (dead) break;
            if (ok) {
              if (gi == 0) mbar_arrive_expect_tx(&misc->kv_full[st], kTileBytes);
              if (g == 0) {
                tma_load_2d(dst + 8 * kBlockBytes, &p.kvmap[si], 8 * 64, page * kMlaBs, &misc->kv_full[st]);
              } else {
                for (int cb = 4 * (g - 1); cb < 4 * g; ++cb)
                  tma_load_2d(dst + cb * kBlockBytes, &p.kvmap[si], cb * 64, page * kMlaBs, &misc->kv_full[st]);
              }
            } else if (gi == 2) {
              mbar_arrive(&misc->kv_full[st]);
            }
          }
          if (dead) break;
          ++issued;
          if (++st == 2) {
            st = 0;
            kv_ph ^= 1u;
          }
        }
        if (dead) break;
      }
      // never leave with a copy into shared memory in flight
      const long first = issued > 2 ? issued - 2 : 0;
      for (long i = first; i < issued; ++i) {
        bool d2 = false;
        wait_or_die(&misc->kv_full[i & 1], (uint32_t)((i >> 1) & 1), d2, p.status);
      }
      if (q_issued) {
        bool d2 = false;
        wait_or_die(&misc->q_full, q_ph ^ 1u, d2, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Two cursors over the CTA's page sequence: S = Q K^T of page js and
    // O^T += V^T P^T of page jo < js, each issued as soon as its inputs are
    // ready (O first: it frees a stage for the next load).  The tensor pipe
    // executes in issue order, so this keeps a late page load from holding
    // back the PV product of the page before it.
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64, false, false);
      const uint32_t idO = idesc_bf16_f32(128, 64, true, false);
      const uint32_t qa = smem_u32(smem + kOffQ);
      struct PageRec {
        bool ok, seg_first, seg_last;
      };
      PageRec ring[4];
      uint32_t q_ph = 0, p_ph = 0, of_ph = 0;
      long js = 0, jo = 0, known = 0;  // S issued, O issued, pages enumerated
      bool dead = false, o_init = false;
      // segment walk producing page records
      int w_sid = plan.sid0, w_pre = plan.pre0, w_j = 0, w_e = 0, w_si = 0, w_b = 0, w_a = 0;
      bool w_live = true;
      auto enumerate = [&]() {  // append the next page record to the ring; false at the end
        while (w_live) {
          if (w_j < w_e) {
            int page;
            PageRec r;
            r.ok = page_ok(p, w_si, w_b, w_j, &page);
            r.seg_first = (w_j == w_a);
            r.seg_last = (w_j == w_e - 1);
            ring[known & 3] = r;
            ++known;
            ++w_j;
            return true;
          }
          if (w_sid >= S) { w_live = false; break; }
          const int si2 = w_sid / B, b2 = w_sid - si2 * B;
          const int n2 = local_pages_r<RULE>(p.seq_lens[b2], kMlaBs, D, p.shard_of_si[si2]);
          if (seg_first_cta(w_pre, n2, T, P) > cta) { w_live = false; break; }
          w_si = si2;
          w_b = b2;
          w_a = w_j = max(w_pre, lo) - w_pre;
          w_e = n2 > 0 ? min(w_pre + n2, hi) - w_pre : 0;
          w_pre += n2;
          ++w_sid;
        }
        return false;
      };
      unsigned long long idle_since = 0;
      while (!dead) {
        if (known == js) enumerate();
        bool progressed = false;
        if (jo < js && mbar_test(&misc->p_full, p_ph)) {
          const PageRec r = ring[jo & 3];
          p_ph ^= 1u;
          if (r.seg_first) {  // the previous segment's epilogue must have read O^T
            wait_or_die(&misc->o_free, of_ph ^ 1u, dead, p.status);
            of_ph ^= 1u;
            o_init = false;
          }
          tc_fence_after();
          const uint32_t ost = (uint32_t)(jo & 1);
          if (r.ok && !dead) {
            const uint64_t ad = sw128_desc(smem_u32(smem + kOffKV + ost * kTileBytes), kBlockBytes, 1024);
            // P^T of this page sits in its stage's rope box (free once QK^T of the page is done)
            const uint64_t bd = sw128_desc(smem_u32(smem + kOffKV + ost * kTileBytes + 8 * kBlockBytes), 16, 1024);
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tbase + kColO + mt * 64, ad + (uint64_t)((2 * mt * kBlockBytes + ks * 2048) >> 4),
                          bd + (uint64_t)((ks * 32) >> 4), idO, (o_init || ks > 0) ? 1u : 0u);
              if (mt == 1) umma_commit(&misc->kv_empty[ost][1]);  // value boxes 0-3 are free
            }
            o_init = true;
          } else {
            umma_commit(&misc->kv_empty[ost][1]);
          }
          umma_commit(&misc->kv_empty[ost][2]);  // value boxes 4-7 are free
          umma_commit(&misc->kv_empty[ost][0]);  // the rope box (P^T) is free
          umma_commit(&misc->o_done);
          ++jo;
          progressed = true;
        }
        if (js < known && js - jo < 2) {
          const PageRec r = ring[js & 3];
          const uint32_t st = (uint32_t)(js & 1), par = (uint32_t)((js >> 1) & 1);
          const bool ready = (!r.seg_first || mbar_test(&misc->q_full, q_ph)) && mbar_test(&misc->kv_full[st], par) &&
                             mbar_test(&misc->s_empty[st], par ^ 1u);
          if (ready) {
            if (r.seg_first) q_ph ^= 1u;
            tc_fence_after();
            if (r.ok) {
              // descriptors advance by adding (byte offset >> 4) to the start-address field
              const uint64_t ad = sw128_desc(qa, 16, 1024);
              const uint64_t bd = sw128_desc(smem_u32(smem + kOffKV + st * kTileBytes), 16, 1024);
              const uint32_t dS = tbase + kColS + st * 64;
#pragma unroll
              for (int ks = 0; ks < 36; ++ks) {
                const uint64_t off = (uint64_t)(((ks >> 2) * kBlockBytes + (ks & 3) * 32) >> 4);
                umma_bf16(dS, ad + off, bd + off, idS, ks > 0 ? 1u : 0u);
              }
            }
            umma_commit(&misc->s_full[st]);
            if (r.seg_last) umma_commit(&misc->q_empty);  // Q is free once these S products are done
            ++js;
            progressed = true;
          }
        }
        if (js == known && jo == js && !w_live) break;
        if (progressed) {
          idle_since = 0;
        } else {
          const unsigned long long now = global_ns();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            atomicOr(p.status, kDevTimeout);
            dead = true;
          }
        }
      }
      umma_commit(&misc->mma_done);  // everything issued has completed before TMEM is released
      bool d2 = false;
      wait_or_die(&misc->mma_done, 0, d2, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 2-9)
    // Warps 2-9: warp w reads TMEM sub-partition q = w % 4, which holds head rows
    // 16q..16q+15 of S (lanes 32q..32q+15), and token half hf = (w - 2) / 4 of
    // the page.  With the 16x256b load thread t holds heads hr0 = 16q + t/4 and
    // hr1 = hr0 + 8, tokens 32*hf + 8k + 2*(t%4) + {0,1}, k = 0..3; the two
    // halves exchange their page maxima through shared memory.
    const int q4 = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int ts = tid - 64;                       // 0..255
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const int quad = lane & 3;
    const int hr0 = 16 * q4 + (lane >> 2), hr1 = hr0 + 8;
    uint32_t gpage = 0, od_ph = 0, st = 0;
    bool dead = false;
    int pre = plan.pre0;
    for (int sid = plan.sid0; sid < S; ++sid) {
      const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
      const int seq_len = p.seq_lens[b];
      const int n = local_pages_r<RULE>(seq_len, kMlaBs, D, shard);
      const int c0 = seg_first_cta(pre, n, T, P);
      if (c0 > cta) break;
      const int c1 = seg_last_cta(pre, n, T, P);
      float* Oout = p.O[si] + ((size_t)b * ql + jq) * kMlaHeads * kMlaDv;
      float* Lout = p.LSE[si] + ((size_t)b * ql + jq) * kMlaHeads;
      const int lim = seq_len - (ql - 1 - jq);  // tokens this query token sees
      // logical block of local page j: g0 + j * gstride (computed once per segment)
      const int g0 = global_block(0, seq_len, kMlaBs, D, shard, RULE);
      if (n == 0) {
        for (int i = ts; i < kMlaHeads * kMlaDv / 4; i += kSoftmaxThreads)
          reinterpret_cast<float4*>(Oout)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ts < kMlaHeads) Lout[ts] = -INFINITY;
        pre += n;
        continue;
      }
      const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
      // One sum of the fp32 weights normalises O and gives the LSE, so pieces of a
      // split sequence merge back to the unsplit result (up to fp32 order); the
      // PV product uses the same weights rounded to bf16.  l0 / l1 are this
      // thread's partial sums (its 16 tokens of each page), reduced at the end.
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      bool have_o = false;
      for (int j = a; j < e; ++j) {
        int page;
        const bool ok = page_ok(p, si, b, j, &page);
        const int tok0 = (g0 + j * (RULE != 0 ? 1 : D)) * kMlaBs;  // first token of the page
        const int valid = min(kMlaBs, seq_len - tok0);
        const int vis = lim - tok0;  // visible tokens of this page (may be <= 0)
        const uint32_t sb = gpage & 1u;
        wait_or_die_warp(&misc->s_full[sb], (gpage >> 1) & 1u, dead, p.status);
        tc_fence_after();
        float s[16];
        if (ok && !dead) {
          tmem_ld16x256b_x4(tbase + lane_off + kColS + sb * 64 + 32 * hf, s);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->s_empty[sb]);
        bool need = false;
        float a0 = 1.f, a1 = 1.f, pm0 = -INFINITY, pm1 = -INFINITY;
        if (ok && !dead) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int tok = 32 * hf + 8 * k + 2 * quad + (i & 1);
              s[4 * k + i] = tok < vis ? s[4 * k + i] * p.scale_log2 : -INFINITY;
            }
          pm0 = fmaxf(fmaxf(fmaxf(s[0], s[1]), fmaxf(s[4], s[5])), fmaxf(fmaxf(s[8], s[9]), fmaxf(s[12], s[13])));
          pm1 = fmaxf(fmaxf(fmaxf(s[2], s[3]), fmaxf(s[6], s[7])), fmaxf(fmaxf(s[10], s[11]), fmaxf(s[14], s[15])));
          pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, 1));
          pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, 2));
          pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, 1));
          pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, 2));
        }
        {  // page maximum over both token halves (the partner warp holds the other half);
           // the exchange runs on every page so both partners meet the barrier
          float* xm = misc->pmax[gpage & 1][hf];
          if (quad == 0) {
            xm[hr0] = pm0;
            xm[hr1] = pm1;
          }
          named_bar_sync(3 + q4, 64);
          const float* om = misc->pmax[gpage & 1][hf ^ 1];
          pm0 = fmaxf(pm0, om[hr0]);
          pm1 = fmaxf(pm1, om[hr1]);
        }
        if (ok && !dead) {
          // integral reference maximum, raised only past the threshold (exact power-of-two rescale)
          if (m0 == -INFINITY || pm0 > m0 + kRescaleThreshold) {
            const float mn = ceilf(pm0);
            a0 = exp2_int(m0 - mn);
            m0 = mn;
            need = have_o;
          }
          if (m1 == -INFINITY || pm1 > m1 + kRescaleThreshold) {
            const float mn = ceilf(pm1);
            a1 = exp2_int(m1 - mn);
            m1 = mn;
            need = need || have_o;
          }
          // a row with no visible token so far keeps -inf: subtract 0 so ex2 gives 0
          const float sub0 = m0 == -INFINITY ? 0.f : m0, sub1 = m1 == -INFINITY ? 0.f : m1;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            s[4 * k + 0] = ex2_approx(s[4 * k + 0] - sub0);
            s[4 * k + 1] = ex2_approx(s[4 * k + 1] - sub0);
            s[4 * k + 2] = ex2_approx(s[4 * k + 2] - sub1);
            s[4 * k + 3] = ex2_approx(s[4 * k + 3] - sub1);
          }
          l0 = l0 * a0 + (((s[0] + s[1]) + (s[4] + s[5])) + ((s[8] + s[9]) + (s[12] + s[13])));
          l1 = l1 * a1 + (((s[2] + s[3]) + (s[6] + s[7])) + ((s[10] + s[11]) + (s[14] + s[15])));
        }
        if (ok && !dead) {
          uint8_t* kv = smem + kOffKV + st * kTileBytes;
          if (valid < kMlaBs) {  // zero the value rows of tokens past the end (dims 0..511)
            const int nchunks = (kMlaBs - valid) * 64;
            for (int i = ts; i < nchunks; i += kSoftmaxThreads) {
              const int row = valid + (i >> 6), cb = (i >> 3) & 7, ch = i & 7;
              *reinterpret_cast<uint4*>(kv + cb * kBlockBytes + row * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          // P^T tile (K-major, 128-byte swizzle) in this stage's rope box, which QK^T of the page
          // has finished reading (s_full): 4-byte pieces, the quad fills each 16-byte chunk.  Each
          // page has its own P^T, so this needs no wait for the previous page's PV product.
          uint8_t* pt = kv + 8 * kBlockBytes + 4 * quad;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t ch = (uint32_t)(4 * hf + k);
            *reinterpret_cast<uint32_t*>(pt + sw128((uint32_t)hr0, ch)) = pack_bf16x2(s[4 * k + 0], s[4 * k + 1]);
            *reinterpret_cast<uint32_t*>(pt + sw128((uint32_t)hr1, ch)) = pack_bf16x2(s[4 * k + 2], s[4 * k + 3]);
          }
        }
        if (j > a) {  // O^T of the previous page is complete: O^T may be rescaled
          wait_or_die_warp(&misc->o_done, od_ph, dead, p.status);
          od_ph ^= 1u;
          tc_fence_after();
        }
        if (bar_red_or(2, kSoftmaxThreads, need)) {
          if (quad == 0 && hf == 0) {
            misc->alpha[hr0] = a0;
            misc->alpha[hr1] = a1;
          }
          named_bar_sync(2, kSoftmaxThreads);
          if (!dead) {
#pragma unroll 1
            for (int mt = 2 * hf; mt < 2 * hf + 2; ++mt)
#pragma unroll 1
              for (int c = 0; c < 64; c += 32) {
                float v[32];
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
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->p_full);
        have_o = have_o || ok;
        ++gpage;
        st ^= 1u;
      }
      // ---------------------------------------------------------- epilogue
      wait_or_die_warp(&misc->o_done, od_ph, dead, p.status);
      od_ph ^= 1u;
      tc_fence_after();
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if (quad == 0 && hf == 1) {
        misc->lpart[hr0] = l0;
        misc->lpart[hr1] = l1;
      }
      named_bar_sync(2, kSoftmaxThreads);
      if (quad == 0 && hf == 0) {
        l0 += misc->lpart[hr0];
        l1 += misc->lpart[hr1];
        misc->inv_l[hr0] = (l0 > 0.f && have_o) ? 1.f / l0 : 0.f;
        misc->lse2[hr0] = (l0 > 0.f && have_o) ? m0 + __log2f(l0) : -INFINITY;
        misc->inv_l[hr1] = (l1 > 0.f && have_o) ? 1.f / l1 : 0.f;
        misc->lse2[hr1] = (l1 > 0.f && have_o) ? m1 + __log2f(l1) : -INFINITY;
      }
      named_bar_sync(2, kSoftmaxThreads);
      const bool complete = (c0 == c1);
      const int slot = complete ? 0 : 2 * cta + ((cta == c0 && pre != c0 * P) ? 1 : 0);
      float* slot_base = p.slots + ((size_t)slot * ql + jq) * p.slot_floats;
      float* dstO = complete ? Oout : slot_base;
      float* dstL = complete ? Lout : slot_base + kMlaHeads * kMlaDv;
#pragma unroll 1
      for (int mt = 2 * hf; mt < 2 * hf + 2; ++mt)
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          float v[32];
          if (!dead) {
            tmem_ld32(tbase + lane_off + kColO + mt * 64 + c, v);
            tmem_ld_wait();
          }
          const int dv = mt * 128 + 32 * q4 + lane;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float inv = misc->inv_l[c + i];
            dstO[(size_t)(c + i) * kMlaDv + dv] = (inv == 0.f || dead) ? 0.f : v[i] * inv;
          }
        }
      if (ts < kMlaHeads) dstL[ts] = complete ? misc->lse2[ts] * kLn2 : misc->lse2[ts];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&misc->o_free);
      if (!complete) {
        __threadfence();
        named_bar_sync(2, kSoftmaxThreads);
        int* ctr = p.counters + (size_t)sid * ql + jq;
        if (ts == 0) misc->bcast = (atomicAdd(ctr, 1) == c1 - c0) ? 1 : 0;
        named_bar_sync(2, kSoftmaxThreads);
        if (misc->bcast) {
          __threadfence();
          const int np = c1 - c0 + 1;
          if (np <= kCombineMax) {
            // Weights of every (piece, row) first, one thread per row, into shared memory;
            // then every thread merges 16-byte chunks of the rows with all of its loads
            // independent of one another (8 rows at a time, every piece), so the pieces
            // stream from L2 with many requests in flight instead of one row at a time.
            float* wt = reinterpret_cast<float*>(smem + kOffW);  // [piece][row]
            if (ts < kMlaHeads) {
              float mx = -INFINITY;
              for (int c = c0; c <= c1; ++c) {
                const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                mx = fmaxf(mx, __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kMlaHeads * kMlaDv + ts));
              }
              float wsum = 0.f;
              for (int i = 0; i < np; ++i) {
                const int c = c0 + i, k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                const float lk = __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kMlaHeads * kMlaDv + ts);
                const float w = (mx == -INFINITY || lk == -INFINITY) ? 0.f : exp2f(lk - mx);
                wsum += w;
                wt[i * kMlaHeads + ts] = w;
              }
              misc->inv_l[ts] = wsum > 0.f ? 1.f / wsum : 0.f;
              Lout[ts] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
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
                reinterpret_cast<float4*>(Oout + (size_t)r * kMlaDv)[ch] =
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
              float4* out = reinterpret_cast<float4*>(Oout + (size_t)r * kMlaDv) + lane * 4;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                out[i] = make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
              if (lane == 0) Lout[r] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
            }
          }
          if (ts == 0) *ctr = 0;  // ready for the next call
        }
      }
      pre += n;
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
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.q_len = d.q_len;
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
      if (encode_tiled_2d(&p.kvmap[si], set.pool[si], kMlaDqk, rows, kMlaDqk * 2, 64, 64) != CUDA_SUCCESS)
        return DCP_ERR_CUDA;
    }
  }
  auto kern = d.shard_rule == DCP_SHARD_INTERLEAVED ? mla_decode_kernel<0> : mla_decode_kernel<1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMlaSmem) != cudaSuccess)
    return DCP_ERR_CUDA;
  kern<<<dim3(L.nctas, d.q_len), kMlaThreads, kMlaSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

}  // namespace dcp
