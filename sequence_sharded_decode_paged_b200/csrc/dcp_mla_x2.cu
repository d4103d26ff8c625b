// dcp_mla_x2.cu -- MLA partial decode attention on CTA pairs (thread-block clusters of two).
//
// What it computes is the MLA partial of "Efficient Decode Context Parallelism
// with vLLM for Long Context Workloads" (A2 方法细节: one latent vector per token
// shared by every query head; DCP splits the latent cache along the sequence):
// for every shard s, request b and head h (64 heads),
//   s_t = scale * q[b][h] . C_t,  O_s[b][h] = sum_t softmax(s)_t * C_t[0:512],  LSE_s[b][h],
// over the tokens of b that shard s stores -- the same result as the one-CTA kernel.
//
// Why two CTAs: with 64 heads the products are narrow (N = 64) and the value
// operand of PV is MN-major, so on one SM a 128-token pair costs about 4,800
// tensor cycles, and the query tile (72 KB) leaves room for only one 144 KB pair
// stage -- load, S, softmax and PV of a pair then run one after the other.  Two
// CTAs on two SMs split the latent dims: CTA r of the cluster owns value dims
// 256r .. 256r + 255 and rope dims 512 + 32r .. + 31 of every token (and of the
// query), so its query slice is 36 KB, a pair stage 72 KB, and two stages fit:
// the next pair streams in while this one is computed.
//  * Each CTA computes the partial scores of its dims for all 64 heads:
//    S^T_r = K_r Q_r^T, tcgen05.mma M = 128 (the pair's tokens) N = 64 K = 288.
//  * The softmax is split by heads: CTA r owns heads 32r .. 32r + 31.  It sends
//    its partial scores of the partner's heads into the partner's shared memory
//    (16 KB per pair) and adds the partner's partial of its own heads, so each
//    head's scores are S_0 + S_1 in one place.
//  * Each CTA writes P^T of its own heads into both CTAs' P^T tiles, then both run
//    O^T_r += V_r^T P^T over their own value dims: two M = 128 tiles, K = 128.
//  * Rescale factors (when a head's integral reference maximum is raised) and the
//    final row sums are exchanged the same way; each CTA stores O for its value
//    dims, the owner of a head its LSE.
// All waits are bounded; every cross-CTA hand-off is an mbarrier arrival with
// release semantics at cluster scope, and no TMA load uses multicast.
#include <float.h>
#include <stddef.h>

#include "dcp_device.cuh"
#include "dcp_internal.h"
#include "dcp_tcgen05.cuh"

namespace dcp {

namespace {

constexpr int kX2Threads = 320;                        // producer warp, MMA warp, 8 softmax warps
constexpr int kHeads = 64;
constexpr int kDv = 512;
constexpr int kBs = 64;
constexpr int kOwnHeads = 32;                          // heads whose softmax a CTA owns
constexpr uint32_t kBox = 8192;                        // 64 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kHBox = 4096;                       // 64 rows x 32 bf16, 64-byte swizzle
constexpr uint32_t kPBox = 2 * kBox;                   // a pair box: page a rows 0-63, page b rows 64-127
constexpr uint32_t kPHBox = 2 * kHBox;                 // the pair's half rope box
constexpr uint32_t kStage = 4 * kPBox + kPHBox;        // 73,728: one pair, this CTA's 288 dims
constexpr uint32_t kQBytes = 4 * kBox + kHBox;         // 36,864: the query's 288 dims
constexpr uint32_t kPageBytes = 4 * kBox + kHBox;      // one page's 288 dims
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffSt = kQBytes;                   // two stages
constexpr uint32_t kOffPT = kOffSt + 2 * kStage;       // P^T: 128 tokens x 64 heads bf16 (MN-major, 16 KB)
constexpr uint32_t kOffXS = kOffPT + 16384;            // the partner's partial scores of my heads: [128][32] fp32
constexpr uint32_t kOffMisc = kOffXS + 16384;          // 217,088
constexpr uint32_t kMiscBytes = 4096;
constexpr int kCombineMax = 16;
constexpr uint32_t kOffW = kOffMisc + kMiscBytes;      // combine weights [piece][64]
constexpr uint32_t kX2Smem = kOffW + kCombineMax * 64 * 4;  // 225,280 bytes
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0;                          // O^T_r: 2 tiles x 64 columns
constexpr uint32_t kColS = 128;                        // S^T_r: 2 buffers x 64 columns
constexpr float kRescaleThreshold = 8.0f;              // log2 units
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = 8;
static_assert(kOffSt % 1024 == 0 && kOffPT % 1024 == 0, "swizzled tiles need 1024-byte alignment");

struct X2Misc {
  uint64_t q_full, q_empty, st_full[2], st_empty[2], s_full[2], s_empty[2];
  uint64_t xs_full, xs_free, pa_full, p_full, o_done, peer_done, o_free, l_full, slot_done, fin, mma_done;
  uint32_t tmem_base;
  int bcast;
  alignas(16) float mref[kOwnHeads];  // integral reference maxima (log2 units) of the own heads
  float alpha[2][kHeads];             // [pair parity][head]: factors of a raise (own heads: this CTA)
  int raised[2][2];                   // [pair parity][cluster rank]: pair index + 1 if that rank raised
  float inv_l[kHeads];                // own heads: this CTA; the partner's: written by the partner
  float lse2[kOwnHeads];
  float part[4][kOwnHeads];           // per-sub-partition partial maxima or sums
  int scratch[32];
};
static_assert(sizeof(X2Misc) <= kMiscBytes, "misc block");
static_assert(offsetof(X2Misc, mref) % 16 == 0, "float4 reads of the reference maxima");

struct X2Params {
  CUtensorMap kvmap[kMaxShards];   // 64 x 64 boxes, 128-byte swizzle
  CUtensorMap kvhmap[kMaxShards];  // 32 x 64 boxes, 64-byte swizzle (half rope)
  CUtensorMap qmap, qhmap;
  const int32_t* table[kMaxShards];
  float* O[kMaxShards];
  float* LSE[kMaxShards];
  int pool_pages[kMaxShards];
  int shard_of_si[kMaxShards];
  const int32_t* seq_lens;
  int* status;
  int* counters;  // [segment][q token][rank]
  float* slots;
  float scale_log2;
  int n_si, B, D, mlb, slot_floats, q_len;
  int Hk;
  size_t own_stride;
};

__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void wait_or_die(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  if (dead) return;
  if (!mbar_wait(bar, parity)) {
    atomicOr(status, kDevTimeout);
    dead = true;
  }
}

// A wait on a barrier that the partner CTA arrives on (acquire at cluster scope).
__device__ __forceinline__ void wait_cluster_or_die(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  if (dead) return;
  if (!mbar_wait_cluster(bar, parity)) {
    atomicOr(status, kDevTimeout);
    dead = true;
  }
}

// Warp-wide variants: the verdict is made uniform across the warp (warp-collective TMEM access follows).
__device__ __forceinline__ void wait_or_die_warp(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  wait_or_die(bar, parity, dead, status);
  dead = __any_sync(0xffffffffu, dead);
}
__device__ __forceinline__ void wait_cluster_or_die_warp(uint64_t* bar, uint32_t parity, bool& dead, int* status) {
  wait_cluster_or_die(bar, parity, dead, status);
  dead = __any_sync(0xffffffffu, dead);
}

__device__ __forceinline__ bool page_ok(const X2Params& p, int si, int b, int j, int* page_out) {
  // a local block past the table row is treated like an out-of-pool page: never read, flagged
  const int page = j < p.mlb ? p.table[si][(size_t)b * p.mlb + j] : -1;
  *page_out = page;
  return page >= 0 && page < p.pool_pages[si];
}

// v[i] reduced over the 32 lanes for i = 0..15, transposed: lane l returns index l & 15 (the
// halves exchange 8, 4, 2, 1 values, then the two half-warps combine).
template <bool MAX>
__device__ __forceinline__ float warp_transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int k = 8; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = upper ? v[i] : v[i + k];
      const float keep = upper ? v[i + k] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, k);
      v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float o = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return MAX ? fmaxf(v[0], o) : v[0] + o;
}

}  // namespace

// RULE: the shard rule (0 interleaved, 1 contiguous chunks).
template <int RULE>
__global__ void __launch_bounds__(kX2Threads, 1) mla_x2_kernel(const __grid_constant__ X2Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  X2Misc* misc = reinterpret_cast<X2Misc*>(smem + kOffMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;  // cluster index and count (the range owner)
  const int jq = blockIdx.y, ql = p.q_len;
  const int B = p.B, D = p.D;
  const bool aligned = (smem_u32(smem) & 1023u) == 0u;  // the same in both CTAs

  if (tid == 0 && aligned) {
    mbar_init(&misc->q_full, 1);
    mbar_init(&misc->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&misc->st_full[i], 1);
      mbar_init(&misc->st_empty[i], 1);
      mbar_init(&misc->s_full[i], 1);
      mbar_init(&misc->s_empty[i], kSoftmaxWarps);
    }
    mbar_init(&misc->xs_full, kSoftmaxWarps);
    mbar_init(&misc->xs_free, kSoftmaxWarps);
    mbar_init(&misc->pa_full, kSoftmaxWarps);
    mbar_init(&misc->p_full, kSoftmaxWarps);
    mbar_init(&misc->o_done, 1);
    mbar_init(&misc->peer_done, 1);
    mbar_init(&misc->o_free, kSoftmaxWarps);
    mbar_init(&misc->l_full, kSoftmaxWarps);
    mbar_init(&misc->slot_done, kSoftmaxWarps);
    mbar_init(&misc->fin, 1);
    mbar_init(&misc->mma_done, 1);
    for (int i = 0; i < 4; ++i) misc->raised[i >> 1][i & 1] = 0;
    fence_barrier_init();
  }
  if (warp == 1 && aligned) {
    tmem_alloc(&misc->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // both CTAs' barriers exist before either arrives on the other's (the only cluster-wide
  // barrier; every thread of both CTAs reaches it)
  cluster_sync_all();
  tc_fence_after();
  if (!aligned) {
    if (tid == 0) atomicOr(p.status, kDevTimeout);
    return;
  }
  const uint32_t tbase = misc->tmem_base;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.qmap);
    prefetch_tmap(&p.qhmap);
    for (int si = 0; si < p.n_si; ++si)
      if (p.pool_pages[si] > 0) {
        prefetch_tmap(&p.kvmap[si]);
        prefetch_tmap(&p.kvhmap[si]);
      }
  }

  // both CTAs of a cluster work on the same page range (the cluster's)
  const CtaPlan plan = plan_cta_r<RULE>(p.seq_lens, B, p.n_si, p.shard_of_si, kBs, D, cl, ncl, misc->scratch);
  const int T = plan.T, P = plan.P;
  const int lo = cl * P, hi = min(lo + P, T);
  const int S = p.n_si * B;
  const int vbox0 = 4 * (int)rank;      // first value box (64 dims) of this CTA
  const int rope_x = 512 + 32 * (int)rank;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t q_ph = 0;
      long pc = 0;
      bool dead = false, q_issued = false;
      int pre = plan.pre0;
      for (int sid = plan.sid0; sid < S && !dead; ++sid) {
        const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
        const int n = local_pages_r<RULE>(p.seq_lens[b], kBs, D, shard);
        if (seg_first_cta(pre, n, T, P) > cl) break;
        const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
        pre += n;
        if (n == 0) continue;
        wait_or_die(&misc->q_empty, q_ph ^ 1u, dead, p.status);
        q_ph ^= 1u;
        if (dead) break;
        mbar_arrive_expect_tx(&misc->q_full, kQBytes);
        const int qrow = (b * ql + jq) * kHeads;
        for (int i = 0; i < 4; ++i) tma_load_2d(smem + kOffQ + i * kBox, &p.qmap, (vbox0 + i) * 64, qrow, &misc->q_full);
        tma_load_2d(smem + kOffQ + 4 * kBox, &p.qhmap, rope_x, qrow, &misc->q_full);
        q_issued = true;
        for (int j = a; j < e && !dead; j += 2) {
          int pa = -1, pb = -1;
          const bool oka = page_ok(p, si, b, j, &pa);
          const bool two = j + 1 < e;
          const bool okb = two && page_ok(p, si, b, j + 1, &pb);
          if (!oka || (two && !okb)) atomicOr(p.status, kDevBadPage);
          const uint32_t st = (uint32_t)(pc & 1);
          wait_or_die(&misc->st_empty[st], (uint32_t)((pc >> 1) & 1) ^ 1u, dead, p.status);
          if (dead) break;
          const uint32_t bytes = kPageBytes * ((oka ? 1u : 0u) + (okb ? 1u : 0u));
          uint8_t* dst = smem + kOffSt + st * kStage;
          if (bytes == 0) {
            mbar_arrive(&misc->st_full[st]);
          } else {
            mbar_arrive_expect_tx(&misc->st_full[st], bytes);
            for (int i = 0; i < 4; ++i) {
              if (oka) tma_load_2d(dst + i * kPBox, &p.kvmap[si], (vbox0 + i) * 64, pa * kBs, &misc->st_full[st]);
              if (okb) tma_load_2d(dst + i * kPBox + kBox, &p.kvmap[si], (vbox0 + i) * 64, pb * kBs, &misc->st_full[st]);
            }
            if (oka) tma_load_2d(dst + 4 * kPBox, &p.kvhmap[si], rope_x, pa * kBs, &misc->st_full[st]);
            if (okb) tma_load_2d(dst + 4 * kPBox + kHBox, &p.kvhmap[si], rope_x, pb * kBs, &misc->st_full[st]);
          }
          ++pc;
        }
      }
      // never leave with a copy into shared memory in flight: the last two stages, the query
      for (long i = pc > 2 ? pc - 2 : 0; i < pc; ++i) {
        bool d2 = false;
        wait_or_die(&misc->st_full[i & 1], (uint32_t)((i >> 1) & 1), d2, p.status);
      }
      if (q_issued) {
        bool d2 = false;
        wait_or_die(&misc->q_full, q_ph ^ 1u, d2, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Two cursors: S^T of pair js (as soon as its stage, its S buffer and -- for a
    // piece's first pair -- the query are there) and PV of pair jo < js (once both
    // halves of P^T are in place), PV first: it frees a stage.
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 64, false, false);
      const uint32_t idO = idesc_bf16_f32(128, 64, true, true);
      struct PairRec {
        bool two, first, last;
      };
      PairRec ring[4];
      uint32_t q_ph = 0, of_ph = 0;
      long js = 0, jo = 0, known = 0;
      bool dead = false;
      int w_sid = plan.sid0, w_pre = plan.pre0, w_j = 0, w_e = 0, w_a = 0;
      bool w_live = true;
      auto enumerate = [&]() {
        while (w_live) {
          if (w_j < w_e) {
            PairRec r;
            r.two = w_j + 1 < w_e;
            r.first = w_j == w_a;
            r.last = w_j + 2 >= w_e;
            ring[known & 3] = r;
            ++known;
            w_j += 2;
            return;
          }
          if (w_sid >= S) {
            w_live = false;
            break;
          }
          const int si2 = w_sid / B, b2 = w_sid - si2 * B;
          const int n2 = local_pages_r<RULE>(p.seq_lens[b2], kBs, D, p.shard_of_si[si2]);
          if (seg_first_cta(w_pre, n2, T, P) > cl) {
            w_live = false;
            break;
          }
          w_a = w_j = max(w_pre, lo) - w_pre;
          w_e = n2 > 0 ? min(w_pre + n2, hi) - w_pre : 0;
          w_pre += n2;
          ++w_sid;
        }
      };
      unsigned long long idle_since = 0;
      while (!dead) {
        if (known == js) enumerate();
        bool progressed = false;
        if (jo < js && mbar_test(&misc->p_full, (uint32_t)(jo & 1))) {
          const PairRec r = ring[jo & 3];
          if (r.first) {  // the previous piece's epilogue must have read O^T
            wait_or_die(&misc->o_free, of_ph ^ 1u, dead, p.status);
            of_ph ^= 1u;
          }
          if (!dead) {
            tc_fence_after();
            const uint32_t st = (uint32_t)(jo & 1);
            // V^T: MN-major, 64-dim atoms one pair box apart; P^T: MN-major, one 64-head atom
            const uint64_t bd = sw128_desc(smem_u32(smem + kOffPT), kPBox, 1024);
            const int kst = r.two ? 8 : 4;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              const uint64_t ad = sw128_desc(smem_u32(smem + kOffSt + st * kStage + 2 * mt * kPBox), kPBox, 1024);
              for (int ks = 0; ks < kst; ++ks)
                umma_bf16(tbase + kColO + mt * 64, ad + (uint64_t)((ks * 2048) >> 4), bd + (uint64_t)((ks * 2048) >> 4),
                          idO, (!r.first || ks > 0) ? 1u : 0u);
            }
            umma_commit(&misc->st_empty[st]);  // the stage is free (its S^T is long done)
            umma_commit(&misc->o_done);
            umma_commit_multicast(&misc->peer_done, (uint16_t)(1u << peer));  // the partner may refill my P^T
            ++jo;
            progressed = true;
          }
        }
        if (!dead && js < known && js - jo < 2) {
          const PairRec r = ring[js & 3];
          const uint32_t st = (uint32_t)(js & 1), par = (uint32_t)((js >> 1) & 1);
          const bool ready = (!r.first || mbar_test(&misc->q_full, q_ph)) && mbar_test(&misc->st_full[st], par) &&
                             mbar_test(&misc->s_empty[st], par ^ 1u);
          if (ready) {
            if (r.first) q_ph ^= 1u;
            tc_fence_after();
            const uint32_t dS = tbase + kColS + st * 64;
            const uint8_t* sbase = smem + kOffSt + st * kStage;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint64_t ad = sw128_desc(smem_u32(sbase + i * kPBox), 16, 1024);
              const uint64_t bd = sw128_desc(smem_u32(smem + kOffQ + i * kBox), 16, 1024);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_bf16(dS, ad + (uint64_t)((ks * 32) >> 4), bd + (uint64_t)((ks * 32) >> 4), idS,
                          (i > 0 || ks > 0) ? 1u : 0u);
            }
            {  // half rope: 32 dims, 64-byte rows (8-row atoms of 512 bytes)
              const uint64_t ad = sw64_desc(smem_u32(sbase + 4 * kPBox), 16, 512);
              const uint64_t bd = sw64_desc(smem_u32(smem + kOffQ + 4 * kBox), 16, 512);
#pragma unroll
              for (int ks = 0; ks < 2; ++ks)
                umma_bf16(dS, ad + (uint64_t)((ks * 32) >> 4), bd + (uint64_t)((ks * 32) >> 4), idS, 1u);
            }
            umma_commit(&misc->s_full[st]);
            if (r.last) umma_commit(&misc->q_empty);  // Q is free once these products are done
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
    // Warp w reads TMEM sub-partition q4 = w % 4: lanes 32*q4 .. +31 = the pair's tokens 32*q4 ..
    // (page a below 64).  Half hf = (w - 2) / 4 owns the 16 heads own0 = 32*rank + 16*hf .. + 15
    // and sends the partner's 16 heads oth0 = 32*peer + 16*hf .. + 15.
    const int q4 = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int ts = tid - 64;  // 0..255
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const int tok = 32 * q4 + lane;
    const int slot = tok >> 6, trow = tok & 63;
    const int own0 = 32 * (int)rank + 16 * hf, oth0 = 32 * (int)peer + 16 * hf;
    // addresses in the partner's shared memory
    const uint32_t r_xs = map_to_rank(smem + kOffXS + (size_t)tok * 128 + 64 * hf, peer);
    const uint32_t r_pt = map_to_rank(smem + kOffPT + (size_t)tok * 128, peer);
    const uint32_t r_xs_full = map_to_rank(&misc->xs_full, peer);
    const uint32_t r_xs_free = map_to_rank(&misc->xs_free, peer);
    const uint32_t r_pa_full = map_to_rank(&misc->pa_full, peer);
    const uint32_t r_l_full = map_to_rank(&misc->l_full, peer);
    const uint32_t r_slot_done = map_to_rank(&misc->slot_done, peer);
    long pc = 0;
    int pieces = 0, cuts = 0;
    bool dead = false;
    int pre = plan.pre0;
    for (int sid = plan.sid0; sid < S; ++sid) {
      const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
      const int seq_len = p.seq_lens[b];
      const int n = local_pages_r<RULE>(seq_len, kBs, D, shard);
      const int c0 = seg_first_cta(pre, n, T, P);
      if (c0 > cl) break;
      const int c1 = seg_last_cta(pre, n, T, P);
      const size_t row0 = ((size_t)b * ql + jq) * p.Hk;
      auto o_row = [&](int h) -> float* {
        const int own = h / p.Hk;
        return p.O[si] + own * p.own_stride + (row0 + (h - own * p.Hk)) * kDv;
      };
      auto l_ptr = [&](int h) -> float* {
        const int own = h / p.Hk;
        return p.LSE[si] + own * p.own_stride + row0 + (h - own * p.Hk);
      };
      const int lim = seq_len - (ql - 1 - jq);
      const int g0 = global_block(0, seq_len, kBs, D, shard, RULE);
      const int gstride = RULE != 0 ? 1 : D;
      if (n == 0) {  // no token here: each CTA writes its value half and its heads' LSE
        for (int i = ts; i < kHeads * 64; i += kSoftmaxThreads)
          reinterpret_cast<float4*>(o_row(i >> 6) + 256 * rank)[i & 63] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ts < kOwnHeads) *l_ptr(32 * (int)rank + ts) = -INFINITY;
        pre += n;
        continue;
      }
      const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
      float l[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) l[i] = 0.f;
      if (ts < kOwnHeads) misc->mref[ts] = -INFINITY;
      named_bar_sync(2, kSoftmaxThreads);
      const float4* mref4 = reinterpret_cast<const float4*>(misc->mref + 16 * hf);
      for (int j = a; j < e; j += 2) {
        const bool two = j + 1 < e;
        int pa = -1, pb = -1;
        const bool oka = page_ok(p, si, b, j, &pa);
        const bool okb = two && page_ok(p, si, b, j + 1, &pb);
        const int tok0a = (g0 + j * gstride) * kBs, tok0b = (g0 + (j + 1) * gstride) * kBs;
        const bool visible = (slot == 0 ? oka : okb) && trow < lim - (slot == 0 ? tok0a : tok0b);
        const uint32_t sb = (uint32_t)(pc & 1);
        const uint32_t pp = (uint32_t)(pc & 1);  // parity of the per-pair barriers
        // 1. this CTA's partial scores: the partner's heads (to send) and its own
        wait_or_die_warp(&misc->s_full[sb], (uint32_t)((pc >> 1) & 1), dead, p.status);
        tc_fence_after();
        float snd[16], s[16];
        if (!dead) {
          tmem_ld16(tbase + lane_off + kColS + sb * 64 + oth0, snd);
          tmem_ld16(tbase + lane_off + kColS + sb * 64 + own0, s);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->s_empty[sb]);
        // 2. send the partner its heads' partial (its buffer must be free: it read the last one)
        if (pc > 0) wait_or_die_warp(&misc->xs_free, (uint32_t)((pc - 1) & 1), dead, p.status);
        if (!dead) {
#pragma unroll
          for (int c = 0; c < 4; ++c) st_cluster_v4(r_xs + 16 * c, snd[4 * c], snd[4 * c + 1], snd[4 * c + 2], snd[4 * c + 3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(r_xs_full);
        // 3. add the partner's partial of my heads: s = S_own + S_partner
        wait_cluster_or_die_warp(&misc->xs_full, pp, dead, p.status);
        if (!dead) {
          const float4* xs = reinterpret_cast<const float4*>(smem + kOffXS + (size_t)tok * 128 + 64 * hf);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float4 x = xs[c];
            s[4 * c] += x.x;
            s[4 * c + 1] += x.y;
            s[4 * c + 2] += x.z;
            s[4 * c + 3] += x.w;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(r_xs_free);
        // 4. scaled scores, masking, and whether some head's reference must be raised
        bool raise = false;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 m4 = mref4[i4];
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = 4 * i4 + k;
            s[i] = (visible && !dead) ? s[i] * p.scale_log2 : -INFINITY;
            raise = raise || s[i] > mm[k] + kRescaleThreshold;
          }
        }
        if (bar_red_or(2, kSoftmaxThreads, raise)) {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = s[i];
          const float pm_l = warp_transpose_reduce16<true>(v, lane);  // head 16*hf + (lane & 15)
          if (lane < 16) misc->part[q4][16 * hf + lane] = pm_l;
          named_bar_sync(2, kSoftmaxThreads);
          if (ts < kOwnHeads) {
            const float pm = fmaxf(fmaxf(misc->part[0][ts], misc->part[1][ts]), fmaxf(misc->part[2][ts], misc->part[3][ts]));
            const float mo = misc->mref[ts];
            float mn = mo;
            if (mo == -INFINITY || pm > mo + kRescaleThreshold) mn = ceilf(pm);
            const float al = mn == mo ? 1.f : exp2_int(mo - mn);
            misc->mref[ts] = mn;
            const int h = 32 * (int)rank + ts;
            misc->alpha[pp][h] = al;
            st_cluster_f32(map_to_rank(&misc->alpha[pp][h], peer), al);
            if (ts == 0) {
              misc->raised[pp][rank] = (int)pc + 1;
              st_cluster_s32(map_to_rank(&misc->raised[pp][rank], peer), (int)pc + 1);
            }
          }
          named_bar_sync(2, kSoftmaxThreads);
#pragma unroll
          for (int i = 0; i < 16; ++i) l[i] *= misc->alpha[pp][own0 + i];
        }
        // 5. zero this CTA's value rows past the sequence end (stale values must not meet zero weights)
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          const bool okx = x == 0 ? oka : okb;
          const int valid = min(kBs, seq_len - (x == 0 ? tok0a : tok0b));
          if (!okx || dead || valid >= kBs) continue;
          const int nchunks = (kBs - valid) * 32;  // rows x (4 boxes x 8 chunks)
          for (int i = ts; i < nchunks; i += kSoftmaxThreads) {
            const int row = valid + (i >> 5), cb = (i >> 3) & 3, ch = i & 7;
            *reinterpret_cast<uint4*>(smem + kOffSt + (pc & 1) * kStage + cb * kPBox + x * kBox + row * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        // 6. weights and running sums of my heads; my 16 heads' P^T chunks (two of the row's
        //    eight 16-byte chunks) into both CTAs' P^T tiles
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 m4 = mref4[i4];
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = 4 * i4 + k;
            s[i] = ex2_approx(s[i] - (mm[k] == -INFINITY ? 0.f : mm[k]));
            l[i] += s[i];
          }
        }
        const uint4 w0 = make_uint4(pack_bf16x2(s[0], s[1]), pack_bf16x2(s[2], s[3]), pack_bf16x2(s[4], s[5]),
                                    pack_bf16x2(s[6], s[7]));
        const uint4 w1 = make_uint4(pack_bf16x2(s[8], s[9]), pack_bf16x2(s[10], s[11]), pack_bf16x2(s[12], s[13]),
                                    pack_bf16x2(s[14], s[15]));
        const uint32_t c0x = (((uint32_t)(own0 >> 3)) ^ (uint32_t)(tok & 7)) << 4;
        const uint32_t c1x = (((uint32_t)((own0 >> 3) + 1)) ^ (uint32_t)(tok & 7)) << 4;
        if (pc > 0) wait_or_die_warp(&misc->o_done, (uint32_t)((pc - 1) & 1), dead, p.status);  // my P^T is free
        if (!dead) {
          uint8_t* prow = smem + kOffPT + tok * 128;
          *reinterpret_cast<uint4*>(prow + c0x) = w0;
          *reinterpret_cast<uint4*>(prow + c1x) = w1;
        }
        if (pc > 0) wait_cluster_or_die_warp(&misc->peer_done, (uint32_t)((pc - 1) & 1), dead, p.status);  // the partner's
        if (!dead) {
          st_cluster_u4(r_pt + c0x, w0);
          st_cluster_u4(r_pt + c1x, w1);
        }
        fence_proxy_async_cluster();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(r_pa_full);
        // 7. the partner's half of P^T and its rescale factors are here: rescale O^T if a raise
        //    happened on either side (not on a piece's first pair: O^T holds nothing yet)
        wait_cluster_or_die_warp(&misc->pa_full, pp, dead, p.status);
        const bool r0 = misc->raised[pp][0] == (int)pc + 1, r1 = misc->raised[pp][1] == (int)pc + 1;
        bool resc = false;
        if (j > a && (r0 || r1)) {
          bool changed = false;
          if (ts < kHeads) changed = (ts < 32 ? r0 : r1) && misc->alpha[pp][ts] != 1.f;
          resc = bar_red_or(2, kSoftmaxThreads, changed);
        }
        if (resc && !dead) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 64; c += 32) {
            float v[32];
            const uint32_t ta = tbase + lane_off + kColO + hf * 64 + c;
            tmem_ld32(ta, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int h = c + i;
              v[i] *= ((h < 32 ? r0 : r1) ? misc->alpha[pp][h] : 1.f);
            }
            tmem_st32(ta, v);
          }
          tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->p_full);
        ++pc;
      }
      // ---------------------------------------------------------- epilogue
      wait_or_die_warp(&misc->o_done, (uint32_t)((pc - 1) & 1), dead, p.status);  // the piece's last PV
      tc_fence_after();
      {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = l[i];
        const float ls = warp_transpose_reduce16<false>(v, lane);
        if (lane < 16) misc->part[q4][16 * hf + lane] = ls;
      }
      named_bar_sync(2, kSoftmaxThreads);
      if (ts < kOwnHeads) {
        const float lt = (misc->part[0][ts] + misc->part[1][ts]) + (misc->part[2][ts] + misc->part[3][ts]);
        const float il = lt > 0.f ? 1.f / lt : 0.f;
        const int h = 32 * (int)rank + ts;
        misc->inv_l[h] = il;
        misc->lse2[ts] = lt > 0.f ? misc->mref[ts] + __log2f(lt) : -INFINITY;
        st_cluster_f32(map_to_rank(&misc->inv_l[h], peer), il);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(r_l_full);
      wait_cluster_or_die_warp(&misc->l_full, (uint32_t)(pieces & 1), dead, p.status);
      named_bar_sync(2, kSoftmaxThreads);
      ++pieces;
      const bool complete = (c0 == c1);
      const int slot_i = complete ? 0 : 2 * cl + ((cl == c0 && pre != c0 * P) ? 1 : 0);
      float* slot_base = p.slots + ((size_t)slot_i * ql + jq) * p.slot_floats;
      {
        // O^T_r tile hf: lanes = value dims 256*rank + 128*hf + 32*q4 + lane, columns = heads
        const int dv = 256 * (int)rank + 128 * hf + 32 * q4 + lane;
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          float v[32];
          if (!dead) {
            tmem_ld32(tbase + lane_off + kColO + hf * 64 + c, v);
            tmem_ld_wait();
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float inv = misc->inv_l[c + i];
            float* dst = complete ? o_row(c + i) : slot_base + (size_t)(c + i) * kDv;
            dst[dv] = (inv == 0.f || dead) ? 0.f : v[i] * inv;
          }
        }
      }
      if (ts < kOwnHeads) {
        const int h = 32 * (int)rank + ts;
        if (complete) *l_ptr(h) = misc->lse2[ts] * kLn2;
        else slot_base[kHeads * kDv + h] = misc->lse2[ts];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&misc->o_free);
      if (!complete) {
        // both CTAs' parts of this piece are written before either counts it
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(r_slot_done);
        wait_cluster_or_die_warp(&misc->slot_done, (uint32_t)(cuts & 1), dead, p.status);
        ++cuts;
        named_bar_sync(2, kSoftmaxThreads);
        __threadfence();
        int* ctr = p.counters + ((size_t)sid * ql + jq) * 2 + rank;
        if (ts == 0) misc->bcast = (atomicAdd(ctr, 1) == c1 - c0) ? 1 : 0;
        named_bar_sync(2, kSoftmaxThreads);
        if (misc->bcast) {
          // the last of this rank's CTAs on the segment merges this rank's value half of all
          // pieces (every piece's LSE of all 64 heads is in place: see above)
          __threadfence();
          const int np = c1 - c0 + 1;
          float* wt = reinterpret_cast<float*>(smem + kOffW);  // [piece][head]
          const int npc = np <= kCombineMax ? np : kCombineMax;
          // maxima and sums first (one thread per head), then the value half chunk by chunk
          float* mxs = &misc->part[0][0];  // per-head maximum of the merge (64 floats)
          float mx_h = -INFINITY, ws_h = 0.f;
          if (ts < kHeads) {
            for (int c = c0; c <= c1; ++c) {
              const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
              mx_h = fmaxf(mx_h, __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kHeads * kDv + ts));
            }
            for (int c = c0; c <= c1; ++c) {
              const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
              const float lk = __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kHeads * kDv + ts);
              ws_h += (mx_h == -INFINITY || lk == -INFINITY) ? 0.f : exp2f(lk - mx_h);
            }
            mxs[ts] = mx_h;
            misc->inv_l[ts] = ws_h > 0.f ? 1.f / ws_h : 0.f;
            if ((ts >> 5) == (int)rank) *l_ptr(ts) = ws_h > 0.f ? (mx_h + __log2f(ws_h)) * kLn2 : -INFINITY;
          }
          named_bar_sync(2, kSoftmaxThreads);
          // 64 heads x 64 float4 chunks of this rank's value half
          const int ch = ts & 63, rq = ts >> 6;  // chunk, and heads rq, rq + 4, ...
          for (int cbase = c0; cbase <= c1; cbase += npc) {
            const int cend = min(c1 + 1, cbase + npc);
            if (ts < kHeads) {
              for (int c = cbase; c < cend; ++c) {
                const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                const float lk = __ldcg(p.slots + ((size_t)k * ql + jq) * p.slot_floats + kHeads * kDv + ts);
                const float mx = mxs[ts];
                wt[(c - cbase) * kHeads + ts] = (mx == -INFINITY || lk == -INFINITY) ? 0.f : exp2f(lk - mx);
              }
            }
            named_bar_sync(2, kSoftmaxThreads);
#pragma unroll 1
            for (int u0 = 0; u0 < kHeads / 4; u0 += 8) {
              float4 acc[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int h = rq + 4 * (u0 + u);
                acc[u] = (cbase == c0) ? make_float4(0.f, 0.f, 0.f, 0.f)
                                       : reinterpret_cast<const float4*>(o_row(h) + 256 * rank)[ch];
              }
#pragma unroll 2
              for (int c = cbase; c < cend; ++c) {
                const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
                const float* sl = p.slots + ((size_t)k * ql + jq) * p.slot_floats + 256 * rank;
                float4 x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  x[u] = __ldcg(reinterpret_cast<const float4*>(sl + (size_t)(rq + 4 * (u0 + u)) * kDv) + ch);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const float w = wt[(c - cbase) * kHeads + rq + 4 * (u0 + u)];
                  acc[u].x += w * x[u].x;
                  acc[u].y += w * x[u].y;
                  acc[u].z += w * x[u].z;
                  acc[u].w += w * x[u].w;
                }
              }
              const bool last = cend == c1 + 1;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int h = rq + 4 * (u0 + u);
                const float inv = last ? misc->inv_l[h] : 1.f;
                reinterpret_cast<float4*>(o_row(h) + 256 * rank)[ch] =
                    make_float4(acc[u].x * inv, acc[u].y * inv, acc[u].z * inv, acc[u].w * inv);
              }
            }
            named_bar_sync(2, kSoftmaxThreads);
          }
          if (ts == 0) *ctr = 0;  // ready for the next call
        }
      }
      pre += n;
    }
  }

  // ---------------------------------------------------------------- end: release TMEM; no CTA
  // leaves while its partner may still write into its shared memory
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_remote(map_to_rank(&misc->fin, peer));
    bool d2 = false;
    wait_cluster_or_die(&misc->fin, 0, d2, p.status);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------- host side
namespace {

template <int RULE>
int x2_clusters(int q_len) {
  // clusters of two that can be resident at once (a persistent grid must fit one wave)
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (cudaFuncSetAttribute(mla_x2_kernel<RULE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kX2Smem) !=
        cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1);
    cfg.blockDim = dim3(kX2Threads);
    cfg.dynamicSmemBytes = kX2Smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, mla_x2_kernel<RULE>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return 0;
    }
    cached[dev] = n;
  }
  const int n = cached[dev] / q_len;
  return n > 0 ? n : 0;
}

}  // namespace

// Clusters per query token that a launch uses (0: clusters of two cannot run here).
int mla_x2_clusters(const dcp_attn_desc& d) {
  return d.shard_rule == DCP_SHARD_INTERLEAVED ? x2_clusters<0>(d.q_len) : x2_clusters<1>(d.q_len);
}

dcp_status launch_mla_decode_x2(const dcp_attn_desc& d, int D, const ShardSet& set, const void* q,
                                const int32_t* seq_lens, void* ws, size_t ws_bytes, cudaStream_t stream) {
  WorkspaceLayout L;
  if (!workspace_layout(d, D, &L)) return DCP_ERR_UNSUPPORTED;
  if (ws_bytes < L.total) return DCP_ERR_CAPACITY;
  const int ncl = mla_x2_clusters(d);
  if (ncl <= 0 || ncl > L.nctas) return DCP_ERR_UNSUPPORTED;  // slots are sized for L.nctas ranges
  X2Params p;
  memset(&p, 0, sizeof(p));
  p.n_si = set.n;
  p.B = d.batch;
  p.D = D;
  p.mlb = d.max_local_blocks;
  p.slot_floats = L.slot_floats;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.q_len = d.q_len;
  p.Hk = set.owner_heads > 0 ? set.owner_heads : kHeads;
  p.own_stride = set.owner_stride;
  p.seq_lens = seq_lens;
  p.status = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.status_off);
  p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.counters_off);
  p.slots = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.slots_off);
  const uint64_t q_rows = (uint64_t)d.batch * d.q_len * kHeads;
  if (q_rows > (uint64_t)INT32_MAX) return DCP_ERR_UNSUPPORTED;
  if (encode_tiled_2d(&p.qmap, q, 576, q_rows, 576 * 2, 64, 64) != CUDA_SUCCESS) return DCP_ERR_CUDA;
  if (encode_tiled_2d_swizzle(&p.qhmap, q, 576, q_rows, 576 * 2, 32, 64, 2, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
    return DCP_ERR_CUDA;
  for (int si = 0; si < set.n; ++si) {
    p.table[si] = set.table[si];
    p.O[si] = set.O[si];
    p.LSE[si] = set.LSE[si];
    p.pool_pages[si] = set.pool_pages[si];
    p.shard_of_si[si] = set.shard[si];
    if (set.pool_pages[si] > 0) {
      const uint64_t rows = (uint64_t)set.pool_pages[si] * kBs;
      if (rows > (uint64_t)INT32_MAX) return DCP_ERR_UNSUPPORTED;
      if (encode_tiled_2d(&p.kvmap[si], set.pool[si], 576, rows, 576 * 2, 64, 64) != CUDA_SUCCESS) return DCP_ERR_CUDA;
      if (encode_tiled_2d_swizzle(&p.kvhmap[si], set.pool[si], 576, rows, 576 * 2, 32, 64, 2,
                                  CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
        return DCP_ERR_CUDA;
    }
  }
  auto kern = d.shard_rule == DCP_SHARD_INTERLEAVED ? mla_x2_kernel<0> : mla_x2_kernel<1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kX2Smem) != cudaSuccess)
    return DCP_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl, d.q_len);
  cfg.blockDim = dim3(kX2Threads);
  cfg.dynamicSmemBytes = kX2Smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return DCP_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

}  // namespace dcp
