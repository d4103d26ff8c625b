// dcp_gqa.cu -- GQA partial decode attention over D interleaved paged shards.
//
// What it computes ("Efficient Decode Context Parallelism with vLLM for Long
// Context Workloads", A2 方法细节, Compute step; "vLLM长序列推理优化：DCP切分KV
// Cache原理与实战" §2.2/§3.2 for the shard layout): for every shard s, request
// b and query head h, softmax attention of q[b][h] over the tokens of b that
// shard s stores, giving the normalised partial O_s[b][h] and LSE_s[b][h].
//
// Design (memory bound: 8 flop per KV byte at 8 query heads per KV head):
//  * Persistent CTAs.  The local page lists of all (shard, request) segments
//    are concatenated and cut into equal contiguous ranges, one per CTA, so
//    long and short requests balance exactly (flash-decoding split with no
//    fixed split size).  A segment cut by a range boundary is finished by the
//    last CTA to arrive on its counter (no spinning, no extra launch).
//  * One producer thread streams whole pages of the CTA's KV-head group into
//    a ring of shared-memory stages with 2-D TMA tiles (128-byte swizzle, no
//    multicast); K and V of all heads of one page arrive on one mbarrier.
//  * Eight consumer warps; each owns one KV head and one 16-row mma tile of
//    the R = q_len * G query rows sharing it (row r = query token r / G, head
//    r % G; R <= 16 is one tile per head).  Per 16-token chunk: S = Q K^T with
//    mma.m16n8k16 (K fragments by ldmatrix), online softmax in fp32 with quad
//    shuffles, P rounded to bf16 in registers and O += P V (V by
//    ldmatrix.trans).  Tokens past the sequence end are masked in both S and
//    the V fragments, so stale cache contents (even NaN) never leak in.
//  * Multi-token decode (q_len > 1): row r sees only the tokens before
//    seq_len - (q_len - 1 - r / G); the rest of its scores are masked.
//  * FP8 cache (KV8, head_dim 128 or 64): pages hold E4M3 codes, a 128-byte
//    (64-byte) row per token and head, so one swizzled box carries a head's K
//    (or V) block and a stage is half the size.  Codes convert exactly to f16 and the products
//    run as f16 mma.  K: each lane reads 4 consecutive codes of a token with
//    one 32-bit load; the query's dimensions are permuted the same way inside
//    each 16-wide k-tile (dims 4c..4c+3 play k = 2c, 2c+1, 2c+8, 2c+9).  V:
//    each lane reads 16 codes (dims 16g..16g+15) of tokens 2c, 2c+1, 2c+8 and
//    2c+9 with 16-byte loads and pairs them by byte permutes, so n-tile nt,
//    column n stands for dim 16n + nt; the output store undoes that order.
//    At head_dim 64 a lane reads 8 codes (dims 8g..8g+7, 8-byte loads) and
//    column n of n-tile nt stands for dim 8n + nt.
//    k_scale is folded into the score scale and v_scale into the final
//    normalisation.  The K products of a chunk run as four independent chains
//    (two token halves x two k halves) so that their latencies overlap.
#include <float.h>

#include <type_traits>

#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {

constexpr int kGqaConsumerWarps = 8;
// The producer is a whole warpgroup (one working thread) so that it can hand its registers to
// the two consumer warpgroups with setmaxnreg: at launch every thread has 168 registers (384
// threads, three warps on some SM sub-partition); the producer group drops to 40 and the
// consumers rise to 232, 4*40 + 8*232 = 12*168 per lane, so the split adds up to the launch's
// allocation.  (With nine warps the consumers stayed at 168 and the FP8 and draft variants
// spilled.)
constexpr int kGqaProducerWarps = 4;
constexpr int kGqaThreads = (kGqaConsumerWarps + kGqaProducerWarps) * 32;
constexpr int kGqaProducerRegs = 40, kGqaConsumerRegs = 232;
static_assert(kGqaProducerWarps * kGqaProducerRegs + kGqaConsumerWarps * kGqaConsumerRegs <=
                  (kGqaProducerWarps + kGqaConsumerWarps) * 168, "register split must fit the launch allocation");
constexpr int kScratchInts = 64;

constexpr float kLn2 = 0.69314718055994530942f;

struct GqaParams {
  CUtensorMap tmap[kMaxShards];
  const int32_t* table[kMaxShards];
  float* O[kMaxShards];
  float* LSE[kMaxShards];
  int pool_pages[kMaxShards];
  int shard_of_si[kMaxShards];
  const __nv_bfloat16* q;
  const int32_t* seq_lens;
  int* status;
  int* counters;
  float* slots;
  float scale_log2;
  float v_scale;  // multiplies O (FP8 cache); 1 for bf16
  int n_si, B, Hq, Hkv, G, bs, D, mlb;
  int q_len, R, rt;  // query tokens per request, rows per KV head (q_len * G), 16-row tiles per head
  int hpc, n_hg, stages, wph;
  uint32_t stage_bytes;
  int slot_floats;
  // Output layout: query heads are owned in consecutive slices of Hk heads; owner 0's O and
  // LSE rows start at O[si] / LSE[si], owner k's (k >= 1) at own_O[k] / own_L[k] (any address
  // this GPU can store to, a peer GPU's memory included).  The standard layout is Hk = Hq (a
  // single owner).
  int Hk;
  float* own_O[kMaxShards];
  float* own_L[kMaxShards];
};

// Output row of head-group row rr = h * R + r (KV head kv0 + h, local row r = query token
// r / G, head r % G) of request b, as (owner block, row within it): head = (kv0 + h) * G + r % G
// lies in owner block head / Hk at row (b * ql + r / G) * Hk + head % Hk.
struct OutRow {
  int own;
  size_t row;
};
__device__ __forceinline__ OutRow gqa_out_row(int rr, int b, int ql, int kv0, int G, int R, int Hk) {
  const int h = rr / R, r = rr - h * R, jq = r / G;
  const int head = (kv0 + h) * G + (r - jq * G);
  const int own = head / Hk;
  return {own, ((size_t)b * ql + jq) * Hk + (head - own * Hk)};
}
template <int HEAD_DIM>
__device__ __forceinline__ float* gqa_o_ptr(const GqaParams& p, int si, OutRow o) {
  return (o.own == 0 ? p.O[si] : p.own_O[o.own]) + o.row * HEAD_DIM;
}
__device__ __forceinline__ float* gqa_l_ptr(const GqaParams& p, int si, OutRow o) {
  return (o.own == 0 ? p.LSE[si] : p.own_L[o.own]) + o.row;
}

template <int HEAD_DIM, bool KV8>
struct GqaGeom {
  // swizzled boxes per row: 64 bf16 (128 bytes) each, or one box of the row's HEAD_DIM FP8 codes
  static constexpr int kBoxes = KV8 ? 1 : HEAD_DIM / 64;
  static constexpr int kBoxElems = KV8 ? HEAD_DIM : 64;
  static constexpr int kRowBytes = KV8 ? HEAD_DIM : 128;  // bytes of one token's row in a box
  static constexpr int kNTiles = HEAD_DIM / 8;  // n-tiles of O
  static constexpr int kKTiles = HEAD_DIM / 16; // k-tiles of Q K^T
  static constexpr int kCombineFloats = kNTiles * 4 + 4;  // per lane per warp
};

// ---- FP8 building blocks: one 16-token chunk of one KV head (128 or 64 dims) ----
// Byte offset of 16-byte chunk `chunk` of row `row` in a swizzled box of ROWB-byte rows (the
// 128-byte swizzle for 128-byte rows, the 64-byte swizzle for 64-byte rows).
template <int ROWB>
__device__ __forceinline__ uint32_t kv8_off(uint32_t row, uint32_t chunk) {
  if constexpr (ROWB == 128) return sw128(row, chunk);
  else return sw64(row, chunk);
}

// S (16 q rows x 16 tokens, f32) = Q K^T from E4M3 K rows at `kbase`, rows krow0 ..
// krow0 + 15 of the swizzled tile.  Lane (g, c) needs codes 4c..4c+3 of k-tile kt of
// tokens g and 8 + g: one ldmatrix (8 x 16-byte rows per matrix) gives that word for
// four (token half, k-tile) pairs -- tokens 0-7 / 8-15 of k-tiles kt and kt + 1.  Two
// accumulator sets (even / odd k-tiles) keep four independent product chains.
template <int KT>
__device__ __forceinline__ void kv8_scores(uint32_t kbase, uint32_t krow0, int lane, const uint32_t (&qa)[KT][4],
                                           float (&s)[2][4]) {
  constexpr int ROWB = KT * 16;  // one code per dim
  const uint32_t lrow = krow0 + (lane & 7) + (((lane >> 3) & 1) << 3);
  float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int kt = 0; kt < KT; kt += 2) {
    uint32_t w0, w1, w2, w3;  // (tokens 0-7, kt), (8-15, kt), (0-7, kt+1), (8-15, kt+1)
    ldsm_x4(kbase + kv8_off<ROWB>(lrow, (uint32_t)(kt + (lane >> 4))), w0, w1, w2, w3);
    uint32_t k0[2], k1[2], k2[2], k3[2];
    e4m3x4_to_f16x2x2(w0, k0[0], k0[1]);
    e4m3x4_to_f16x2x2(w1, k1[0], k1[1]);
    e4m3x4_to_f16x2x2(w2, k2[0], k2[1]);
    e4m3x4_to_f16x2x2(w3, k3[0], k3[1]);
    mma_f16_16816(s[0], qa[kt], k0[0], k0[1]);
    mma_f16_16816(s[1], qa[kt], k1[0], k1[1]);
    mma_f16_16816(s2[0], qa[kt + 1], k2[0], k2[1]);
    mma_f16_16816(s2[1], qa[kt + 1], k3[0], k3[1]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s[0][i] += s2[0][i];
    s[1][i] += s2[1][i];
  }
}

// O (16 q rows x 128 dims) += P V from E4M3 V rows at `vbase` (rows vrow0 .. vrow0 + 15).
// Lane (g, c) reads codes of dims 16g..16g+15 of tokens 2c, 2c+1 (b0) and 2c+8, 2c+9
// (b1) and pairs them by byte permutes, so n-tile nt, column n stands for dim 16n + nt.
// Tokens masked by keep0 / keep1 (tail chunks) get zero values.
template <int NT>
__device__ __forceinline__ void kv8_pv(uint32_t vbase, uint32_t vrow0, int g4, int c4, const uint32_t (&pa)[4],
                                       float (&o)[NT][4], bool tail, uint32_t keep0, uint32_t keep1) {
  const uint32_t vr = vrow0 + 2u * c4;
  if constexpr (NT == 8) {
    // head_dim 64: dims 8g..8g+7 (half g % 2 of the row's chunk g / 2); n-tile 4w + k, column n
    // stands for dim 8n + 4w + k
    const uint32_t off = (uint32_t)(g4 & 1) * 8u;
    const uint2 ta = lds64(vbase + kv8_off<64>(vr, (uint32_t)(g4 >> 1)) + off);
    const uint2 tb = lds64(vbase + kv8_off<64>(vr + 1u, (uint32_t)(g4 >> 1)) + off);
    const uint2 tc = lds64(vbase + kv8_off<64>(vr + 8u, (uint32_t)(g4 >> 1)) + off);
    const uint2 td = lds64(vbase + kv8_off<64>(vr + 9u, (uint32_t)(g4 >> 1)) + off);
    const uint32_t xa[2] = {ta.x, ta.y}, xb[2] = {tb.x, tb.y}, xc[2] = {tc.x, tc.y}, xd[2] = {td.x, td.y};
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      uint32_t b0[4], b1[4];
      e4m3x4_to_f16x2x2(__byte_perm(xa[w], xb[w], 0x5140), b0[0], b0[1]);
      e4m3x4_to_f16x2x2(__byte_perm(xa[w], xb[w], 0x7362), b0[2], b0[3]);
      e4m3x4_to_f16x2x2(__byte_perm(xc[w], xd[w], 0x5140), b1[0], b1[1]);
      e4m3x4_to_f16x2x2(__byte_perm(xc[w], xd[w], 0x7362), b1[2], b1[3]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (tail) {
          b0[k] &= keep0;
          b1[k] &= keep1;
        }
        mma_f16_16816(o[4 * w + k], pa, b0[k], b1[k]);
      }
    }
    return;
  }
  const uint4 ta = lds128(vbase + sw128(vr, (uint32_t)g4));
  const uint4 tb = lds128(vbase + sw128(vr + 1u, (uint32_t)g4));
  const uint4 tc = lds128(vbase + sw128(vr + 8u, (uint32_t)g4));
  const uint4 td = lds128(vbase + sw128(vr + 9u, (uint32_t)g4));
  const uint32_t xa[4] = {ta.x, ta.y, ta.z, ta.w}, xb[4] = {tb.x, tb.y, tb.z, tb.w};
  const uint32_t xc[4] = {tc.x, tc.y, tc.z, tc.w}, xd[4] = {td.x, td.y, td.z, td.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    // byte k of word w is dim 16g + 4w + k, i.e. n-tile 4w + k: pair the two tokens' codes
    uint32_t b0[4], b1[4];
    e4m3x4_to_f16x2x2(__byte_perm(xa[w], xb[w], 0x5140), b0[0], b0[1]);
    e4m3x4_to_f16x2x2(__byte_perm(xa[w], xb[w], 0x7362), b0[2], b0[3]);
    e4m3x4_to_f16x2x2(__byte_perm(xc[w], xd[w], 0x5140), b1[0], b1[1]);
    e4m3x4_to_f16x2x2(__byte_perm(xc[w], xd[w], 0x7362), b1[2], b1[3]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (tail) {
        b0[k] &= keep0;
        b1[k] &= keep1;
      }
      mma_f16_16816(o[4 * w + k], pa, b0[k], b1[k]);
    }
  }
}

// ---- bf16 building blocks: one 16-token chunk of one KV head ----
// S = Q K^T with K fragments by ldmatrix from the 128-byte swizzled boxes (64 dims each).
template <int KT>
__device__ __forceinline__ void bf16_scores(uint32_t kbase, uint32_t box_bytes, uint32_t krow0, int lane,
                                            const uint32_t (&qa)[KT][4], float (&s)[2][4]) {
  const uint32_t krow = krow0 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    const uint32_t chunk = (uint32_t)((kt & 3) * 2 + ((lane >> 3) & 1));
    uint32_t b00, b01, b10, b11;
    ldsm_x4(kbase + (kt >> 2) * box_bytes + sw128(krow, chunk), b00, b01, b10, b11);
    mma_bf16_16816(s[0], qa[kt], b00, b01);
    mma_bf16_16816(s[1], qa[kt], b10, b11);
  }
}

// O += P V with V fragments by ldmatrix.trans; tokens masked by keep0 / keep1 get zero values.
template <int NT>
__device__ __forceinline__ void bf16_pv(uint32_t vbase, uint32_t box_bytes, uint32_t vrow0, int lane,
                                        const uint32_t (&pa)[4], float (&o)[NT][4], bool tail, uint32_t keep0,
                                        uint32_t keep1) {
  const uint32_t vrow = vrow0 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
  for (int np = 0; np < NT / 2; ++np) {
    const uint32_t chunk = (uint32_t)((np & 3) * 2 + (lane >> 4));
    uint32_t v0, v1, v2, v3;
    ldsm_x4_t(vbase + (np >> 2) * box_bytes + sw128(vrow, chunk), v0, v1, v2, v3);
    if (tail) {
      v0 &= keep0;
      v1 &= keep1;
      v2 &= keep0;
      v3 &= keep1;
    }
    mma_bf16_16816(o[2 * np], pa, v0, v1);
    mma_bf16_16816(o[2 * np + 1], pa, v2, v3);
  }
}

__device__ __forceinline__ uint32_t keep_lo(int c4, int vrem) {  // tokens 2c, 2c+1 of a chunk
  return (c4 * 2 < vrem ? 0xFFFFu : 0u) | (c4 * 2 + 1 < vrem ? 0xFFFF0000u : 0u);
}
__device__ __forceinline__ uint32_t keep_hi(int c4, int vrem) {  // tokens 2c+8, 2c+9
  return (c4 * 2 + 8 < vrem ? 0xFFFFu : 0u) | (c4 * 2 + 9 < vrem ? 0xFFFF0000u : 0u);
}

// MULTI: multi-token decode (q_len > 1, per-row causal limits); the single-token
// instantiation keeps the plain end-of-sequence mask and its register budget.
// KV8: the pools hold FP8 E4M3 codes.  RULE: the shard rule (0 interleaved, 1 contiguous chunks).
template <int HEAD_DIM, bool MULTI, bool KV8, int RULE>
__global__ void __launch_bounds__(kGqaThreads, 1) gqa_decode_kernel(const __grid_constant__ GqaParams p) {
  using Geo = GqaGeom<HEAD_DIM, KV8>;
  static_assert(!KV8 || HEAD_DIM == 128 || HEAD_DIM == 64, "FP8 pages: one 128- or 64-byte row per token and head");
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stage_mem = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * p.stage_bytes);
  uint64_t* empty = full + p.stages;
  int* stage_ok = reinterpret_cast<int*>(empty + p.stages);
  int* scratch = stage_ok + 8;
  int* bcast = scratch + kScratchInts;
  float* combine = reinterpret_cast<float*>(bcast + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hg = blockIdx.y, cta = blockIdx.x, nctas = gridDim.x;
  const int B = p.B, bs = p.bs, D = p.D;
  const uint32_t box_bytes = (uint32_t)(p.hpc * bs * Geo::kRowBytes);

  if ((smem_u32(smem) & 1023u) != 0u) {  // swizzled TMA tiles need 1024-byte aligned stages
    if (tid == 0) atomicOr(p.status, kDevTimeout);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGqaConsumerWarps);
    }
    fence_barrier_init();
  }
  if (warp == kGqaConsumerWarps && lane == 0)
    for (int si = 0; si < p.n_si; ++si)
      if (p.pool_pages[si] > 0) prefetch_tmap(&p.tmap[si]);
  __syncthreads();

  const CtaPlan plan = plan_cta_r<RULE>(p.seq_lens, B, p.n_si, p.shard_of_si, bs, D, cta, nctas, scratch);
  const int T = plan.T, P = plan.P;
  const int lo = cta * P, hi = min(lo + P, T);
  const int S = p.n_si * B;

  // ------------------------------------------------------------------ producer
  if (warp >= kGqaConsumerWarps) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kGqaProducerRegs) : "memory");
    if (warp != kGqaConsumerWarps || lane != 0) return;
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool aborted = false;
    int pre = plan.pre0;
    for (int sid = plan.sid0; sid < S && !aborted; ++sid) {
      const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
      const int n = local_pages_r<RULE>(p.seq_lens[b], bs, D, shard);
      if (seg_first_cta(pre, n, T, P) > cta) break;
      const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;
      const int32_t* trow = p.table[si] + (size_t)b * p.mlb;
      for (int j = a; j < e; ++j) {
        // a local block past the table row (lengths grown beyond max_local_blocks) is
        // treated like an out-of-pool page: never read, flagged in the status word
        const int page = j < p.mlb ? trow[j] : -1;
        const bool ok = page >= 0 && page < p.pool_pages[si];
        if (!ok) atomicOr(p.status, kDevBadPage);
        if (!mbar_wait(&empty[stage], phase ^ 1u)) {
          atomicOr(p.status, kDevTimeout);
          aborted = true;
          break;
        }
        stage_ok[stage] = ok ? 1 : 0;
        if (ok) {
          mbar_arrive_expect_tx(&full[stage], p.stage_bytes);
          uint8_t* dst = stage_mem + (size_t)stage * p.stage_bytes;
          const int row_k = ((page * 2 + 0) * p.Hkv + hg * p.hpc) * bs;
          const int row_v = ((page * 2 + 1) * p.Hkv + hg * p.hpc) * bs;
#pragma unroll
          for (int bx = 0; bx < Geo::kBoxes; ++bx) {
            tma_load_2d(dst + bx * box_bytes, &p.tmap[si], bx * Geo::kBoxElems, row_k, &full[stage]);
            tma_load_2d(dst + (Geo::kBoxes + bx) * box_bytes, &p.tmap[si], bx * Geo::kBoxElems, row_v,
                        &full[stage]);
          }
        } else {
          mbar_arrive(&full[stage]);
        }
        ++issued;
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      pre += n;
    }
    // Never leave the CTA while a copy into its shared memory is in flight.
    const long first = issued > p.stages ? issued - p.stages : 0;
    for (long i = first; i < issued; ++i) {
      const int s = (int)(i % p.stages);
      const uint32_t par = (uint32_t)((i / p.stages) & 1);
      if (!mbar_wait(&full[s], par)) atomicOr(p.status, kDevTimeout);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kGqaConsumerRegs) : "memory");
  const int hpc = p.hpc, G = p.G, wph = p.wph, R = MULTI ? p.R : p.G, ql = MULTI ? p.q_len : 1;
  const int hu = MULTI ? hpc * p.rt : hpc;  // (KV head, row tile) units of one CTA; one tile if q_len = 1
  const bool active = warp < hu * wph;
  const int u = warp % hu, sub = warp / hu;
  const int hh = MULTI ? u % hpc : u, tile = MULTI ? u / hpc : 0;
  const int g4 = lane >> 2, c4 = lane & 3;
  const int rows_hg = hpc * R;  // rows of one head group: (head hh, row r) at hh * R + r
  int stage = 0;
  uint32_t phase = 0;
  int pre = plan.pre0;
  bool dead = false;

  for (int sid = plan.sid0; sid < S; ++sid) {
    const int si = sid / B, b = sid - si * B, shard = p.shard_of_si[si];
    const int seq_len = p.seq_lens[b];
    const int n = local_pages_r<RULE>(seq_len, bs, D, shard);
    // logical block of local page j: g0 + j * gstride (interleaved: shard + j * D; contiguous: chunk start + j)
    const int g0 = global_block(0, seq_len, bs, D, shard, RULE);
    const int gstride = RULE != 0 ? 1 : D;
    const int c0 = seg_first_cta(pre, n, T, P);
    if (c0 > cta) break;
    const int c1 = seg_last_cta(pre, n, T, P);
    if (n == 0) {  // no token of this request in this shard
      for (int i = tid; i < rows_hg * HEAD_DIM; i += kGqaConsumerWarps * 32)
        gqa_o_ptr<HEAD_DIM>(p, si, gqa_out_row(i / HEAD_DIM, b, ql, hg * hpc, G, R, p.Hk))[i % HEAD_DIM] = 0.f;
      for (int i = tid; i < rows_hg; i += kGqaConsumerWarps * 32)
        *gqa_l_ptr(p, si, gqa_out_row(i, b, ql, hg * hpc, G, R, p.Hk)) = -INFINITY;
      pre += n;
      continue;
    }
    const int a = max(pre, lo) - pre, e = min(pre + n, hi) - pre;

    // query fragments (16-row A tile; rows >= R are zero)
    uint32_t qa[Geo::kKTiles][4];
    const int kvh = hg * hpc + hh;
    int lim0 = seq_len, lim1 = seq_len;  // tokens each row may see
    {
      // this thread's two accumulator rows (r and r + 8 of the warp's tile), their query tokens
      const int r0 = tile * 16 + g4, r1 = r0 + 8;
      const bool row0 = active && r0 < R, row1 = active && r1 < R;
      const int j0 = (MULTI && row0) ? r0 / G : 0, j1 = (MULTI && row1) ? r1 / G : 0;
      const size_t q0 = (((size_t)b * ql + j0) * p.Hq + (size_t)kvh * G + (r0 - j0 * G)) * HEAD_DIM;
      const size_t q1 = (((size_t)b * ql + j1) * p.Hq + (size_t)kvh * G + (r1 - j1 * G)) * HEAD_DIM;
      const uint32_t* qb0 = reinterpret_cast<const uint32_t*>(p.q + (row0 ? q0 : 0));
      const uint32_t* qb1 = reinterpret_cast<const uint32_t*>(p.q + (row1 ? q1 : 0));
      if constexpr (KV8) {
        // f16 query, dims 16kt + 4c .. 4c+3 in the k slots 2c, 2c+1 (a0/a1) and 2c+8, 2c+9 (a2/a3)
#pragma unroll
        for (int kt = 0; kt < Geo::kKTiles; ++kt) {
          const int col = kt * 16 + c4 * 4;
          const uint2 x0 = row0 ? __ldg(reinterpret_cast<const uint2*>(qb0 + col / 2)) : make_uint2(0u, 0u);
          const uint2 x1 = row1 ? __ldg(reinterpret_cast<const uint2*>(qb1 + col / 2)) : make_uint2(0u, 0u);
          qa[kt][0] = bf16x2_to_f16x2(x0.x);
          qa[kt][1] = bf16x2_to_f16x2(x1.x);
          qa[kt][2] = bf16x2_to_f16x2(x0.y);
          qa[kt][3] = bf16x2_to_f16x2(x1.y);
        }
      } else {
#pragma unroll
        for (int kt = 0; kt < Geo::kKTiles; ++kt) {
          const int col = kt * 16 + c4 * 2;
          qa[kt][0] = row0 ? __ldg(qb0 + col / 2) : 0u;
          qa[kt][1] = row1 ? __ldg(qb1 + col / 2) : 0u;
          qa[kt][2] = row0 ? __ldg(qb0 + (col + 8) / 2) : 0u;
          qa[kt][3] = row1 ? __ldg(qb1 + (col + 8) / 2) : 0u;
        }
      }
      if (MULTI) {  // up to the row's own draft position
        lim0 = seq_len - (ql - 1 - j0);
        lim1 = seq_len - (ql - 1 - j1);
      }
    }
    float o[Geo::kNTiles][4];
#pragma unroll
    for (int i = 0; i < Geo::kNTiles; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    // One sum of the fp32 weights serves both the normalisation of O and the LSE, so
    // pieces of a split sequence merge back to exactly the unsplit result (up to
    // fp32 order); the PV product uses the same weights rounded to bf16.
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    int j = a;
    if constexpr (KV8 || MULTI) {
      // One warp per (head, row tile) and one chunk per page: two pages per step -- four
      // independent product chains and one softmax update per 32 tokens.  This hides the
      // latencies that leave a warp short of work when its chunk carries few bytes (FP8) or
      // its CTA streams few heads (several row tiles per head); single-token bf16 is HBM-bound
      // without it.
      if (wph == 1 && bs == 16) {
        // LO: rows 8..15 of the warp's tile are empty (single-token decode with G <= 8): their
        // maxima, weights, sums and rescales are skipped (zero weights, no ex2 issued).
        auto steps = [&](auto np_tag, auto lo_tag, int jj) {
          constexpr int NP = decltype(np_tag)::value;
          constexpr bool LO = decltype(lo_tag)::value;
          for (; jj + NP - 1 < e; jj += NP) {
            int st[NP];
            uint32_t ph[NP];
#pragma unroll
            for (int k = 0; k < NP; ++k) {
              st[k] = stage;
              ph[k] = phase;
              if (++stage == p.stages) {
                stage = 0;
                phase ^= 1u;
              }
            }
#pragma unroll
            for (int k = 0; k < NP; ++k)
              if (!dead && !mbar_wait(&full[st[k]], ph[k])) {
                atomicOr(p.status, kDevTimeout);
                dead = true;
              }
            if (!dead && active) {
              bool ok[NP];
              int vv[NP], t0[NP];
              uint32_t kb[NP];
              float sc[NP][2][4];
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                ok[k] = stage_ok[st[k]] != 0;
                t0[k] = (g0 + (jj + k) * gstride) * 16;
                vv[k] = min(16, seq_len - t0[k]);
                kb[k] = smem_u32(stage_mem + (size_t)st[k] * p.stage_bytes);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) sc[k][nt][0] = sc[k][nt][1] = sc[k][nt][2] = sc[k][nt][3] = 0.f;
              }
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                if constexpr (KV8) {
                  if (ok[k]) kv8_scores(kb[k], (uint32_t)(hh * 16), lane, qa, sc[k]);
                } else {
                  if (ok[k]) bf16_scores(kb[k], box_bytes, (uint32_t)(hh * 16), lane, qa, sc[k]);
                }
              }
              // visible tokens of each page for rows g4 / g4 + 8 (a page that was not loaded adds nothing)
              float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                const int w0 = !ok[k] ? 0 : (MULTI ? lim0 - t0[k] : vv[k]);
                const int w1 = !ok[k] ? 0 : (MULTI ? lim1 - t0[k] : vv[k]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                  for (int i = 0; i < (LO ? 2 : 4); ++i) {
                    const int tok = nt * 8 + c4 * 2 + (i & 1);
                    sc[k][nt][i] = tok < (i < 2 ? w0 : w1) ? sc[k][nt][i] * p.scale_log2 : -INFINITY;
                  }
                mx0 = fmaxf(mx0, fmaxf(fmaxf(sc[k][0][0], sc[k][0][1]), fmaxf(sc[k][1][0], sc[k][1][1])));
                if (!LO) mx1 = fmaxf(mx1, fmaxf(fmaxf(sc[k][0][2], sc[k][0][3]), fmaxf(sc[k][1][2], sc[k][1][3])));
              }
              mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
              mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
              if (!LO) {
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
              }
              const float mn0 = mx0 > m0 ? ceilf(mx0) : m0, mn1 = mx1 > m1 ? ceilf(mx1) : m1;
              const float al0 = exp2_int(m0 - mn0), al1 = exp2_int(m1 - mn1);
              m0 = mn0;
              m1 = mn1;
              const float sub0 = mn0 == -INFINITY ? 0.f : mn0, sub1 = mn1 == -INFINITY ? 0.f : mn1;
              float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
              for (int k = 0; k < NP; ++k) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                  sc[k][nt][0] = ex2_approx(sc[k][nt][0] - sub0);
                  sc[k][nt][1] = ex2_approx(sc[k][nt][1] - sub0);
                  sc[k][nt][2] = LO ? 0.f : ex2_approx(sc[k][nt][2] - sub1);
                  sc[k][nt][3] = LO ? 0.f : ex2_approx(sc[k][nt][3] - sub1);
                }
                ls0 += sc[k][0][0] + sc[k][0][1] + sc[k][1][0] + sc[k][1][1];
                if (!LO) ls1 += sc[k][0][2] + sc[k][0][3] + sc[k][1][2] + sc[k][1][3];
              }
              l0 = l0 * al0 + ls0;
              if (!LO) l1 = l1 * al1 + ls1;
              if (__any_sync(0xffffffffu, al0 != 1.f || (!LO && al1 != 1.f))) {
#pragma unroll
                for (int i = 0; i < Geo::kNTiles; ++i) {
                  o[i][0] *= al0;
                  o[i][1] *= al0;
                  if (!LO) {
                    o[i][2] *= al1;
                    o[i][3] *= al1;
                  }
                }
              }
              // values of tokens past the sequence end are zeroed (stale slots); causal masking
              // within the sequence is carried by P = 0
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                if (!ok[k]) continue;
                if constexpr (KV8) {
                  const uint32_t pa[4] = {pack_f16x2(sc[k][0][0], sc[k][0][1]), pack_f16x2(sc[k][0][2], sc[k][0][3]),
                                          pack_f16x2(sc[k][1][0], sc[k][1][1]), pack_f16x2(sc[k][1][2], sc[k][1][3])};
                  kv8_pv(kb[k] + Geo::kBoxes * box_bytes, (uint32_t)(hh * 16), g4, c4, pa, o, vv[k] < 16,
                         keep_lo(c4, vv[k]), keep_hi(c4, vv[k]));
                } else {
                  const uint32_t pa[4] = {pack_bf16x2(sc[k][0][0], sc[k][0][1]), pack_bf16x2(sc[k][0][2], sc[k][0][3]),
                                          pack_bf16x2(sc[k][1][0], sc[k][1][1]), pack_bf16x2(sc[k][1][2], sc[k][1][3])};
                  bf16_pv(kb[k] + Geo::kBoxes * box_bytes, box_bytes, (uint32_t)(hh * 16), lane, pa, o, vv[k] < 16,
                          keep_lo(c4, vv[k]), keep_hi(c4, vv[k]));
                }
              }
            }
            __syncwarp();
            if (lane == 0)
#pragma unroll
              for (int k = 0; k < NP; ++k) mbar_arrive(&empty[st[k]]);
          }
          return jj;
        };
        // two pages per step (four measured slower on the FP8 layer: 560 vs 497 us, fewer stages in flight)
        if (!MULTI && R <= 8) j = steps(std::integral_constant<int, 2>{}, std::true_type{}, j);
        else j = steps(std::integral_constant<int, 2>{}, std::false_type{}, j);
      }
    }
    for (; j < e; ++j) {
      // a wait that times out marks this warp dead: it stops waiting and computing
      // but keeps the block-wide barrier sequence, so nothing else can hang on it
      if (!dead && !mbar_wait(&full[stage], phase)) {
        atomicOr(p.status, kDevTimeout);
        dead = true;
      }
      if (!dead && active && ((j - a) % wph) == sub && stage_ok[stage]) {
        const int gblk = g0 + j * gstride;
        const int valid = min(bs, seq_len - gblk * bs);
        const uint32_t kbase = smem_u32(stage_mem + (size_t)stage * p.stage_bytes);
        const uint32_t vbase = kbase + Geo::kBoxes * box_bytes;
        for (int t0 = 0; t0 < valid; t0 += 16) {
          // ---- S = Q K^T for 16 tokens (two 8-token n-tiles)
          float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          if constexpr (KV8) {
            kv8_scores(kbase, (uint32_t)(hh * bs + t0), lane, qa, s);
          } else {
            bf16_scores(kbase, box_bytes, (uint32_t)(hh * bs + t0), lane, qa, s);
          }
          // ---- online softmax (log2 domain), rows g4 and g4 + 8
          const int vrem = valid - t0;
          const int vr0 = MULTI ? lim0 - (gblk * bs + t0) : vrem;
          const int vr1 = MULTI ? lim1 - (gblk * bs + t0) : vrem;
          if (MULTI || vrem < 16) {  // a chunk with masked tokens
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int tok = nt * 8 + c4 * 2 + (i & 1);
                s[nt][i] = tok < (i < 2 ? vr0 : vr1) ? s[nt][i] * p.scale_log2 : -INFINITY;
              }
          } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) s[nt][i] *= p.scale_log2;
          }
          float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
          float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
          // integral running maximum (exact power-of-two rescales, split-independent P)
          const float mn0 = mx0 > m0 ? ceilf(mx0) : m0, mn1 = mx1 > m1 ? ceilf(mx1) : m1;
          const float al0 = exp2_int(m0 - mn0), al1 = exp2_int(m1 - mn1);
          m0 = mn0;
          m1 = mn1;
          // a row that has seen no visible token yet keeps -inf: subtract 0 so exp2 gives 0
          // (single-token decode always has a visible token in every chunk it processes)
          const float sub0 = (MULTI && mn0 == -INFINITY) ? 0.f : mn0;
          const float sub1 = (MULTI && mn1 == -INFINITY) ? 0.f : mn1;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            s[nt][0] = ex2_approx(s[nt][0] - sub0);
            s[nt][1] = ex2_approx(s[nt][1] - sub0);
            s[nt][2] = ex2_approx(s[nt][2] - sub1);
            s[nt][3] = ex2_approx(s[nt][3] - sub1);
          }
          l0 = l0 * al0 + (s[0][0] + s[0][1] + s[1][0] + s[1][1]);
          l1 = l1 * al1 + (s[0][2] + s[0][3] + s[1][2] + s[1][3]);
          // the integral maximum rarely moves, so the rescale is usually a multiply by 1: skip it then
          if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
            for (int i = 0; i < Geo::kNTiles; ++i) {
              o[i][0] *= al0;
              o[i][1] *= al0;
              o[i][2] *= al1;
              o[i][3] *= al1;
            }
          }
          uint32_t pa[4];
          if constexpr (KV8) {
            pa[0] = pack_f16x2(s[0][0], s[0][1]);
            pa[1] = pack_f16x2(s[0][2], s[0][3]);
            pa[2] = pack_f16x2(s[1][0], s[1][1]);
            pa[3] = pack_f16x2(s[1][2], s[1][3]);
          } else {
            pa[0] = pack_bf16x2(s[0][0], s[0][1]);
            pa[1] = pack_bf16x2(s[0][2], s[0][3]);
            pa[2] = pack_bf16x2(s[1][0], s[1][1]);
            pa[3] = pack_bf16x2(s[1][2], s[1][3]);
          }
          // ---- O += P V; V fragments of tokens past the end are zeroed
          const bool tail = vrem < 16;
          const uint32_t keep0 = keep_lo(c4, vrem), keep1 = keep_hi(c4, vrem);
          if constexpr (KV8) {
            kv8_pv(vbase, (uint32_t)(hh * bs + t0), g4, c4, pa, o, tail, keep0, keep1);
          } else {
            bf16_pv(vbase, box_bytes, (uint32_t)(hh * bs + t0), lane, pa, o, tail, keep0, keep1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }

    // ---- finish the (warp-local) softmax state
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (wph > 1) {  // several warps shared this head: combine their states
      float* mine = combine + (size_t)warp * Geo::kCombineFloats * 32;
#pragma unroll
      for (int i = 0; i < Geo::kNTiles; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) mine[(i * 4 + k) * 32 + lane] = o[i][k];
      mine[(Geo::kNTiles * 4 + 0) * 32 + lane] = m0;
      mine[(Geo::kNTiles * 4 + 1) * 32 + lane] = m1;
      mine[(Geo::kNTiles * 4 + 2) * 32 + lane] = l0;
      mine[(Geo::kNTiles * 4 + 3) * 32 + lane] = l1;
      named_bar_sync(1, kGqaConsumerWarps * 32);
      if (active && sub == 0) {
        for (int w2 = 1; w2 < wph; ++w2) {
          const float* other = combine + (size_t)(w2 * hu + u) * Geo::kCombineFloats * 32;
          const float om0 = other[(Geo::kNTiles * 4 + 0) * 32 + lane];
          const float om1 = other[(Geo::kNTiles * 4 + 1) * 32 + lane];
          const float ol0 = other[(Geo::kNTiles * 4 + 2) * 32 + lane];
          const float ol1 = other[(Geo::kNTiles * 4 + 3) * 32 + lane];
          const float nm0 = fmaxf(m0, om0), nm1 = fmaxf(m1, om1);
          const float sa0 = exp2_int(m0 - nm0), sb0 = exp2_int(om0 - nm0);
          const float sa1 = exp2_int(m1 - nm1), sb1 = exp2_int(om1 - nm1);
#pragma unroll
          for (int i = 0; i < Geo::kNTiles; ++i) {
            o[i][0] = o[i][0] * sa0 + other[(i * 4 + 0) * 32 + lane] * sb0;
            o[i][1] = o[i][1] * sa0 + other[(i * 4 + 1) * 32 + lane] * sb0;
            o[i][2] = o[i][2] * sa1 + other[(i * 4 + 2) * 32 + lane] * sb1;
            o[i][3] = o[i][3] * sa1 + other[(i * 4 + 3) * 32 + lane] * sb1;
          }
          l0 = l0 * sa0 + ol0 * sb0;
          l1 = l1 * sa1 + ol1 * sb1;
          m0 = nm0;
          m1 = nm1;
        }
      }
      named_bar_sync(1, kGqaConsumerWarps * 32);
    }

    const bool complete = (c0 == c1);
    int slot = 0;
    if (!complete) slot = 2 * cta + ((cta == c0 && pre != c0 * P) ? 1 : 0);
    if (active && sub == 0) {
      // base-2 log-sum-exp of each row; empty state (all pages skipped) -> -inf
      const float lse0 = l0 > 0.f ? m0 + __log2f(l0) : -INFINITY;
      const float lse1 = l1 > 0.f ? m1 + __log2f(l1) : -INFINITY;
      const float inv0 = l0 > 0.f ? p.v_scale / l0 : 0.f, inv1 = l1 > 0.f ? p.v_scale / l1 : 0.f;
      // destination rows: the outputs, or this CTA's slot (rows in head-group order)
      auto out_row = [=](int rr) { return gqa_out_row(rr, b, ql, hg * hpc, G, R, p.Hk); };
      const int r0 = tile * 16 + g4, r1 = r0 + 8;
      const bool row0 = r0 < R, row1 = r1 < R;
      float* sl = p.slots + ((size_t)slot * p.n_hg + hg) * p.slot_floats;
      float* dO0 = complete ? gqa_o_ptr<HEAD_DIM>(p, si, out_row(hh * R + r0)) : sl + (size_t)(hh * R + r0) * HEAD_DIM;
      float* dO1 = complete ? gqa_o_ptr<HEAD_DIM>(p, si, out_row(hh * R + r1)) : sl + (size_t)(hh * R + r1) * HEAD_DIM;
      float* dL0 = complete ? gqa_l_ptr(p, si, out_row(hh * R + r0)) : sl + (size_t)rows_hg * HEAD_DIM + hh * R + r0;
      float* dL1 = complete ? gqa_l_ptr(p, si, out_row(hh * R + r1)) : sl + (size_t)rows_hg * HEAD_DIM + hh * R + r1;
      if constexpr (KV8) {
        // n-tile i, column 2c (+1) holds dim 2c * NT + i (+NT), NT = kNTiles: two runs of NT
        // consecutive dims (head_dim 128: 32c + i, +16; head_dim 64: 16c + i, +8)
        constexpr int NT = Geo::kNTiles;
        if (row0) {
#pragma unroll
          for (int i = 0; i < Geo::kNTiles; i += 4) {
            *reinterpret_cast<float4*>(dO0 + 2 * NT * c4 + i) =
                make_float4(o[i][0] * inv0, o[i + 1][0] * inv0, o[i + 2][0] * inv0, o[i + 3][0] * inv0);
            *reinterpret_cast<float4*>(dO0 + 2 * NT * c4 + NT + i) =
                make_float4(o[i][1] * inv0, o[i + 1][1] * inv0, o[i + 2][1] * inv0, o[i + 3][1] * inv0);
          }
          if (c4 == 0) *dL0 = complete ? lse0 * kLn2 : lse0;
        }
        if (row1) {
#pragma unroll
          for (int i = 0; i < Geo::kNTiles; i += 4) {
            *reinterpret_cast<float4*>(dO1 + 2 * NT * c4 + i) =
                make_float4(o[i][2] * inv1, o[i + 1][2] * inv1, o[i + 2][2] * inv1, o[i + 3][2] * inv1);
            *reinterpret_cast<float4*>(dO1 + 2 * NT * c4 + NT + i) =
                make_float4(o[i][3] * inv1, o[i + 1][3] * inv1, o[i + 2][3] * inv1, o[i + 3][3] * inv1);
          }
          if (c4 == 0) *dL1 = complete ? lse1 * kLn2 : lse1;
        }
      } else {
        if (row0) {
#pragma unroll
          for (int i = 0; i < Geo::kNTiles; ++i)
            *reinterpret_cast<float2*>(dO0 + i * 8 + c4 * 2) = make_float2(o[i][0] * inv0, o[i][1] * inv0);
          if (c4 == 0) *dL0 = complete ? lse0 * kLn2 : lse0;
        }
        if (row1) {
#pragma unroll
          for (int i = 0; i < Geo::kNTiles; ++i)
            *reinterpret_cast<float2*>(dO1 + i * 8 + c4 * 2) = make_float2(o[i][2] * inv1, o[i][3] * inv1);
          if (c4 == 0) *dL1 = complete ? lse1 * kLn2 : lse1;
        }
      }
    }
    if (!complete) {
      // publish this CTA's piece; the last CTA to arrive merges all pieces
      __threadfence();
      named_bar_sync(1, kGqaConsumerWarps * 32);
      int* ctr = p.counters + (size_t)sid * p.n_hg + hg;
      if (tid == 0) bcast[0] = (atomicAdd(ctr, 1) == c1 - c0) ? 1 : 0;
      named_bar_sync(1, kGqaConsumerWarps * 32);
      if (bcast[0]) {
        __threadfence();
        constexpr int kPer = HEAD_DIM / 32;
        for (int r = warp; r < rows_hg; r += kGqaConsumerWarps) {
          float mx = -INFINITY;
          for (int c = c0; c <= c1; ++c) {
            const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
            const float* sl = p.slots + ((size_t)k * p.n_hg + hg) * p.slot_floats;
            mx = fmaxf(mx, __ldcg(sl + (size_t)rows_hg * HEAD_DIM + r));
          }
          float acc[kPer];
#pragma unroll
          for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
          float wsum = 0.f;
          if (mx != -INFINITY) {
            for (int c = c0; c <= c1; ++c) {
              const int k = 2 * c + ((c == c0 && pre != c0 * P) ? 1 : 0);
              const float* sl = p.slots + ((size_t)k * p.n_hg + hg) * p.slot_floats;
              const float lk = __ldcg(sl + (size_t)rows_hg * HEAD_DIM + r);
              const float w = lk == -INFINITY ? 0.f : exp2f(lk - mx);
              wsum += w;
#pragma unroll
              for (int i = 0; i < kPer; ++i) acc[i] += w * __ldcg(sl + (size_t)r * HEAD_DIM + lane * kPer + i);
            }
          }
          const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
          const OutRow orow = gqa_out_row(r, b, ql, hg * hpc, G, R, p.Hk);
          float* dO = gqa_o_ptr<HEAD_DIM>(p, si, orow);
#pragma unroll
          for (int i = 0; i < kPer; ++i) dO[lane * kPer + i] = acc[i] * inv;
          if (lane == 0) *gqa_l_ptr(p, si, orow) = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
        }
        if (tid == 0) *ctr = 0;  // leave the counter ready for the next call
      }
    }
    pre += n;
  }
}

// ---------------------------------------------------------------------------- host side
// KV heads one CTA streams per page: a divisor of Hkv, at most 8 / row_tiles
// (one consumer warp per head and 16-row tile), a TMA box of at most 256 rows,
// and a stage (K and V of those heads for one page) of at most 64 KB so that
// three or more stages fit.
int gqa_row_tiles(int G, int q_len) { return (G * q_len + 15) / 16; }

int gqa_heads_per_cta(int Hkv, int bs, int head_dim, int row_tiles, int elem_bytes) {
  int cap = min(kGqaConsumerWarps / row_tiles, 256 / bs);
  cap = min(cap, 65536 / (bs * head_dim * 2 * elem_bytes));
  int best = 1;
  for (int h = 1; h <= cap; ++h)
    if (Hkv % h == 0) best = h;
  return best;
}

static int gqa_stage_count(uint32_t stage_bytes, size_t fixed_bytes) {
  const size_t budget = 225 * 1024 - fixed_bytes;
  int st = (int)(budget / stage_bytes);
  return st > 8 ? 8 : st;
}

template <int HEAD_DIM, bool MULTI, bool KV8>
static dcp_status launch_gqa_impl(const dcp_attn_desc& d, int D, const ShardSet& set, const void* q,
                                  const int32_t* seq_lens, void* ws, size_t ws_bytes, cudaStream_t st) {
  WorkspaceLayout L;
  if (!workspace_layout(d, D, &L)) return DCP_ERR_UNSUPPORTED;
  if (ws_bytes < L.total) return DCP_ERR_CAPACITY;
  GqaParams p;
  memset(&p, 0, sizeof(p));
  p.n_si = set.n;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.bs = d.block_size;
  p.D = D;
  p.mlb = d.max_local_blocks;
  p.q_len = d.q_len;
  p.R = p.G * p.q_len;
  p.rt = gqa_row_tiles(p.G, p.q_len);
  const int eb = KV8 ? 1 : 2;  // bytes per cached element
  p.hpc = gqa_heads_per_cta(p.Hkv, p.bs, HEAD_DIM, p.rt, eb);
  p.n_hg = p.Hkv / p.hpc;
  p.wph = kGqaConsumerWarps / (p.hpc * p.rt);
  p.stage_bytes = (uint32_t)(2 * p.hpc * p.bs * HEAD_DIM * eb);
  const size_t combine_bytes =
      p.wph > 1 ? (size_t)kGqaConsumerWarps * GqaGeom<HEAD_DIM, KV8>::kCombineFloats * 32 * sizeof(float) : 0;
  const size_t fixed = 16 * 8 + 8 * 4 + kScratchInts * 4 + 8 * 4 + combine_bytes;
  p.stages = gqa_stage_count(p.stage_bytes, fixed);
  if (p.stages < 2) return DCP_ERR_UNSUPPORTED;
  // FP8: scores carry k_scale, outputs v_scale
  p.scale_log2 = (float)((double)d.softmax_scale * (KV8 ? (double)d.k_scale : 1.0) * 1.4426950408889634);
  p.v_scale = KV8 ? d.v_scale : 1.f;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.seq_lens = seq_lens;
  p.status = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.status_off);
  p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.counters_off);
  p.slots = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.slots_off);
  p.slot_floats = L.slot_floats;
  p.Hk = set.owner_heads > 0 ? set.owner_heads : d.num_q_heads;
  for (int k = 0; k < kMaxShards; ++k) {
    p.own_O[k] = set.owner_O[k];
    p.own_L[k] = set.owner_L[k];
  }
  for (int si = 0; si < set.n; ++si) {
    p.table[si] = set.table[si];
    p.O[si] = set.O[si];
    p.LSE[si] = set.LSE[si];
    p.pool_pages[si] = set.pool_pages[si];
    p.shard_of_si[si] = set.shard[si];
    if (set.pool_pages[si] > 0) {
      const uint64_t rows = (uint64_t)set.pool_pages[si] * 2 * p.Hkv * p.bs;
      if (rows > (uint64_t)INT32_MAX) return DCP_ERR_UNSUPPORTED;  // TMA row coordinates are int32
      // boxes of 128-byte rows use the 128-byte swizzle; FP8 at head_dim 64 (64-byte rows) the 64-byte one
      if (encode_tiled_2d(&p.tmap[si], set.pool[si], HEAD_DIM, rows, HEAD_DIM * eb, GqaGeom<HEAD_DIM, KV8>::kBoxElems,
                          (uint32_t)(p.hpc * p.bs), eb, GqaGeom<HEAD_DIM, KV8>::kRowBytes) != CUDA_SUCCESS)
        return DCP_ERR_CUDA;
    }
  }
  const size_t smem = (size_t)p.stages * p.stage_bytes + fixed;
  auto kern = d.shard_rule == DCP_SHARD_INTERLEAVED ? gqa_decode_kernel<HEAD_DIM, MULTI, KV8, 0>
                                                    : gqa_decode_kernel<HEAD_DIM, MULTI, KV8, 1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return DCP_ERR_CUDA;
  // setmaxnreg.inc waits until the registers it asks for are free: never launch a build whose
  // launch allocation is smaller than the producer/consumer split
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return DCP_ERR_CUDA;
  if (fa.numRegs * (kGqaProducerWarps + kGqaConsumerWarps) <
      kGqaProducerWarps * kGqaProducerRegs + kGqaConsumerWarps * kGqaConsumerRegs)
    return DCP_ERR_CUDA;
  dim3 grid(L.nctas, p.n_hg);
  kern<<<grid, kGqaThreads, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

dcp_status launch_gqa_decode(const dcp_attn_desc& d, int D, const ShardSet& set, const void* q,
                             const int32_t* seq_lens, void* ws, size_t ws_bytes, cudaStream_t st) {
  const bool multi = d.q_len > 1;
  if (d.kv_dtype == DCP_KV_FP8_E4M3) {
    if (d.head_dim_qk == 128)
      return multi ? launch_gqa_impl<128, true, true>(d, D, set, q, seq_lens, ws, ws_bytes, st)
                   : launch_gqa_impl<128, false, true>(d, D, set, q, seq_lens, ws, ws_bytes, st);
    if (d.head_dim_qk == 64)
      return multi ? launch_gqa_impl<64, true, true>(d, D, set, q, seq_lens, ws, ws_bytes, st)
                   : launch_gqa_impl<64, false, true>(d, D, set, q, seq_lens, ws, ws_bytes, st);
    return DCP_ERR_UNSUPPORTED;
  }
  if (d.head_dim_qk == 128)
    return multi ? launch_gqa_impl<128, true, false>(d, D, set, q, seq_lens, ws, ws_bytes, st)
                 : launch_gqa_impl<128, false, false>(d, D, set, q, seq_lens, ws, ws_bytes, st);
  if (d.head_dim_qk == 64)
    return multi ? launch_gqa_impl<64, true, false>(d, D, set, q, seq_lens, ws, ws_bytes, st)
                 : launch_gqa_impl<64, false, false>(d, D, set, q, seq_lens, ws, ws_bytes, st);
  return DCP_ERR_UNSUPPORTED;
}

}  // namespace dcp
