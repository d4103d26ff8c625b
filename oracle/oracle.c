/*
 * oracle.c -- float64 CPU oracle for decode context parallelism (DCP).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  It shares
 * no code with the CUDA library: no headers, helpers, tables or constants.
 *
 * Sources (web pages; cited by title and section):
 *   [P1] "Efficient Decode Context Parallelism with vLLM for Long Context
 *        Workloads" (papercache.org summary of the vLLM blog), section
 *        "A2 方法细节" (method details): KV cache split along the sequence,
 *        AllGather Q -> Compute -> AllGather + ReduceScatter, and the merge
 *        O = sum_i exp(LSE_i) / sum_j exp(LSE_j) * O_i; section "速读"
 *        (the MLA / GQA configuration constraints).
 *   [P3] "vLLM长序列推理优化：DCP切分KV Cache原理与实战", §2.1 (KV-size
 *        arithmetic), §2.2 (interleaved sharding block_idx % D == rank),
 *        §2.3 (local max m_i, local sum l_i, rescaled merge), §3.2 (per-rank
 *        physical blocks, global -> local block remap: global block 4 on
 *        rank 0 of D=4 is local block 1).
 *
 * Everything is computed in double precision from bf16 inputs that are
 * widened exactly.  Readings where the pages are silent (each also listed in
 * the design notes):
 *   - block_idx is the logical block index of a token inside its request,
 *     floor(t / block_size);
 *   - local block index = floor(global block / D) (P3 §3.2 example);
 *   - physical pages of a shard are handed out in (request, local block)
 *     order, optionally permuted by a seeded Fisher-Yates shuffle;
 *   - softmax scale is an input; LSE is the natural-log log-sum-exp of the
 *     scaled scores; each partial O_i is normalised by its own sum;
 *   - an empty token set has O = 0 and LSE = -inf and carries merge weight 0;
 *   - MLA: a token's key is its whole latent row (d_qk wide), its value is
 *     the first d_v entries of the same row;
 *   - an FP8 (E4M3) cache holds code = e4m3(float32(x) * float32(1/scale)),
 *     standing for scale * e4m3_value(code), with one scale for GQA keys,
 *     one for GQA values, and one for the whole MLA latent row (the latent
 *     is a single tensor read as key and value).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_GQA 0
#define OR_MLA 1

/* ------------------------------------------------------------------ */
/* bf16 -> double (exact)                                              */
/* ------------------------------------------------------------------ */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* Shard assignment (P3 §2.2, §3.2)                                    */
/* ------------------------------------------------------------------ */

/* Shard owning token t: its logical block floor(t/bs) taken modulo D. */
int oracle_token_shard(int64_t t, int block_size, int D) {
    return (int)((t / block_size) % D);
}

/* Local block index of token t inside its shard: floor(floor(t/bs) / D). */
int64_t oracle_token_local_block(int64_t t, int block_size, int D) {
    return (t / block_size) / D;
}

/*
 * Contiguous-chunk rule (the [P1] "A2 方法细节" illustration "GPU0 holds 0-50K,
 * GPU1 50K-100K, ..." for a 200K sequence on 4 GPUs): the nblk = ceil(len/bs)
 * logical blocks of a request are cut into D consecutive chunks, shard s
 * holding blocks floor(s*nblk/D) .. floor((s+1)*nblk/D) - 1; its local block
 * index counts from the start of its chunk.  The chunking depends on the
 * request's total length `seq_len`.  rule 0 is the interleaved rule above,
 * rule 1 this one.
 */
static int64_t or_chunk_begin(int64_t nblk, int D, int s) { return ((int64_t)s * nblk) / D; }

int oracle_token_shard_rule(int64_t t, int block_size, int D, int rule, int64_t seq_len) {
    if (rule == 0) return oracle_token_shard(t, block_size, D);
    int64_t g = t / block_size, nblk = (seq_len + block_size - 1) / block_size;
    for (int s = 0; s < D; ++s)
        if (g < or_chunk_begin(nblk, D, s + 1)) return s;
    return D - 1;
}

int64_t oracle_token_local_block_rule(int64_t t, int block_size, int D, int rule, int64_t seq_len) {
    if (rule == 0) return oracle_token_local_block(t, block_size, D);
    int64_t nblk = (seq_len + block_size - 1) / block_size;
    int s = oracle_token_shard_rule(t, block_size, D, rule, seq_len);
    return t / block_size - or_chunk_begin(nblk, D, s);
}

/* SplitMix64 (Steele, Lea & Flood 2014), used only for the optional page permutation. */
static uint64_t or_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/*
 * Per-shard block tables.  For shard s and request b, entry j of the table
 * is the physical page (in shard s's own pool) that stores global block
 * g = j*D + s of request b.  Entries past the request's local block count
 * are -1.  local_len[s][b] counts the tokens of b that shard s stores.
 * num_pages[s] is the number of pages shard s needs.
 *
 * Pages are numbered by walking the tokens of every request in order and
 * giving each (shard, local block) its next free page on first sight, which
 * is (request, local block) order.  With perm_seed != 0 the page ids of
 * shard s are then relabelled by the permutation pi_s produced by a
 * Fisher-Yates shuffle of [0, num_pages[s]) driven by the SplitMix64 stream
 * whose state starts at perm_seed + (s + 1) * 0xD1B54A32D192ED03: for
 * i = n-1 down to 1, j = next() mod (i + 1), swap(pi[i], pi[j]).
 *
 * Returns 0 on success, -1 on bad arguments, -2 if max_local_blocks is too
 * small for some request.
 */
int oracle_block_tables_rule(const int32_t *seq_lens, int B, int block_size, int D, int rule, uint64_t perm_seed,
                             int max_local_blocks, int32_t *tables, int32_t *local_len, int32_t *num_pages) {
    if (B < 0 || block_size <= 0 || D <= 0 || max_local_blocks < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0) return -1;
    for (int64_t i = 0; i < (int64_t)D * B * max_local_blocks; ++i) tables[i] = -1;
    for (int64_t i = 0; i < (int64_t)D * B; ++i) local_len[i] = 0;
    int64_t *next_page = (int64_t *)calloc((size_t)D, sizeof(int64_t));
    int rc = 0;
    for (int b = 0; b < B && rc == 0; ++b) {
        for (int64_t t = 0; t < seq_lens[b]; ++t) {
            int s = oracle_token_shard_rule(t, block_size, D, rule, seq_lens[b]);
            int64_t j = oracle_token_local_block_rule(t, block_size, D, rule, seq_lens[b]);
            if (j >= max_local_blocks) { rc = -2; break; }
            int32_t *entry = &tables[((int64_t)s * B + b) * max_local_blocks + j];
            if (*entry < 0) *entry = (int32_t)next_page[s]++;
            local_len[(int64_t)s * B + b] += 1;
        }
    }
    for (int s = 0; s < D; ++s) num_pages[s] = (int32_t)next_page[s];
    if (rc == 0 && perm_seed != 0) {
        for (int s = 0; s < D; ++s) {
            int64_t n = next_page[s];
            if (n < 2) continue;
            int32_t *pi = (int32_t *)malloc((size_t)n * sizeof(int32_t));
            for (int64_t i = 0; i < n; ++i) pi[i] = (int32_t)i;
            uint64_t state = perm_seed + (uint64_t)(s + 1) * 0xD1B54A32D192ED03ULL;
            for (int64_t i = n - 1; i >= 1; --i) {
                state += 0x9E3779B97F4A7C15ULL;
                uint64_t j = or_mix(state) % (uint64_t)(i + 1);
                int32_t tmp = pi[i];
                pi[i] = pi[j];
                pi[j] = tmp;
            }
            for (int b = 0; b < B; ++b)
                for (int j = 0; j < max_local_blocks; ++j) {
                    int32_t *e = &tables[((int64_t)s * B + b) * max_local_blocks + j];
                    if (*e >= 0) *e = pi[*e];
                }
            free(pi);
        }
    }
    free(next_page);
    return rc;
}

/* The tables under the interleaved rule. */
int oracle_block_tables(const int32_t *seq_lens, int B, int block_size, int D, uint64_t perm_seed,
                        int max_local_blocks, int32_t *tables, int32_t *local_len, int32_t *num_pages) {
    return oracle_block_tables_rule(seq_lens, B, block_size, D, 0, perm_seed, max_local_blocks, tables, local_len,
                                    num_pages);
}

/*
 * Incremental growth of the shard tables when requests gain tokens
 * ([P3] §6.2: when a sequence grows only its newly added blocks are remapped;
 * existing entries keep their pages).  Walking the new tokens
 * t in [old_len[b], new_len[b]) of every request in order, a (shard, local
 * block) seen for the first time takes the next free page of its shard,
 * next_page[s]++; local_len[s][b] counts the tokens added to shard s.
 * Returns 0, -1 on bad arguments (new < old, negative lengths), -2 when a
 * local block index reaches max_local_blocks, -3 when a shard runs out of
 * pages (next_page[s] == pool_pages[s]).  Tables of a failed call are partly
 * updated.
 */
int oracle_grow_tables(const int32_t *old_lens, const int32_t *new_lens, int B, int block_size, int D,
                       int max_local_blocks, int32_t *tables, int32_t *local_len, int32_t *next_page,
                       const int32_t *pool_pages) {
    if (B < 0 || block_size <= 0 || D <= 0 || max_local_blocks < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (old_lens[b] < 0 || new_lens[b] < old_lens[b]) return -1;
    for (int b = 0; b < B; ++b) {
        for (int64_t t = old_lens[b]; t < new_lens[b]; ++t) {
            int s = oracle_token_shard(t, block_size, D);
            int64_t j = oracle_token_local_block(t, block_size, D);
            if (j >= max_local_blocks) return -2;
            int32_t *entry = &tables[((int64_t)s * B + b) * max_local_blocks + j];
            if (*entry < 0) {
                if (next_page[s] >= pool_pages[s]) return -3;
                *entry = next_page[s]++;
            }
            local_len[(int64_t)s * B + b] += 1;
        }
    }
    return 0;
}

/*
 * Reference placement of one request's unsharded KV rows into the shard
 * pools (the cache write that precedes decoding).  Token t of request b goes
 * to pool shard(t), page table[shard][b][local block], slot t mod bs.
 *   GQA pool page layout: [2 (K,V)][Hkv][bs][d]     (source row [2][Hkv][d])
 *   MLA pool page layout: [bs][d_qk]               (source row [d_qk])
 * pools[s] points at shard s's pool (bytes, bf16 elements).
 */
void oracle_place_request_rule(int layout, int Hkv, int d, int block_size, int D, int rule, int B, int b,
                               int max_local_blocks, const int32_t *tables, int64_t n_tok, const uint16_t *src,
                               uint16_t **pools) {
    for (int64_t t = 0; t < n_tok; ++t) {
        int s = oracle_token_shard_rule(t, block_size, D, rule, n_tok);
        int64_t j = oracle_token_local_block_rule(t, block_size, D, rule, n_tok);
        int64_t page = tables[((int64_t)s * B + b) * max_local_blocks + j];
        int64_t slot = t % block_size;
        if (layout == OR_GQA) {
            for (int kv = 0; kv < 2; ++kv)
                for (int h = 0; h < Hkv; ++h)
                    for (int k = 0; k < d; ++k) {
                        int64_t dst = (((page * 2 + kv) * Hkv + h) * block_size + slot) * d + k;
                        pools[s][dst] = src[((t * 2 + kv) * Hkv + h) * d + k];
                    }
        } else {
            for (int k = 0; k < d; ++k) pools[s][(page * block_size + slot) * d + k] = src[t * d + k];
        }
    }
}

void oracle_place_request(int layout, int Hkv, int d, int block_size, int D, int B, int b,
                          int max_local_blocks, const int32_t *tables, int64_t n_tok, const uint16_t *src,
                          uint16_t **pools) {
    oracle_place_request_rule(layout, Hkv, d, block_size, D, 0, B, b, max_local_blocks, tables, n_tok, src, pools);
}

/* ------------------------------------------------------------------ */
/* Attention of one request over a token subset                        */
/* ------------------------------------------------------------------ */

/*
 * Softmax attention of the single decode query of one request against the
 * tokens t in [0, n_tok) that satisfy the filter: all tokens when shard < 0,
 * else the tokens that shard `shard` stores under `rule` (interleaved: logical
 * block floor(t/bs) % D == shard, P3 §2.2; contiguous: the chunk of a request
 * of rule_len tokens, see above).  Direct definition, two passes, no blocking:
 *   s_t   = scale * sum_k q[h][k] * K_t[k]
 *   M     = max_t s_t,  Z = sum_t exp(s_t - M)
 *   O[h]  = sum_t exp(s_t - M) V_t / Z,   LSE[h] = M + ln Z
 * GQA: q head h reads KV head floor(h / (Hq / Hkv)); K_t = K[t][kvh][:],
 *      V_t = V[t][kvh][:]  (src row layout [2][Hkv][d]).
 * MLA: K_t = C[t][0:d_qk], V_t = C[t][0:d_v]  (src row layout [d_qk]).
 * Heads are computed for h in [h_begin, h_end); outputs are indexed by the
 * absolute head: O[h][d_v], LSE[h].
 */
void oracle_attend_rule_f64(int layout, int Hq, int Hkv, int d_qk, int d_v, const uint16_t *q, int64_t n_tok,
                            const double *src, double scale, int block_size, int D, int shard, int rule,
                            int64_t rule_len, int h_begin, int h_end, double *O, double *LSE) {
    double *s = (double *)malloc((size_t)(n_tok > 0 ? n_tok : 1) * sizeof(double));
    double *qd = (double *)malloc((size_t)d_qk * sizeof(double));
    int group = (layout == OR_GQA) ? Hq / Hkv : Hq;
    for (int h = h_begin; h < h_end; ++h) {
        int kvh = (layout == OR_GQA) ? h / group : 0;
        for (int k = 0; k < d_qk; ++k) qd[k] = bf16_to_double(q[(int64_t)h * d_qk + k]);
        double M = -INFINITY;
        int64_t count = 0;
        for (int64_t t = 0; t < n_tok; ++t) {
            if (shard >= 0 && oracle_token_shard_rule(t, block_size, D, rule, rule_len) != shard) continue;
            const double *krow = (layout == OR_GQA) ? src + ((t * 2 + 0) * Hkv + kvh) * (int64_t)d_qk
                                                    : src + t * (int64_t)d_qk;
            double acc = 0.0;
            for (int k = 0; k < d_qk; ++k) acc += qd[k] * krow[k];
            s[t] = scale * acc;
            if (s[t] > M) M = s[t];
            ++count;
        }
        double *o = O + (int64_t)h * d_v;
        for (int k = 0; k < d_v; ++k) o[k] = 0.0;
        if (count == 0) {
            LSE[h] = -INFINITY;
            continue;
        }
        double Z = 0.0;
        for (int64_t t = 0; t < n_tok; ++t) {
            if (shard >= 0 && oracle_token_shard_rule(t, block_size, D, rule, rule_len) != shard) continue;
            const double *vrow = (layout == OR_GQA) ? src + ((t * 2 + 1) * Hkv + kvh) * (int64_t)d_qk
                                                    : src + t * (int64_t)d_qk;
            double w = exp(s[t] - M);
            Z += w;
            for (int k = 0; k < d_v; ++k) o[k] += w * vrow[k];
        }
        for (int k = 0; k < d_v; ++k) o[k] /= Z;
        LSE[h] = M + log(Z);
    }
    free(qd);
    free(s);
}

/* Interleaved-rule attention over a float64-valued source. */
void oracle_attend_f64(int layout, int Hq, int Hkv, int d_qk, int d_v, const uint16_t *q, int64_t n_tok,
                       const double *src, double scale, int block_size, int D, int shard, int h_begin, int h_end,
                       double *O, double *LSE) {
    oracle_attend_rule_f64(layout, Hq, Hkv, d_qk, d_v, q, n_tok, src, scale, block_size, D, shard, 0, n_tok, h_begin,
                           h_end, O, LSE);
}

/* The same attention with the key/value source given as bf16 bit patterns
 * (widened exactly to double first). */
void oracle_attend(int layout, int Hq, int Hkv, int d_qk, int d_v, const uint16_t *q, int64_t n_tok,
                   const uint16_t *src, double scale, int block_size, int D, int shard, int h_begin, int h_end,
                   double *O, double *LSE) {
    int64_t row = (layout == OR_GQA) ? 2 * (int64_t)Hkv * d_qk : d_qk;
    int64_t n = n_tok * row;
    double *wide = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    for (int64_t i = 0; i < n; ++i) wide[i] = bf16_to_double(src[i]);
    oracle_attend_f64(layout, Hq, Hkv, d_qk, d_v, q, n_tok, wide, scale, block_size, D, shard, h_begin, h_end, O,
                      LSE);
    free(wide);
}

/* ------------------------------------------------------------------ */
/* FP8 KV cache: E4M3 codes with a per-tensor scale                    */
/* ------------------------------------------------------------------ */

/*
 * The FP8 E4M3 format (the OCP 8-bit floating-point specification's E4M3,
 * "fn" variant): bit 7 sign, bits 6..3 exponent e (bias 7), bits 2..0
 * mantissa m.  e = 0: subnormal, value m/8 * 2^-6; e = 1..15: (1 + m/8) *
 * 2^(e-7), except e = 15, m = 7 which is NaN.  No infinities; the largest
 * finite magnitude is 448 (e = 15, m = 6).
 */
double oracle_e4m3_decode(uint8_t c) {
    int sign = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/*
 * Nearest E4M3 code to x, ties to the even code (even mantissa), magnitudes
 * above 448 saturated to +-448 (the "satfinite" rule); NaN -> 0x7F.  Found by
 * scanning the 127 non-negative finite codes, which are increasing in value.
 */
uint8_t oracle_e4m3_encode(double x) {
    if (x != x) return 0x7F;
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int best = 0;
    for (int c = 1; c <= 0x7E; ++c) {
        double dc = fabs(oracle_e4m3_decode((uint8_t)c) - a), db = fabs(oracle_e4m3_decode((uint8_t)best) - a);
        if (dc < db || (dc == db && (c & 1) == 0)) best = c;
    }
    return (uint8_t)(sign | best);
}

/*
 * Quantisation of bf16 cache values to E4M3 codes with a per-tensor scale:
 * code = e4m3(float32(x) * inv_scale), the product rounded to float32 first
 * (the decision is taken in the kernel's precision), inv_scale = float32 of
 * 1 / scale.  The value a code stands for is scale * e4m3_value(code).
 */
void oracle_quantize_e4m3(const uint16_t *src, int64_t n, float inv_scale, uint8_t *out) {
    /* The code is a function of the 16-bit input alone: encode each of the 65,536 bf16 patterns
       once (only when the input is long enough to make that cheaper) and look the rest up. */
    uint8_t *table = n > 65536 ? (uint8_t *)malloc(65536) : NULL;
    int use_table = table != NULL;
    if (use_table)
        for (int b = 0; b < 65536; ++b) table[b] = oracle_e4m3_encode((double)((float)bf16_to_double((uint16_t)b) * inv_scale));
    for (int64_t i = 0; i < n; ++i) {
        if (use_table) {
            out[i] = table[src[i]];
            continue;
        }
        float x = (float)bf16_to_double(src[i]);
        float p = x * inv_scale;
        out[i] = oracle_e4m3_encode((double)p);
    }
    free(table);
}

/* scale * value(code) for n codes (exact in double). */
void oracle_dequantize_e4m3(const uint8_t *codes, int64_t n, double scale, double *out) {
    double value[256];
    for (int c = 0; c < 256; ++c) value[c] = scale * oracle_e4m3_decode((uint8_t)c);
    for (int64_t i = 0; i < n; ++i) out[i] = value[codes[i]];
}

/*
 * Placement of one request's quantised GQA rows (codes [n_tok][2][Hkv][d],
 * one byte per element) into byte pools whose pages are [2][Hkv][bs][d]:
 * the same token walk as oracle_place_request_rule, one byte per element.
 */
void oracle_place_request_u8(int Hkv, int d, int block_size, int D, int rule, int B, int b, int max_local_blocks,
                             const int32_t *tables, int64_t n_tok, const uint8_t *src, uint8_t **pools) {
    for (int64_t t = 0; t < n_tok; ++t) {
        int s = oracle_token_shard_rule(t, block_size, D, rule, n_tok);
        int64_t j = oracle_token_local_block_rule(t, block_size, D, rule, n_tok);
        int64_t page = tables[((int64_t)s * B + b) * max_local_blocks + j];
        int64_t slot = t % block_size;
        for (int kv = 0; kv < 2; ++kv)
            for (int h = 0; h < Hkv; ++h)
                for (int k = 0; k < d; ++k)
                    pools[s][(((page * 2 + kv) * Hkv + h) * block_size + slot) * d + k] =
                        src[((t * 2 + kv) * Hkv + h) * d + k];
    }
}

/*
 * Placement of one request's quantised MLA latent rows (codes [n_tok][576],
 * one byte per element, the whole row quantised with the latent's one scale)
 * into byte pools whose pages are [bs][576]: the same token walk as
 * oracle_place_request_rule, one byte per element.
 */
void oracle_place_request_mla_u8(int d, int block_size, int D, int rule, int B, int b, int max_local_blocks,
                                 const int32_t *tables, int64_t n_tok, const uint8_t *src, uint8_t **pools) {
    for (int64_t t = 0; t < n_tok; ++t) {
        int s = oracle_token_shard_rule(t, block_size, D, rule, n_tok);
        int64_t j = oracle_token_local_block_rule(t, block_size, D, rule, n_tok);
        int64_t page = tables[((int64_t)s * B + b) * max_local_blocks + j];
        int64_t slot = t % block_size;
        for (int k = 0; k < d; ++k) pools[s][(page * block_size + slot) * d + k] = src[t * d + k];
    }
}

/* ------------------------------------------------------------------ */
/* Merge of partial results                                            */
/* ------------------------------------------------------------------ */

/*
 * [P1] merge: O = sum_i exp(LSE_i) / sum_j exp(LSE_j) * O_i, evaluated with
 * the largest LSE as the common reference so no exponential overflows:
 *   M = max_i LSE_i, w_i = exp(LSE_i - M), O = sum_i w_i O_i / sum_i w_i,
 *   LSE = M + ln sum_i w_i.
 * Parts with LSE_i = -inf have weight 0; if every part is -inf the result is
 * O = 0, LSE = -inf.  Layout: O_parts[D][rows][d_v], LSE_parts[D][rows].
 */
void oracle_merge(const double *O_parts, const double *LSE_parts, int D, int64_t rows, int d_v, double *O,
                  double *LSE) {
    for (int64_t r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int i = 0; i < D; ++i)
            if (LSE_parts[(int64_t)i * rows + r] > M) M = LSE_parts[(int64_t)i * rows + r];
        double *o = O + r * d_v;
        for (int k = 0; k < d_v; ++k) o[k] = 0.0;
        if (M == -INFINITY) {
            LSE[r] = -INFINITY;
            continue;
        }
        double W = 0.0;
        for (int i = 0; i < D; ++i) {
            double li = LSE_parts[(int64_t)i * rows + r];
            if (li == -INFINITY) continue;
            double w = exp(li - M);
            W += w;
            const double *oi = O_parts + ((int64_t)i * rows + r) * d_v;
            for (int k = 0; k < d_v; ++k) o[k] += w * oi[k];
        }
        for (int k = 0; k < d_v; ++k) o[k] /= W;
        LSE[r] = M + log(W);
    }
}

/*
 * [P3 §2.3] form of the same merge: every rank keeps its local max m_i, its
 * local sum l_i = sum exp(s - m_i) and its UNnormalised output
 * U_i = sum exp(s - m_i) v.  Then m = max m_i, l = sum l_i exp(m_i - m),
 * O = sum U_i exp(m_i - m) / l.  Ranks with l_i = 0 are skipped.
 * Layout: U_parts[D][rows][d_v], m_parts[D][rows], l_parts[D][rows].
 */
void oracle_merge_ml(const double *U_parts, const double *m_parts, const double *l_parts, int D, int64_t rows,
                     int d_v, double *O) {
    for (int64_t r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int i = 0; i < D; ++i)
            if (l_parts[(int64_t)i * rows + r] > 0.0 && m_parts[(int64_t)i * rows + r] > m)
                m = m_parts[(int64_t)i * rows + r];
        double *o = O + r * d_v;
        for (int k = 0; k < d_v; ++k) o[k] = 0.0;
        if (m == -INFINITY) continue;
        double l = 0.0;
        for (int i = 0; i < D; ++i) {
            double li = l_parts[(int64_t)i * rows + r];
            if (li <= 0.0) continue;
            double c = exp(m_parts[(int64_t)i * rows + r] - m);
            l += li * c;
            const double *ui = U_parts + ((int64_t)i * rows + r) * d_v;
            for (int k = 0; k < d_v; ++k) o[k] += ui[k] * c;
        }
        for (int k = 0; k < d_v; ++k) o[k] /= l;
    }
}

/* ------------------------------------------------------------------ */
/* Arithmetic and configuration rules                                  */
/* ------------------------------------------------------------------ */

/* [P3 §2.1] KV bytes per token per layer: 2 (K and V) x heads x head_dim x element bytes. */
int64_t oracle_kv_bytes_per_token(int num_kv_heads, int head_dim, int elem_bytes) {
    return 2LL * num_kv_heads * head_dim * elem_bytes;
}

/*
 * [P1 "速读" and the MLA / GQA backend paragraphs of "A2 方法细节"]
 *   MLA: tp >= dcp and tp % dcp == 0.
 *   GQA: (tp / kv_heads) >= dcp and (tp / kv_heads) % dcp == 0 (integer division).
 * dcp == 1 (no context parallelism) is always allowed.
 * Returns 1 if the combination is allowed, 0 if not, -1 on bad arguments.
 */
int oracle_validate_config(int tp, int dcp, int num_kv_heads, int layout) {
    if (tp <= 0 || dcp <= 0) return -1;
    if (dcp == 1) return 1; /* reading: D = 1 is plain decoding, no constraint applies */
    if (layout == OR_MLA) return (tp >= dcp && tp % dcp == 0) ? 1 : 0;
    if (num_kv_heads <= 0) return -1;
    int rep = tp / num_kv_heads;
    return (rep >= dcp && rep % dcp == 0) ? 1 : 0;
}
