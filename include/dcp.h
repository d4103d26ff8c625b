/*
 * dcp.h -- C ABI of the decode-context-parallel (DCP) attention library.
 *
 * The operation (sources, cited by page title and section):
 *   [P1] "Efficient Decode Context Parallelism with vLLM for Long Context
 *        Workloads" (papercache.org summary of the vLLM blog), "A2 方法细节":
 *        the KV cache of every request is split along the sequence into D
 *        shards; each shard attends the full single-token query against its
 *        local KV slice and emits a partial output O_i with its log-sum-exp
 *        LSE_i; the partials are combined as
 *            O = sum_i exp(LSE_i) / sum_j exp(LSE_j) * O_i.
 *   [P3] "vLLM长序列推理优化：DCP切分KV Cache原理与实战", §2.2: logical block
 *        b of a request belongs to shard b % D (interleaved sharding);
 *        §3.2: each shard stores its blocks in its own physical pool and
 *        addresses them through a global -> local remap (global block 4 of
 *        shard 0 with D = 4 is local block 1).
 *
 * All D shards live on ONE GPU here: D separate paged pools in the same HBM,
 * and the pages' AllGather / ReduceScatter exchange becomes an on-device
 * merge kernel (dcp_lse_merge).
 *
 * Conventions for every call:
 *   - The caller owns all memory.  The library never allocates device or
 *     host memory on the compute path and keeps no global state (it caches
 *     two driver entry points, each looked up once).  Calls are thread-safe.
 *   - "device" pointers are CUDA device addresses (e.g. a torch tensor's
 *     data_ptr()); "host" pointers are ordinary CPU memory.
 *   - GPU calls are asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = legacy default stream).  They never synchronise, except
 *     dcp_read_device_error and dcp_noalloc_read_device_error, which are
 *     documented as synchronous.
 *   - Return value: DCP_OK, or an error code.  Argument errors are detected
 *     on the host before anything is launched (nothing is written then).
 *     DCP_ERR_CUDA means a CUDA runtime call or a launch failed.
 *   - Data types: queries and KV sources are bf16 (raw 16-bit patterns);
 *     pools hold bf16 or FP8 E4M3 codes (dcp_kv_dtype); outputs and LSE are
 *     fp32, LSE in natural-log units of the SCALED scores; tables and
 *     lengths are int32.
 *   - Supported shapes (anything else is DCP_ERR_UNSUPPORTED):
 *       GQA: head_dim_qk == head_dim_v in {64, 128}; Hq % Hkv == 0 and
 *            Hq / Hkv <= 16; block_size a multiple of 16 with
 *            block_size * head_dim <= 16384 (up to 256 tokens at head_dim
 *            64, 128 tokens at head_dim 128).
 *       MLA: Hq == 64, Hkv == 1, head_dim_qk == 576, head_dim_v == 512,
 *            block_size == 64.
 *       1 <= D <= 16 shards; batch >= 1; seq_lens[b] >= 0.
 *       Multi-token decode: 1 <= q_len <= 4 query tokens per request
 *       (GQA and MLA).
 *       FP8 cache (kv_dtype DCP_KV_FP8_E4M3): GQA (head_dim 64 or 128) and MLA
 *       (whose latent takes one scale: k_scale == v_scale).
 *       Shard rules: interleaved (default) or contiguous chunks (dcp_shard_rule).
 */
#ifndef DCP_H
#define DCP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DCP_API __attribute__((visibility("default")))
#else
#define DCP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dcp_status {
    DCP_OK = 0,
    DCP_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent arguments */
    DCP_ERR_UNSUPPORTED = 2, /* shape outside the supported set listed above */
    DCP_ERR_CAPACITY = 3,    /* a caller buffer (table row, workspace) is too small */
    DCP_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    DCP_ERR_DEVICE = 5       /* the device recorded an invalid page id (see dcp_read_device_error) */
} dcp_status;

typedef enum dcp_layout {
    DCP_LAYOUT_GQA = 0, /* grouped-query attention: Hkv KV heads, q head h reads KV head h / (Hq/Hkv) */
    DCP_LAYOUT_MLA = 1  /* multi-head latent attention, absorbed form: one shared latent row per token */
} dcp_layout;

/*
 * Element type of the KV cache pools.  [P3 §7: an FP8 KV cache complements
 * DCP by shrinking the cache further; the page does not fix a format.]
 *   DCP_KV_BF16      bf16 values.
 *   DCP_KV_FP8_E4M3  one byte per value: an E4M3 code (the OCP FP8 E4M3 "fn"
 *                    format: bias 7, no infinities, largest finite 448) and a
 *                    per-tensor scale, value = scale * e4m3(code); K uses
 *                    k_scale, V uses v_scale.  The MLA latent is one tensor
 *                    (key = all 576 entries, value = the first 512), so it has
 *                    one scale: k_scale, which v_scale must equal
 *                    (DCP_ERR_INVALID_ARG otherwise).  The cache writes quantise bf16
 *                    rows as code = e4m3_rn_satfinite(float32(x) * inv), inv =
 *                    float32(1 / scale): the product rounded to float32, then to
 *                    the nearest code (ties to even), magnitudes past 448
 *                    saturated.  The decode kernel feeds the codes (exact in
 *                    f16) and the query converted to f16 to f16 tensor-core
 *                    products; query elements outside f16's normal range
 *                    (|q| > 65504 or |q| < 2^-14) lose precision there.
 */
/*
 * How a request's logical blocks are dealt to the D shards.
 *   DCP_SHARD_INTERLEAVED  block g -> shard g % D as local block g / D ([P3] §2.2/§3.2; the
 *                          rule the pages' implementation uses).
 *   DCP_SHARD_CONTIGUOUS   the nblk = ceil(len / block_size) blocks are cut into D consecutive
 *                          chunks: shard s holds blocks floor(s*nblk/D) .. floor((s+1)*nblk/D) - 1,
 *                          local block g - floor(s*nblk/D) ([P1] "A2 方法细节" illustrates
 *                          sequence sharding as "GPU0 holds 0-50K, GPU1 50K-100K, ...").  A
 *                          token's shard depends on the request's total length, so contiguous
 *                          tables cannot grow: dcp_grow_block_table and dcp_append_kv are
 *                          interleaved only.
 */
typedef enum dcp_shard_rule {
    DCP_SHARD_INTERLEAVED = 0,
    DCP_SHARD_CONTIGUOUS = 1
} dcp_shard_rule;

typedef enum dcp_kv_dtype {
    DCP_KV_BF16 = 0,
    DCP_KV_FP8_E4M3 = 1
} dcp_kv_dtype;

/*
 * Problem description shared by the decode calls.
 *   layout           dcp_layout.
 *   batch            B, number of requests (q_len decode tokens each).
 *   num_q_heads      Hq.
 *   num_kv_heads     Hkv (GQA); must be 1 for MLA.
 *   head_dim_qk      query/key width (GQA head_dim; MLA 576 = 512 latent + 64 rope).
 *   head_dim_v       value width (GQA head_dim; MLA 512 = the first 512 entries of the latent row).
 *   block_size       tokens per KV page.
 *   max_local_blocks row length of each shard's block table (>= the largest local block count).
 *   softmax_scale    multiplier of q.k (e.g. 1/sqrt(head_dim); MLA 1/sqrt(192)).
 *   q_len            query tokens per request: 1 = single-token decode; 2..4 = multi-token
 *                    decode (MTP / speculative drafts; [P1] "A5 结论", future-work item 3,
 *                    names MTP and speculative decoding as what DCP must support next).
 *                    The q_len new tokens are the LAST q_len tokens of the request and their
 *                    KV is already in the cache (seq_len counts them); query token j
 *                    (0-based) attends the tokens t < seq_len - (q_len - 1 - j), i.e.
 *                    causally within the draft.  A query token with no visible token in a
 *                    shard gets O = 0, LSE = -inf there.
 *   kv_dtype         dcp_kv_dtype of the pools.
 *   k_scale, v_scale per-tensor scales of an FP8 cache (positive, finite); ignored for bf16.
 *   shard_rule       dcp_shard_rule the tables were built with (pools, tables and seq_lens must agree).
 */
typedef struct dcp_attn_desc {
    int32_t layout;
    int32_t batch;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim_qk;
    int32_t head_dim_v;
    int32_t block_size;
    int32_t max_local_blocks;
    float softmax_scale;
    int32_t q_len;
    int32_t kv_dtype;
    float k_scale;
    float v_scale;
    int32_t shard_rule;
} dcp_attn_desc;

/* Library version, major * 10000 + minor * 100 + patch. */
DCP_API int32_t dcp_version(void);

/* Static string naming a status code. */
DCP_API const char *dcp_status_string(dcp_status status);

/*
 * Table extent (host only).  [P3 §2.2, §3.2]
 *   seq_lens          host int32[batch], tokens already in the cache per request (>= 0).
 *   max_local_blocks  out: largest number of blocks any request has in any shard.
 *   num_pages         out, host int32[D]: pages shard s needs (sum over requests).
 * Errors: DCP_ERR_INVALID_ARG for null pointers, batch < 0, block_size <= 0,
 * D < 1 or D > 16, or a negative length.
 */
DCP_API dcp_status dcp_block_table_extent(const int32_t *seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                  int32_t *max_local_blocks, int32_t *num_pages);

/*
 * Per-shard block tables (host only).  [P3 §2.2 interleaved rule, §3.2 remap]
 * Token t of request b lies in logical block g = t / block_size, owned by
 * shard s = g % D as local block j = g / D.  For every shard s:
 *   tables[s][b][j]  = physical page of shard s's pool holding global block
 *                      j*D + s of request b; -1 past the request's local blocks;
 *   local_len[s][b]  = tokens of request b stored by shard s.
 * Pages of each shard are numbered 0.. in (request, local block) order.  If
 * perm_seed != 0, the ids of shard s are relabelled by the permutation of
 * [0, num_pages[s]) that a Fisher-Yates shuffle produces from the SplitMix64
 * stream whose state starts at perm_seed + (s+1) * 0xD1B54A32D192ED03
 * (i from n-1 down to 1: state += 0x9E3779B97F4A7C15, j = mix(state) % (i+1),
 * swap entries i and j) -- non-contiguous page ids for testing allocators.
 *   tables     out, host int32[D][batch][max_local_blocks].
 *   local_len  out, host int32[D][batch]; may be NULL.
 * Errors: as dcp_block_table_extent; DCP_ERR_CAPACITY if max_local_blocks is
 * smaller than a request's local block count (tables then undefined).
 */
DCP_API dcp_status dcp_build_block_table(const int32_t *seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                 uint64_t perm_seed, int32_t max_local_blocks, int32_t *tables,
                                 int32_t *local_len);

/*
 * The same two calls under a chosen dcp_shard_rule (the calls above use
 * DCP_SHARD_INTERLEAVED).  Under DCP_SHARD_CONTIGUOUS, tables[s][b][j] holds
 * the page of global block floor(s*nblk_b/D) + j, pages are still numbered in
 * (request, local block) order, and local_len counts the chunk's tokens.
 * Errors: as above, and DCP_ERR_INVALID_ARG for an unknown rule.
 */
DCP_API dcp_status dcp_block_table_extent_rule(const int32_t *seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                               int32_t shard_rule, int32_t *max_local_blocks, int32_t *num_pages);
DCP_API dcp_status dcp_build_block_table_rule(const int32_t *seq_lens, int32_t batch, int32_t block_size, int32_t D,
                                              int32_t shard_rule, uint64_t perm_seed, int32_t max_local_blocks,
                                              int32_t *tables, int32_t *local_len);

/* Bytes of one KV page for `desc` (GQA: 2*Hkv*block_size*head_dim*e; MLA: block_size*576*2; e = 2 for
 * bf16, 1 for FP8); 0 if invalid. */
DCP_API size_t dcp_kv_page_bytes(const dcp_attn_desc *desc);

/*
 * Cache placement: scatter every request's unsharded KV rows into the D
 * shard pools (the cache write that precedes decoding).  [P3 §3.2]
 *   kv_src      device bf16, requests concatenated in order:
 *               GQA rows [token][2 (K,V)][Hkv][head_dim]; MLA rows [token][576].
 *   cu_seqlens  device int64[batch+1], prefix sums of seq_lens (row offsets in kv_src).
 *   seq_lens    device int32[batch] (the contiguous rule reads them to find each token's shard).
 *   tables      host array of D device pointers, each int32[batch][max_local_blocks]
 *               (as built by dcp_build_block_table / _rule with desc->shard_rule).
 *   kv_pools    host array of D device pointers; pool s holds pool_pages[s] pages:
 *               GQA page [2 (K,V)][Hkv][block_size][head_dim] of the pool's
 *               kv_dtype (bf16, or FP8 codes quantised on the way in);
 *               MLA page [block_size][576] of the pool's kv_dtype.
 *   pool_pages  host int32[D].
 *   device_error optional device int32 (may be NULL): set to 1 if a table entry
 *               lies outside its pool; such rows are skipped, never written.
 * Slots past a request's last token keep whatever they held.
 */
DCP_API dcp_status dcp_place_kv(const dcp_attn_desc *desc, int32_t D, const void *kv_src, const int64_t *cu_seqlens,
                        const int32_t *seq_lens, const int32_t *const *tables, void *const *kv_pools,
                        const int32_t *pool_pages, int32_t *device_error, void *stream);

/*
 * Incremental table growth (host only) for requests that gained tokens since
 * the tables were built.  [P3 §6.2: when a sequence grows only the newly
 * added blocks are remapped; existing entries keep their pages.]  For each
 * request b in order and each new logical block g in
 * [ceil(old_seq_lens[b]/bs), ceil(new_seq_lens[b]/bs)) in order, shard s =
 * g % D gives local block g / D the page next_page[s]++.  local_len (may be
 * NULL) gains the tokens each shard received.  Growing from all-zero lengths
 * with next_page = 0 reproduces dcp_build_block_table (perm_seed 0).
 *   old_seq_lens, new_seq_lens  host int32[batch], new >= old.
 *   tables      in/out, host int32[D][batch][max_local_blocks].
 *   local_len   in/out, host int32[D][batch], or NULL.
 *   next_page   in/out, host int32[D]: first free page of each shard pool.
 *   pool_pages  host int32[D]: pages each pool holds.
 * Errors: DCP_ERR_INVALID_ARG (nulls, a shrinking request, bad sizes);
 * DCP_ERR_CAPACITY if a local block index reaches max_local_blocks or a pool
 * runs out of pages.  On error nothing is modified.
 */
DCP_API dcp_status dcp_grow_block_table(const int32_t *old_seq_lens, const int32_t *new_seq_lens, int32_t batch,
                                        int32_t block_size, int32_t D, int32_t max_local_blocks, int32_t *tables,
                                        int32_t *local_len, int32_t *next_page, const int32_t *pool_pages);

/*
 * Cache write of new tokens (the decode step's append).  [P3 §3.2, §6.2]
 * Request b's new rows are rows [cu_rows[b], cu_rows[b+1]) of kv_new and hold
 * tokens first_pos[b], first_pos[b]+1, ...; each goes to shard
 * (t / block_size) % D, page tables[shard][b][(t / block_size) / D], slot
 * t % block_size (layouts as in dcp_place_kv).
 *   kv_new      device bf16 rows ([2][Hkv][head_dim] GQA, [576] MLA).
 *   cu_rows     device int64[batch+1];  first_pos  device int32[batch].
 *   tables, kv_pools, pool_pages, device_error: as in dcp_place_kv (tables
 *               already grown to cover the new tokens).
 * Interleaved shard rule only (DCP_ERR_UNSUPPORTED otherwise).
 */
DCP_API dcp_status dcp_append_kv(const dcp_attn_desc *desc, int32_t D, const void *kv_new, const int64_t *cu_rows,
                                 const int32_t *first_pos, const int32_t *const *tables, void *const *kv_pools,
                                 const int32_t *pool_pages, int32_t *device_error, void *stream);

/*
 * Workspace bytes the decode calls need for `desc` and D shards on the
 * current device (split partials, arrival counters, a status word).  The
 * workspace must be zeroed once by dcp_workspace_init before its first use;
 * every decode call leaves its counters at zero again.  One workspace may
 * not be used by two decode calls that overlap in time.  0 if invalid.
 */
DCP_API size_t dcp_decode_workspace_bytes(const dcp_attn_desc *desc, int32_t D);

/* Zero a workspace (asynchronous, on `stream`). */
DCP_API dcp_status dcp_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Partial attention of ONE shard.  [P1 "A2 方法细节", Compute step]
 * For every request b and query head h, over the tokens of b that shard
 * `shard` stores (logical blocks g with g % D == shard, or its chunk under
 * the contiguous rule):
 *   s_t = softmax_scale * q[b][h] . k_t,  m = max s_t,  l = sum exp(s_t - m),
 *   O_i[b][h] = sum exp(s_t - m) v_t / l,  LSE_i[b][h] = m + ln l.
 * GQA: k_t, v_t are KV head h / (Hq/Hkv) of token t.  MLA: k_t is the whole
 * 576-wide latent row, v_t its first 512 entries.  A request with no token
 * in this shard gets O_i = 0 and LSE_i = -inf.
 *   q           device bf16 [batch][q_len][Hq][head_dim_qk] (the full query: every shard reads it).
 *   kv_pool     device, this shard's pool (layout as in dcp_place_kv), pool_pages pages.
 *   table       device int32 [batch][max_local_blocks], this shard's block table.
 *   seq_lens    device int32 [batch], GLOBAL lengths; the local token count is
 *               derived from (seq_len, block_size, shard, D, desc->shard_rule).
 *   O_i         device fp32 [batch][q_len][Hq][head_dim_v];  LSE_i  device fp32 [batch][q_len][Hq].
 * With q_len > 1 each (request, query token j, head) row follows the same
 * formulas over the visible tokens t < seq_len - (q_len - 1 - j).
 *   workspace   device, >= dcp_decode_workspace_bytes(desc, D) bytes, initialised.
 * Page ids outside [0, pool_pages) are not read: their tokens are left out
 * of the softmax, and the workspace status records the error (see
 * dcp_read_device_error).
 */
DCP_API dcp_status dcp_decode_partial(const dcp_attn_desc *desc, const void *q, const void *kv_pool, int32_t pool_pages,
                              const int32_t *table, const int32_t *seq_lens, int32_t shard, int32_t D, float *O_i,
                              float *LSE_i, void *workspace, size_t workspace_bytes, void *stream);

/*
 * One shard's partial laid out for the exchange between D ranks of the
 * multi-GPU form.  [P1 "A2 方法细节", step 3: after computing, the ranks
 * all-gather their (O_i, LSE_i) and reduce-scatter the reweighted sum, so
 * that every rank ends with the merged output of its own slice of heads.]
 * n_owners ranks own consecutive slices of Hk = Hq / n_owners query heads
 * (rank k: heads k*Hk .. k*Hk + Hk - 1).  The partial of dcp_decode_partial
 * is written owner by owner into `send`, fp32, n_owners chunks of
 * dcp_owner_chunk_floats(desc, n_owners) floats each:
 *   chunk k:  O rows  [batch][q_len][Hk][head_dim_v]   (row (b, j, h) at
 *                     ((b*q_len + j)*Hk + h - k*Hk) * head_dim_v),
 *             then LSE rows [batch][q_len][Hk], padded to a multiple of 64 floats.
 * Chunk k is what this rank sends to rank k in an all-to-all; a rank that
 * receives chunk k from every shard merges them with dcp_lse_merge (O parts
 * at the chunk starts, LSE parts after their O rows, rows = batch*q_len*Hk).
 * With n_owners = 1 chunk 0 is dcp_decode_partial's O_i followed by LSE_i.
 *   send       device fp32, n_owners * dcp_owner_chunk_floats(desc, n_owners) floats, 16-byte aligned.
 * Other arguments, results and errors as dcp_decode_partial; DCP_ERR_INVALID_ARG
 * if n_owners < 1, n_owners > 16 or it does not divide num_q_heads.
 */
DCP_API size_t dcp_owner_chunk_floats(const dcp_attn_desc *desc, int32_t n_owners);
DCP_API dcp_status dcp_decode_partial_owner_major(const dcp_attn_desc *desc, const void *q, const void *kv_pool,
                                                  int32_t pool_pages, const int32_t *table, const int32_t *seq_lens,
                                                  int32_t shard, int32_t D, int32_t n_owners, float *send,
                                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * The same partial with the exchange folded into the decode kernel: owner k's
 * chunk (the layout above) is written straight to owner_chunks[k], so no send
 * buffer and no separate all-to-all are needed.  [P1 "A2 方法细节", step 3.]
 * owner_chunks[k] may point into another GPU's memory that this process has
 * mapped (peer access, or dcp_ipc_open below): the kernel's epilogue and split
 * combine store the rows with ordinary global stores, so the transfer happens
 * while the last pieces of the partial are still being computed.  The caller
 * orders the stores before the owner reads its chunks (e.g. the stream's
 * completion followed by a barrier of the rank group) and, when it reuses a
 * chunk buffer, the owner's previous read before this call.
 *   owner_chunks  host array of n_owners device pointers, each 16-byte aligned,
 *                 dcp_owner_chunk_floats(desc, n_owners) floats.
 * Other arguments, results and errors as dcp_decode_partial_owner_major;
 * DCP_ERR_INVALID_ARG for a null or misaligned chunk pointer.
 */
DCP_API dcp_status dcp_decode_partial_to_owners(const dcp_attn_desc *desc, const void *q, const void *kv_pool,
                                                int32_t pool_pages, const int32_t *table, const int32_t *seq_lens,
                                                int32_t shard, int32_t D, int32_t n_owners,
                                                float *const *owner_chunks, void *workspace,
                                                size_t workspace_bytes, void *stream);

/*
 * Mapping a device buffer of another process (CUDA IPC), for owner chunks on
 * other GPUs.  [The multi-GPU form above; the pages name no mechanism.]
 *   dcp_ipc_handle_bytes  size of a handle (host bytes).
 *   dcp_ipc_export        device_ptr: device memory of this process from
 *                         cudaMalloc (e.g. PyTorch's default caching allocator;
 *                         not stream-ordered pool memory).  Writes the handle of
 *                         the allocation that holds it to handle_out (host,
 *                         dcp_ipc_handle_bytes()) and device_ptr's byte offset
 *                         inside that allocation to *offset_out.
 *                         DCP_ERR_INVALID_ARG if device_ptr is not device memory;
 *                         DCP_ERR_CUDA if its allocation cannot be exported.
 *   dcp_ipc_open          maps the allocation a handle names (from another
 *                         process; peer access is enabled when needed) and
 *                         returns its base in *base_out; the buffer is at
 *                         base + offset.  Must not be called on a handle that
 *                         this process exported.
 *   dcp_ipc_close         unmaps a base returned by dcp_ipc_open.
 * Host calls; DCP_ERR_CUDA when the CUDA runtime refuses.  No multicast object
 * is created.
 */
DCP_API size_t dcp_ipc_handle_bytes(void);
DCP_API dcp_status dcp_ipc_export(const void *device_ptr, void *handle_out, uint64_t *offset_out);
DCP_API dcp_status dcp_ipc_open(const void *handle, void **base_out);
DCP_API dcp_status dcp_ipc_close(void *base);

/*
 * All D partials in one launch.  Host arrays of D device pointers:
 * kv_pools[s], tables[s], O_parts[s], LSE_parts[s]; pool_pages host int32[D].
 * Each launch splits the concatenated page lists of its shards into equal
 * ranges, one per CTA, so the rounding of a result depends on which shards
 * share the launch: this call and D calls of dcp_decode_partial agree to
 * rounding (not bit for bit).  Repeating the same call on the same inputs
 * gives bit-identical results.
 */
DCP_API dcp_status dcp_decode_partial_all(const dcp_attn_desc *desc, const void *q, const void *const *kv_pools,
                                  const int32_t *pool_pages, const int32_t *const *tables, const int32_t *seq_lens,
                                  int32_t D, float *const *O_parts, float *const *LSE_parts, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * dcp_decode_partial_all for callers that cannot allocate device memory
 * (GQA layout only).  The pages have no counterpart of this call.
 *
 * Some callers cannot call cudaMalloc where they run a decode step: code
 * that is handed only its input and output buffers (an inference-engine
 * plugin, an embedded runtime without a device allocator), serving loops
 * that forbid allocation after start-up so that memory never fragments and
 * no step waits on the allocator, and code that must not touch the
 * allocator while other work is being captured.  This call takes no
 * workspace: it uses a 16 MiB scratch array that lives in the library and
 * that every GPU which loads the library holds until the process exits.
 * Inputs, outputs and results are those of dcp_decode_partial_all.
 *   - The first call on each device looks up the scratch array's device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture.
 *   - Each call clears the scratch's status word and arrival counters on
 *     `stream`, then launches the decode kernel.  It allocates nothing.
 *   - All calls share the scratch, which keeps the last call's contents:
 *     calls that overlap on the GPU (e.g. on two streams) race; serialise them.
 *   - The status bits that dcp_read_device_error reports for a workspace
 *     (bit 0: an out-of-range page id was skipped; bit 1: a pipeline wait
 *     timed out and that call's results are invalid) go to the scratch's own
 *     status word; dcp_noalloc_read_device_error reads and clears it.  Each
 *     call clears it first, so it describes the latest call only.
 * Errors: as dcp_decode_partial_all; DCP_ERR_UNSUPPORTED for MLA;
 * DCP_ERR_CAPACITY if the problem needs more than the 16 MiB scratch
 * (dcp_decode_workspace_bytes(desc, D) > 16 MiB, e.g. very wide head groups).
 */
DCP_API dcp_status dcp_decode_partial_all_noalloc(const dcp_attn_desc *desc, const void *q,
                                                  const void *const *kv_pools, const int32_t *pool_pages,
                                                  const int32_t *const *tables, const int32_t *seq_lens, int32_t D,
                                                  float *const *O_parts, float *const *LSE_parts, void *stream);

/*
 * Status word of dcp_decode_partial_all_noalloc's scratch on the current
 * device: waits for `stream`, stores the bits in *error_out (meanings as in
 * dcp_read_device_error) and clears the word.  Allocates nothing; like the
 * decode call, its first use on a device looks up the scratch address.
 */
DCP_API dcp_status dcp_noalloc_read_device_error(int32_t *error_out, void *stream);

/*
 * Diagnostic of the decode kernels' bounded pipeline waits (no attention is
 * computed).  One thread waits, through the same bounded wait the decode
 * kernels use for every mbarrier, on a barrier that nothing ever arrives on;
 * when the wait gives up (after about 4 s) it sets bit 1 of the workspace's
 * status word, as a decode kernel does when a pipeline wait times out.
 *   workspace  device, a workspace as for dcp_decode_partial (only its status
 *              word, the first int32, is touched); read the bit back with
 *              dcp_read_device_error.
 * Asynchronous on `stream`; the stream is busy for the wait limit.  Nothing
 * is left in flight when the wait gives up, so the CUDA context stays usable.
 * Errors: DCP_ERR_INVALID_ARG for a null workspace; DCP_ERR_CUDA if the launch fails.
 */
DCP_API dcp_status dcp_check_wait_timeout(void *workspace, void *stream);

/*
 * LSE merge of D partials.  [P1 "A2 方法细节", merge equation;
 * P3 §2.3 equivalent local-max/local-sum form]
 *   O[r] = sum_i w_i O_i[r] / sum_i w_i,  w_i = exp(LSE_i[r] - max_j LSE_j[r]),
 *   LSE_out[r] = max_j LSE_j[r] + ln sum_i w_i.
 * Parts with LSE = -inf weigh 0; if all are -inf then O = 0, LSE_out = -inf.
 *   O_parts, LSE_parts  host arrays of D device pointers: fp32 [rows][d_v] and fp32 [rows].
 *   rows                number of (request, query token, head) rows (batch * q_len * Hq).
 *   O                   device fp32 [rows][d_v]; LSE_out device fp32 [rows] or NULL.
 * d_v must be a multiple of 4 and all pointers 16-byte aligned.
 */
DCP_API dcp_status dcp_lse_merge(const float *const *O_parts, const float *const *LSE_parts, int32_t D, int32_t rows,
                         int32_t d_v, float *O, float *LSE_out, void *stream);

/*
 * One whole decode step with HOST inputs and outputs.  [P1 "A2 方法细节": the
 * shards attend the full query against their local KV slices, then the
 * partials are merged by the equation above.]  On `stream`, in order: the
 * query, the lengths and the D block tables are copied from host memory into
 * `staging`; the D shard partials run in one launch (as
 * dcp_decode_partial_all) into `staging`; dcp_lse_merge combines them; the
 * merged O (and LSE) are copied back to host memory.
 *   host_q         host bf16 [batch][q_len][Hq][head_dim_qk].
 *   host_seq_lens  host int32 [batch], global lengths.
 *   host_tables    host int32 [D][batch][max_local_blocks] (as dcp_build_block_table writes them).
 *   kv_pools       host array of D device pointers (pools already written); pool_pages host int32[D].
 *   staging        device, >= dcp_host_step_staging_bytes(desc, D) bytes, 256-byte aligned: the
 *                  uploaded inputs, the D partials and the merged output live there (caller-owned;
 *                  one staging buffer may not serve two steps that overlap in time).
 *   workspace      as for dcp_decode_partial_all (initialised).
 *   host_O         host fp32 [batch][q_len][Hq][head_dim_v];  host_LSE host fp32 [batch][q_len][Hq] or NULL.
 * Asynchronous like every GPU call: host_O / host_LSE are valid once `stream` has been
 * synchronised, and the host inputs must stay untouched until then.  Pinned (page-locked)
 * host memory keeps the copies asynchronous; pageable memory works, but the CUDA runtime
 * then stages it and the call may block the calling thread.
 * Errors: as dcp_decode_partial_all; DCP_ERR_CAPACITY if staging or workspace is too small.
 */
DCP_API size_t dcp_host_step_staging_bytes(const dcp_attn_desc *desc, int32_t D);
DCP_API dcp_status dcp_decode_step_host(const dcp_attn_desc *desc, int32_t D, const void *host_q,
                                        const int32_t *host_seq_lens, const int32_t *host_tables,
                                        const void *const *kv_pools, const int32_t *pool_pages, void *staging,
                                        size_t staging_bytes, void *workspace, size_t workspace_bytes,
                                        float *host_O, float *host_LSE, void *stream);

/*
 * Read (synchronously: waits for `stream`) and clear the status word of a
 * workspace.  *error_out is a bit set, 0 if nothing was recorded since the
 * last read: bit 0 (1) = a block-table entry lay outside its pool; bit 1
 * (2) = an internal pipeline wait exceeded its time limit (the results of
 * that call are invalid; never expected in correct operation).
 */
DCP_API dcp_status dcp_read_device_error(void *workspace, int32_t *error_out, void *stream);

/*
 * Parallel-configuration rule of [P1 "A2 方法细节"] (MLA and GQA backend paragraphs):
 *   MLA: tp >= dcp and tp % dcp == 0;
 *   GQA: (tp / num_kv_heads) >= dcp and (tp / num_kv_heads) % dcp == 0.
 * dcp == 1 is always accepted.  DCP_OK if allowed, DCP_ERR_UNSUPPORTED if
 * not, DCP_ERR_INVALID_ARG for non-positive arguments.
 */
DCP_API dcp_status dcp_validate_config(int32_t tp, int32_t dcp, int32_t num_kv_heads, int32_t layout);

#ifdef __cplusplus
}
#endif

#endif /* DCP_H */
