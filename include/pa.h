/*
 * pa.h -- C ABI of the B200 paged-attention library (libpagedattn.so).
 *
 * The library implements the data-parallel hot path of PagedAttention:
 * scaled-dot-product attention whose K/V are read through per-sequence block
 * tables from a fixed pool of non-contiguous physical blocks, the block-table
 * KV append (reshape_and_cache) and the copy-on-write block copy, plus the
 * host block manager that decides tables, slot mappings and copies.
 *
 * Pages the operations follow (cited by title and section):
 *   [P1] "abhik.ai examples/pagedattention.py" -- KVPool: physical pool,
 *        allocation order, append, fork, copy-on-write, release, Eq. 3.
 *   [P2] "vladkulikov.com modern-llms module 9 notebook" -- PagedKVPool:
 *        preflighted multi-token append, share_prefix, snapshot, validate.
 *   [P3] "docs.rs ferrum-kv 0.4.0 src/attention.rs" -- paged_attention:
 *        query [q_tokens, num_heads, head_dim], GQA (kv_h = h / (H / Hkv)),
 *        scale = 1/sqrt(head_dim), causal rule max_visible = kv_len -
 *        q_tokens + qt, softmax, weighted sum of V.
 *   [P4] "semidirectx cmu11-667 lecture19 infer_world.py", section 3 --
 *        online softmax (m, l) and the tiled (m, l, acc) recurrence.
 *
 * Conventions shared by every entry point
 *   - Pool layout: k_cache and v_cache are device arrays
 *     [num_blocks, block_size, num_kv_heads, head_dim], row-major, dtype
 *     pa_dtype.  Slot s = block * block_size + offset; element
 *     (blk, off, h, i) sits at ((blk * block_size + off) * num_kv_heads + h)
 *     * head_dim + i.  This is [P3]'s per-token layout [kv_len, Hkv, d]
 *     stored block by block.
 *   - Ownership: every device pointer (pool, key/value, query, output, block
 *     tables, kv_lens, workspace) belongs to the caller and must stay valid
 *     until the work queued on the given stream has finished.  The pool
 *     borrows k_cache/v_cache; pa_free never frees them.  The pool owns its
 *     manager state (free list, refcounts, tables), a small device staging
 *     area for append plans and a device error word.
 *   - Devices: a device pool belongs to the device that was current when it
 *     was created.  Every device call runs there: the library makes that
 *     device current for the call, when it is not already, and restores the
 *     caller's device before returning.  Streams, buffers and workspaces
 *     passed in must belong to the pool's device.  The tensor-core kernels
 *     opt into their large shared memory once per device, the first time
 *     they launch there (any host thread may be the first), so pools on
 *     several devices of one process all work.
 *   - Streams: device work is queued asynchronously on the caller's stream
 *     (cudaStream_t passed as void*; NULL = legacy default stream).  Calls on
 *     one pool must be issued from one host thread and on one stream, or be
 *     externally ordered.
 *   - Errors: status codes only; nothing aborts or traps.  Host-detectable
 *     errors are checked before any state changes (the preflight of [P1]
 *     append and [P2] append).  Device-detectable errors (a table entry
 *     outside [0, num_blocks), a slot outside the pool, kv_len < q_tokens or
 *     beyond the table, a wait that ran out of iterations) set bits of the
 *     pool's device error word (PA_DEVERR_*), the affected output rows are
 *     written as zeros and the kernel finishes; pa_get_error reads them.
 *   - A pool created with k_cache == v_cache == NULL is host-only: the
 *     manager calls work (no GPU needed), device calls return
 *     PA_ERR_NO_DEVICE.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_pool pa_pool; /* opaque */

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,     /* bad size, null pointer, misaligned pointer  */
  PA_ERR_UNKNOWN_SEQ = 2,     /* sequence id not live ([P1] _existing)       */
  PA_ERR_DUP_SEQ = 3,         /* sequence id already live ([P1] create)      */
  PA_ERR_POOL_EXHAUSTED = 4,  /* preflight found too few free blocks         */
  PA_ERR_CUDA = 5,            /* a CUDA runtime call failed                  */
  PA_ERR_DEVICE = 6,          /* pa_get_error found device error bits        */
  PA_ERR_UNSUPPORTED = 7,     /* shape/dtype outside what the kernels take   */
  PA_ERR_NO_DEVICE = 8,       /* device call on a host-only pool             */
  PA_ERR_INTERNAL = 9,        /* pa_validate found a broken invariant        */
  PA_ERR_SCRATCH_LIMIT = 10   /* request needs more than the fixed scratch   */
} pa_status;

/* PA_INT8: int8 codes with one float32 scale per (token, head) row; only
 * through pa_pool_create_int8 (or pa_pool_create_layers).  PA_FP8: E4M3
 * codes in the same record; only through pa_pool_create_fp8 (or
 * pa_pool_create_layers). */
typedef enum pa_dtype { PA_F32 = 0, PA_BF16 = 1, PA_INT8 = 2, PA_FP8 = 3 } pa_dtype;

/* Bits of the device error word. */
#define PA_DEVERR_BLOCK_ID 1  /* block-table entry outside [0, num_blocks)   */
#define PA_DEVERR_SLOT 2      /* slot outside [0, num_blocks * block_size)   */
#define PA_DEVERR_KV_LEN 4    /* kv_len < q_tokens, < 0 or beyond the table  */
#define PA_DEVERR_TIMEOUT 8   /* a bounded wait gave up                      */

/* [P2] PagedKVPool.snapshot figures (token counts). */
typedef struct pa_stats {
  int64_t allocated_blocks;
  int64_t free_blocks;
  int64_t physical_capacity_tokens;  /* allocated_blocks * block_size       */
  int64_t physical_payload_tokens;   /* sum over blocks of max sharer fill  */
  int64_t logical_tokens;            /* sum of sequence lengths             */
  int64_t internal_waste_tokens;     /* capacity - payload                  */
  int64_t sharing_savings_tokens;    /* logical - payload                   */
  int64_t live_sequences;
} pa_stats;

/* ---- pool lifetime ----------------------------------------------------- */

/* Create a pool over caller-owned k_cache/v_cache (see layout above).
 * alloc_order: host array, a permutation of [0, num_blocks); a new block is
 * the first free id in this order ([P1] KVPool._allocate).  NULL = identity
 * order.  Copied; the caller may free it after the call.
 * Errors: PA_ERR_INVALID_ARG (non-positive size, not a permutation, exactly
 * one of k_cache/v_cache NULL, cache pointer not 16-byte aligned, kv_dtype
 * PA_INT8 / PA_FP8: use pa_pool_create_int8 / pa_pool_create_fp8). */
pa_status pa_pool_create(int32_t num_blocks, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim,
                         pa_dtype kv_dtype, void* k_cache, void* v_cache,
                         const int32_t* alloc_order, pa_pool** out);

/* A pool whose caches hold num_layers layers ([P3] paged_attention's
 * `layer` argument: one block table per sequence serves every layer).
 * k_cache/v_cache: [num_layers, <one layer as for pa_pool_create>] (bf16 /
 * f32), or for PA_INT8 / PA_FP8 k_cache = [num_layers, num_blocks,
 * num_kv_heads, PA_INT8_RECORD_BYTES] records and v_cache NULL.  The
 * returned handle is layer 0; pa_pool_layer gives the others.  All layers share the host
 * manager: sequence and plan calls on any of them act on the same tables.
 * A step over L layers plans once (pa_plan_append), copies once
 * (pa_cow_copy copies each pair in every layer), then writes and attends
 * per layer (pa_reshape_and_cache, pa_decode, ... on each layer's handle);
 * pa_append_kv on a layer plans, copies in every layer and writes only that
 * layer.  Errors: as pa_pool_create / pa_pool_create_int8, INVALID_ARG for
 * num_layers < 1, a NULL k_cache or an unknown kv_dtype. */
pa_status pa_pool_create_layers(int32_t num_blocks, int32_t block_size,
                                int32_t num_kv_heads, int32_t head_dim,
                                pa_dtype kv_dtype, int32_t num_layers,
                                void* k_cache, void* v_cache,
                                const int32_t* alloc_order, pa_pool** out);

/* Handle of layer `layer` of a pool (the pool itself for 0).  Layer handles
 * belong to the pool: pa_free(pool) releases them, pa_free(layer handle)
 * returns INVALID_ARG. */
pa_status pa_pool_layer(pa_pool* pool, int32_t layer, pa_pool** layer_pool);

/* Pool of int8 KV rows ([P2] KV quantisation experiment, 8 bits: per
 * (token, head) row, scale = max|x| / 127 (1 for a zero row), code =
 * round-half-even(x / scale) clipped to +-127, decided in float64; the
 * scale is stored as float32 and a row reads back as code * scale).
 *   kv_records: device bytes [num_blocks, num_kv_heads, PA_INT8_RECORD_BYTES],
 *   16-byte aligned, caller-owned.  One record per (block, head):
 *     [0, 2048)     K codes, 16 tokens x 128; token t's 16-byte chunk k is
 *                   stored at t * 128 + (k ^ (t & 7)) * 16 (pre-swizzled)
 *     [2048, 4096)  V codes, 128 rows d of 16 bytes (token t at d * 16 + t)
 *     [4096, 4160)  16 float32 K scales, token order
 *     [4160, 4224)  16 float32 V scales
 *   The decode loads a (block, head) record with one copy.  Only
 *   block_size 16 and head_dim 128.
 * On such a pool pa_append_kv / pa_reshape_and_cache take bf16 key/value
 * [T, Hkv, 128] and quantise them into their slots; pa_cow_copy copies whole
 * records; pa_decode and pa_decode_window (and pa_decode_append /
 * pa_decode_window_append, as two launches) dequantise in the tensor-core
 * kernels for H / Hkv <= 8.  pa_prefill_chunk, and pa_decode for larger
 * groups, take the CUDA-core path, which dequantises every element it reads
 * (correct, not fast), windows included.
 * Errors: PA_ERR_UNSUPPORTED (block_size != 16 or head_dim != 128),
 * PA_ERR_INVALID_ARG (NULL or misaligned kv_records, bad size or order),
 * PA_ERR_CUDA. */
#define PA_INT8_RECORD_BYTES 4224
pa_status pa_pool_create_int8(int32_t num_blocks, int32_t block_size,
                              int32_t num_kv_heads, int32_t head_dim,
                              void* kv_records, const int32_t* alloc_order,
                              pa_pool** out);

/* Pool of FP8 KV rows: the per-row absmax recipe of pa_pool_create_int8 on
 * the E4M3 grid of the OCP 8-bit floating point specification (exponent
 * bias 7, 3 mantissa bits, subnormals, no infinities, largest finite 448):
 * scale = max|x| / 448 (1 for a zero row); code = the E4M3 value nearest to
 * x / scale, ties to the even code, decided in float64; a zero magnitude is
 * stored as +0; the scale is stored as float32 and a row reads back as
 * value(code) * scale.  The records, their layout (PA_INT8_RECORD_BYTES per
 * (block, head), E4M3 bytes in place of the int8 codes), the calls that
 * take them and the errors are those of pa_pool_create_int8. */
pa_status pa_pool_create_fp8(int32_t num_blocks, int32_t block_size,
                             int32_t num_kv_heads, int32_t head_dim,
                             void* kv_records, const int32_t* alloc_order,
                             pa_pool** out);

/* Destroy the manager, its staging area and error word (synchronises the
 * device first).  Never frees k_cache/v_cache.  NULL is a no-op. */
pa_status pa_free(pa_pool* pool);

/* ---- host block manager ([P1] KVPool, [P2] PagedKVPool) ----------------- */

/* New empty sequence; no block is reserved ([P1] create). */
pa_status pa_seq_create(pa_pool* pool, int32_t seq);

/* New sequence `child` sharing the blocks that cover the first
 * prefix_tokens tokens of `parent` (refcount +1 each) ([P2] share_prefix);
 * prefix_tokens = -1 shares the whole parent ([P1] fork).
 * Errors: UNKNOWN_SEQ, DUP_SEQ, INVALID_ARG (prefix > parent length). */
pa_status pa_seq_fork(pa_pool* pool, int32_t parent, int32_t child,
                      int32_t prefix_tokens);

/* Drop one reference per block of `seq`; blocks reaching zero return to the
 * free list ([P1] release, [P2] release). */
pa_status pa_seq_release(pa_pool* pool, int32_t seq);

/* Keep the first lengths[i] tokens of sequence seqs[i], for n distinct
 * sequences (a rollback of their newest tokens, e.g. drafted tokens that were
 * not accepted).  Not on the pages: it is [P1] release applied to the dropped
 * tail -- every block wholly past lengths[i] loses this sequence's reference
 * and returns to the free list at zero -- and equals [P2] share_prefix of the
 * kept tokens into a new sequence followed by release of the old one.  A
 * kept partial tail block is left as it is (a copy-on-write already made is
 * not undone).  seqs, lengths: host [n].  All-or-nothing: UNKNOWN_SEQ, or
 * INVALID_ARG (length < 0 or beyond the sequence, an id named twice, NULL
 * arrays with n > 0), before any change. */
pa_status pa_seq_truncate(pa_pool* pool, const int32_t* seqs,
                          const int32_t* lengths, int32_t n);

/* Prefix cache ([P2] prefix-hash trace, "complete block boundaries"): the
 * block that ends at token `end` is identified by (scope, revision, every
 * token id before `end`), and only full blocks are keyed.  The cache maps a
 * key to the physical block that first held it and keeps one reference of
 * its own on that block, so cached blocks outlive their writers until
 * pa_prefix_clear.  scope and revision are caller-chosen 64-bit ids (a hash
 * of a tenant name, of a model revision, ...); token ids are compared
 * exactly, not by hash.
 *
 * pa_seq_create_cached: new sequence `seq` that starts with the longest run
 * of leading full blocks of tokens[0, n_tokens) (host) whose keys are cached,
 * shared with their current holders (refcount + 1 each).  *hit_tokens =
 * the tokens covered (a multiple of block_size); append the rest with
 * pa_append_kv.  Errors: DUP_SEQ, INVALID_ARG (n_tokens < 0, tokens NULL). */
pa_status pa_seq_create_cached(pa_pool* pool, int32_t seq, uint64_t scope,
                               uint64_t revision, const int32_t* tokens,
                               int32_t n_tokens, int32_t* hit_tokens);

/* Key the full blocks of `seq` among its first n_tokens tokens, whose ids
 * are tokens[0, n_tokens) (host; n_tokens <= the sequence length).  A key
 * already cached keeps its block.  *added_blocks = new keys.  Errors:
 * UNKNOWN_SEQ, INVALID_ARG. */
pa_status pa_prefix_publish(pa_pool* pool, int32_t seq, uint64_t scope,
                            uint64_t revision, const int32_t* tokens,
                            int32_t n_tokens, int32_t* added_blocks);

/* Drop every reference the prefix cache holds; *freed_blocks = blocks that
 * returned to the free list (may be NULL). */
pa_status pa_prefix_clear(pa_pool* pool, int32_t* freed_blocks);

/* Number of keys the prefix cache holds. */
int64_t pa_prefix_entries(const pa_pool* pool);

/* Length and table of `seq`.  blocks_out (host, capacity cap) may be NULL to
 * query only n_blocks/length.  INVALID_ARG if cap is too small. */
pa_status pa_seq_table(const pa_pool* pool, int32_t seq, int32_t* blocks_out,
                       int32_t cap, int32_t* n_blocks, int32_t* length);

/* Batch tables for a decode/prefill call: tables_out host [n, width] int32
 * (row i = table of seqs[i], padded with 0), kv_lens_out host [n] int32.
 * INVALID_ARG if a table is wider than `width`. */
pa_status pa_block_tables(const pa_pool* pool, const int32_t* seqs, int32_t n,
                          int32_t width, int32_t* tables_out,
                          int32_t* kv_lens_out);

/* Plan an append on the host only (step a1 of the path): for each i append
 * n_new[i] tokens to seqs[i] (distinct ids) in order.  The whole batch is
 * preflighted first ([P2] _blocks_needed_for_append, counting a copy for a
 * shared partial tail); on PA_ERR_POOL_EXHAUSTED nothing changes.  Then per
 * sequence a shared partial tail is replaced by a fresh block (a copy pair
 * (src, dst), [P1] _private_tail) and tokens are placed at
 * table[pos / block_size] * block_size + pos % block_size, a fresh block
 * being claimed at each boundary ([P1] append).
 * Outputs (host, may be NULL): slot_mapping_out [sum n_new] int64 in batch
 * order; cow_src_out/cow_dst_out [cow_cap] int32; n_cow_out.  INVALID_ARG if
 * more copies than cow_cap (checked before any change; at most n_seqs). */
pa_status pa_plan_append(pa_pool* pool, const int32_t* seqs,
                         const int32_t* n_new, int32_t n_seqs,
                         int64_t* slot_mapping_out, int32_t* cow_src_out,
                         int32_t* cow_dst_out, int32_t cow_cap,
                         int32_t* n_cow_out);

/* [P2] snapshot figures. */
pa_status pa_pool_stats(const pa_pool* pool, pa_stats* out);

/* Refcount of every block: out host [num_blocks] int32. */
pa_status pa_refcounts(const pa_pool* pool, int32_t* out);

/* [P2] validate: PA_OK, or PA_ERR_INTERNAL if an invariant is broken. */
pa_status pa_validate(const pa_pool* pool);

/* ---- device hot path ---------------------------------------------------- */

/* Append tokens to sequences and write their K/V into the pool:
 * pa_plan_append, then (on `stream`) the copy-on-write block copies, then
 * reshape_and_cache.  key/value: device [T, num_kv_heads, head_dim] in the
 * pool dtype, T = sum n_new, rows in batch order (all of seqs[0]'s new tokens
 * first).  slot_mapping_out: optional host [T] int64 copy of the plan.
 * Errors: those of pa_plan_append (no change), NO_DEVICE, CUDA. */
pa_status pa_append_kv(pa_pool* pool, const int32_t* seqs,
                       const int32_t* n_new, int32_t n_seqs, const void* key,
                       const void* value, int64_t* slot_mapping_out,
                       void* stream);

/* reshape_and_cache alone: k_cache[slot] = key[t], v_cache[slot] = value[t]
 * for t < T, all heads ([P1] append write).  d_slot_mapping: device [T]
 * int64; a negative slot skips the token; a slot >= num_blocks*block_size
 * sets PA_DEVERR_SLOT and skips it.  key/value: device [T, Hkv, d]. */
pa_status pa_reshape_and_cache(pa_pool* pool, const void* key,
                               const void* value,
                               const int64_t* d_slot_mapping, int32_t T,
                               void* stream);

/* Copy-on-write block copies: for i < n, whole block d_dst[i] := block
 * d_src[i] in both k_cache and v_cache, every slot and head
 * ([P1] _private_tail).  d_src/d_dst: device [n] int32; an id outside
 * [0, num_blocks) sets PA_DEVERR_BLOCK_ID and skips the pair.  Pairs must
 * not chain (no dst of one pair is the src of another). */
pa_status pa_cow_copy(pa_pool* pool, const int32_t* d_src,
                      const int32_t* d_dst, int32_t n, void* stream);

/* Scratch bytes pa_decode needs for a batch of B sequences with H query
 * heads and tables of width max_blocks (max kv_len = max_blocks *
 * block_size) at the given partition_tokens (0 = automatic choice).  0 when
 * no split is used. */
size_t pa_decode_workspace_bytes(const pa_pool* pool, int32_t B, int32_t H,
                                 int32_t max_blocks, int32_t partition_tokens);

/* Decode attention (q_tokens = 1, every cached token visible; [P3] with
 * q_tokens = 1, [P1] Eq. 3): out[b, h, :] = sum_j softmax_j(q[b,h].k_j *
 * scale) v_j over j < kv_lens[b], k_j/v_j of KV head h / (H / Hkv) read
 * through block_tables[b].
 *   q: device [B, H, head_dim], pool dtype (bf16 on an int8 or FP8 pool).
 *   out: device [B, H, head_dim] float32.  d_block_tables: device [B, max_blocks] int32.  d_kv_lens:
 *   device [B] int32 (0 gives a zero row).  scale: usually 1/sqrt(head_dim).
 *   partition_tokens: 0 = automatic, > 0 = split each sequence into
 *   partitions of that many tokens (a multiple of block_size) whose softmax
 *   statistics are merged by a log-sum-exp combine ([P4] recurrence applied
 *   across partitions).  workspace: device scratch of
 *   pa_decode_workspace_bytes bytes (16-byte aligned), may be NULL when that
 *   is 0.
 * Errors: INVALID_ARG (H not a multiple of Hkv, null/misaligned pointer,
 * workspace too small, partition not a multiple of block_size), NO_DEVICE,
 * CUDA. */
pa_status pa_decode(pa_pool* pool, const void* q, int32_t B, int32_t H,
                    const int32_t* d_block_tables, int32_t max_blocks,
                    const int32_t* d_kv_lens, float scale,
                    int32_t partition_tokens, void* workspace,
                    size_t workspace_bytes, float* out, void* stream);

/* Decode attention over a sink + recent window ([P2] streaming_keep_indices
 * with budget = sinks + window, and its sliding-window cache for sinks = 0):
 * key j of sequence b is visible iff j < kv_lens[b] and (j < sinks or
 * j >= kv_lens[b] - window); with kv_lens[b] <= sinks + window every key is.
 * The kernels walk only the blocks that hold a visible key, so a long
 * sequence costs about sinks + window tokens.  Arguments, layouts and errors
 * as pa_decode, plus window >= 1 and sinks >= 0 (else INVALID_ARG).  Shapes
 * outside the tensor-core kernels (fp32 pools, other head_dim or block sizes,
 * groups above 8) take the CUDA-core kernel, which walks the visible keys
 * only.  partition_tokens splits the walked blocks (tensor-core paths);
 * workspace: pa_decode_window_workspace_bytes bytes (0 on the CUDA-core
 * path). */
size_t pa_decode_window_workspace_bytes(const pa_pool* pool, int32_t B, int32_t H,
                                        int32_t max_blocks, int32_t window,
                                        int32_t sinks, int32_t partition_tokens);
pa_status pa_decode_window(pa_pool* pool, const void* q, int32_t B, int32_t H,
                           const int32_t* d_block_tables, int32_t max_blocks,
                           const int32_t* d_kv_lens, float scale, int32_t window,
                           int32_t sinks, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, float* out,
                           void* stream);

/* Decode step with the new token's append fused in: for each sequence b,
 * token kv_lens[b] - 1 is the one being decoded; its K/V rows
 * key[b]/value[b] (device [B, Hkv, head_dim], pool dtype) are written to pool
 * slot d_slot_mapping[b] (device [B] int64, from pa_plan_append; negative =
 * no write) and attended in the same pass -- the result equals
 * pa_reshape_and_cache followed by pa_decode ([P1] append, then Eq. 3).
 * Tables and kv_lens already include the new token; a copy-on-write the plan
 * asked for must have been issued (pa_cow_copy) on the same stream before.
 * On the tensor-core path it is one kernel; elsewhere the two calls.
 * Other arguments, workspace and errors as pa_decode. */
pa_status pa_decode_append(pa_pool* pool, const void* q, const void* key,
                           const void* value, const int64_t* d_slot_mapping,
                           int32_t B, int32_t H, const int32_t* d_block_tables,
                           int32_t max_blocks, const int32_t* d_kv_lens,
                           float scale, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, float* out,
                           void* stream);

/* pa_decode_append over a sink + recent window: writes each sequence's new
 * token (key/value [B, Hkv, head_dim] at d_slot_mapping[b], as
 * pa_decode_append) and decodes over the window exactly as pa_decode_window
 * -- the result equals pa_reshape_and_cache followed by pa_decode_window.
 * The new token, at kv_lens[b] - 1, is always visible.  One kernel on a
 * bf16 pool; two launches (quantising append, then the windowed decode) on
 * an int8 or FP8 pool.  Workspace: pa_decode_window_workspace_bytes bytes.
 * Errors as pa_decode_window, plus INVALID_ARG for null or misaligned key /
 * value / d_slot_mapping. */
pa_status pa_decode_window_append(pa_pool* pool, const void* q, const void* key,
                                  const void* value, const int64_t* d_slot_mapping,
                                  int32_t B, int32_t H, const int32_t* d_block_tables,
                                  int32_t max_blocks, const int32_t* d_kv_lens,
                                  float scale, int32_t window, int32_t sinks,
                                  int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, float* out, void* stream);

/* Chunked prefill attention ([P3] with q_tokens > 1): for each sequence b
 * the chunk's q_tokens queries are its last q_tokens positions; query qt
 * sees cached positions j <= kv_lens[b] - q_tokens + qt.  The chunk's own
 * K/V must already be in the pool (pa_append_kv).
 *   q: device [B, q_tokens, H, head_dim], pool dtype (bf16 on an int8 or FP8
 *   pool, whose records the CUDA-core path dequantises element by element).
 *   out: device [B, q_tokens, H, head_dim] float32.  Tables/kv_lens as
 *   pa_decode.
 *   max_kv_splits: on the tensor-core path, the query tiles of the last,
 *   partial wave of CTAs may be split over their keys (at most this many
 *   parts; 0 = automatic, up to 4; 1 = never) and merged with the [P4]
 *   log-sum-exp rule, so that the wave fills the GPU.  The split uses
 *   scratch owned by the pool (about 20 MB, allocated with it): calls on one
 *   pool that overlap on the GPU (unordered streams) race on it unless they
 *   pass 1.
 * Errors: as pa_decode (INVALID_ARG also for max_kv_splits < 0). */
pa_status pa_prefill_chunk(pa_pool* pool, const void* q, int32_t B,
                           int32_t q_tokens, int32_t H,
                           const int32_t* d_block_tables, int32_t max_blocks,
                           const int32_t* d_kv_lens, float scale,
                           int32_t max_kv_splits, float* out, void* stream);

/* ---- prepared decode batch --------------------------------------------- */

/* A serving decode loop in one call per step.  The pages' path for one step
 * is: plan each sequence's next token ([P1] append, [P2] preflight), copy a
 * shared partial tail ([P1] copy-on-write), write the new token's K/V and
 * attend over the cache ([P3] with q_tokens = 1).  A batch fixes the
 * sequences of such a loop once, keeps their block tables, lengths and
 * scratch on the device, and runs the whole step from host buffers.
 *
 * pa_batch_create: seqs (host, n distinct live sequences) of `pool`, queries
 * with H heads, tables up to max_blocks wide (a sequence may grow to
 * max_blocks * block_size tokens), partition_tokens as pa_decode.  Uploads
 * the current tables and allocates the batch's device buffers (two sets of
 * q, new K/V, output and staging), pinned staging mapped into the device's
 * address space, an upload stream and a download stream.
 * Errors: NO_DEVICE, UNKNOWN_SEQ, INVALID_ARG (n <= 0, a sequence twice, a
 * table wider than max_blocks, H not a multiple of num_kv_heads), CUDA. */
typedef struct pa_batch pa_batch; /* opaque */
pa_status pa_batch_create(pa_pool* pool, const int32_t* seqs, int32_t n,
                          int32_t H, int32_t max_blocks,
                          int32_t partition_tokens, pa_batch** out);

/* One decode step: appends one token to every sequence of the batch (the
 * plan runs on the host manager, all-or-nothing as pa_plan_append) and
 * decodes it.
 *   h_q: host [n, H, head_dim], h_key / h_value: host [n, Hkv, head_dim], all
 *   in the pool dtype (bf16 on an int8 or FP8 pool); h_out: host [n, H,
 *   head_dim] float32.  Use pinned host memory for asynchronous copies.
 * The plan, the table entries that changed since the previous step and the
 * inputs are uploaded on the batch's upload stream (highest priority): by one
 * kernel that reads the host buffers in place when all are pinned, mapped into
 * the device's address space and 16-byte aligned, the pool is bf16 or float32
 * and the step's upload is at most 1 MiB; else by one copy per buffer
 * (pageable memory works, synchronously slower); the table patches,
 * copy-on-write copies and the fused append + decode (pa_decode_append, or
 * pa_decode_window_append after pa_batch_set_window) run on `stream`; the
 * output is downloaded on the batch's download stream.  That download is
 * queued by the next pa_batch_step call, after the next step's uploads, or by
 * pa_batch_sync: queued ahead of the next uploads, a copy that waits for this
 * step's kernels would hold them up whenever the two copy streams share a
 * hardware queue.  Successive steps alternate two buffer sets, so a step's
 * transfers overlap its neighbours' kernels.  The call returns once the work
 * is queued: h_out holds the result after pa_batch_sync (pa_batch_free also
 * completes it), and the input buffers must not change before then.  The batch's sequences change only through the batch between
 * steps, or through pa_seq_truncate (any other change is picked up by
 * comparing whole tables).
 * Errors: those of pa_plan_append (nothing changes), UNKNOWN_SEQ (a sequence
 * was released), INVALID_ARG (a null pointer, a sequence at max_blocks *
 * block_size tokens), CUDA (the plan has been applied: treat the pool as
 * lost), and those of pa_decode_append. */
pa_status pa_batch_step(pa_batch* batch, const void* h_q, const void* h_key,
                        const void* h_value, float scale, float* h_out,
                        void* stream);

/* Undo the last step's token of every sequence of the batch (drafted tokens
 * that were not accepted): pa_seq_truncate to one token less, host-only.  A
 * copy-on-write the step made stays. */
pa_status pa_batch_rollback(pa_batch* batch);

/* Decode the batch's later steps over a sink + recent window: key j is
 * visible iff j < sinks or j >= kv_len - window ([P2] streaming_keep_indices
 * with budget = sinks + window, as pa_decode_window_append); window = 0
 * returns to full attention.  Waits for the device (the batch's partition
 * scratch may be resized), so it belongs between phases of a loop, not in
 * every step.  Errors: INVALID_ARG (window < 0, sinks < 0, sinks without a
 * window), CUDA. */
pa_status pa_batch_set_window(pa_batch* batch, int32_t window, int32_t sinks);

/* Wait until every step's output has reached its host buffer. */
pa_status pa_batch_sync(pa_batch* batch);

/* Synchronise the device and release the batch (never the pool). */
pa_status pa_batch_free(pa_batch* batch);

/* Bytes of the fixed device scratch array used by pa_decode_static_scratch. */
#define PA_STATIC_SCRATCH_BYTES (16u << 20)

/* pa_decode for callers that cannot allocate device memory.  The pages
 * describe no counterpart: this is an integration convenience of this
 * library.  A serving process that gives all device memory to its KV pool and
 * weights at start-up, or a plugin whose host framework owns the device
 * allocator, cannot provide pa_decode's workspace; this entry point takes the
 * partition scratch from a file-scope __device__ array of
 * PA_STATIC_SCRATCH_BYTES (16 MiB) that every GPU loading the library holds
 * until the process exits, and calls no cudaMalloc, cudaFree or other
 * allocating routine.  Arguments and results are those of pa_decode without
 * the workspace pair; it runs on the pool's device like every device call.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents.  Nothing in it needs to start at zero (each partition
 *     writes all its entries before they are read), but calls whose kernels
 *     overlap on the GPU (different streams, no ordering between them) race
 *     on the array.
 * Errors: those of pa_decode, plus PA_ERR_SCRATCH_LIMIT (nothing launched)
 * when pa_decode_workspace_bytes for this shape exceeds
 * PA_STATIC_SCRATCH_BYTES -- use fewer or larger partitions, or pa_decode. */
pa_status pa_decode_static_scratch(pa_pool* pool, const void* q, int32_t B,
                                   int32_t H, const int32_t* d_block_tables,
                                   int32_t max_blocks,
                                   const int32_t* d_kv_lens, float scale,
                                   int32_t partition_tokens, float* out,
                                   void* stream);

/* Synchronise the device, read and clear the pool's device error word.
 * *device_code = OR of PA_DEVERR_* bits seen since the last call.  Returns
 * PA_ERR_DEVICE when it is non-zero. */
pa_status pa_get_error(pa_pool* pool, int32_t* device_code);

/* Static description of a status code. */
const char* pa_status_string(pa_status status);

/* Which kernel family pa_decode / pa_prefill_chunk would use for this pool
 * and batch shape: 0 = generic CUDA-core kernel, 1 = the sm_100a fast path. */
int32_t pa_decode_path(const pa_pool* pool, int32_t H);
int32_t pa_prefill_path(const pa_pool* pool, int32_t H);

#ifdef __cplusplus
}
#endif
#endif /* PA_H_ */
