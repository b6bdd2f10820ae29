/*
 * pagedkv.h -- C ABI of the paged KV-cache hot path for NVIDIA B200 (sm_100a).
 *
 * What it computes (PagedAttention):
 *  - The KV cache of every request is split into fixed-size physical blocks of
 *    `block_size` tokens (16) that may sit anywhere in a pool shared by all
 *    requests; a per-request block table records which physical block holds
 *    each logical block, in order ("PagedAttention" glossary entry,
 *    ultralytics.com, section "Como funciona la paginacion"; iplexlaw.co.kr
 *    blog, section on logical order vs physical placement).
 *  - Token `pos` of a request lives at row (block_table[pos / block_size],
 *    pos % block_size) of the pool (same glossary entry, worked example).
 *  - The attention kernel gathers keys and values block by block through the
 *    table (same section); decode attention of one new token attends to the
 *    K and V of all previous tokens ("Le cache KV et PagedAttention",
 *    gyaansetu.com, section "Qu'est-ce que le KV Cache ?").
 *  - Blocks are shared between sequences through their tables, with a
 *    reference count per block; a writer copies a block others still use
 *    (copy-on-write) (glossary entry, section "Compartir bloques entre
 *    secuencias"; iplexlaw.co.kr, section "two answers to one request").
 *  - Grouped-query attention shares key/value heads among query heads; the
 *    cache may be stored in FP8 (glossary entry, section "Tecnicas
 *    relacionadas").
 *
 * Data layout (all row-major, C order):
 *  - pools:        [num_blocks][block_size][num_kv_heads][head_dim]; K and V in
 *                  separate pools of the same shape and dtype.  A slot is
 *                  block * block_size + offset, so the pools are also
 *                  [num_blocks * block_size][num_kv_heads][head_dim].
 *  - block_tables: int32 [num_seqs][max_blocks_per_seq]; entries at or past
 *                  ceil(context_len / block_size) are never read (any padding).
 *  - context_lens: int32 [num_seqs], including the token written this step.
 *  - q, out:       [num_seqs][num_heads][head_dim]; query head h uses key/value
 *                  head h / (num_heads / num_kv_heads).
 *  - new k, v:     [num_tokens][num_kv_heads][head_dim].
 *
 * Conventions for every call below:
 *  - Pointers are caller-owned DEVICE pointers unless stated otherwise; the
 *    library never frees or retains them.  The compute calls allocate no
 *    memory; the decode's scratch is the caller's `workspace`.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  A return of PKV_OK means the work was enqueued.
 *  - Host-side argument errors are returned synchronously and nothing is
 *    launched.  Errors in DEVICE data (a slot or block id out of range, a
 *    context length above the stated bounds) cannot be seen by the host without
 *    a synchronisation: the kernels skip the offending item and, when
 *    `err_count` is non-NULL, atomically add the number of such items to the
 *    int32 it points to (device memory).  Nothing traps.
 *  - Kernels never wait on another GPU or another launch; their only waits are
 *    on their own asynchronous copies, each bounded in time.  A wait that runs
 *    out (a hardware fault, not a data error) abandons that work, adds 1 to
 *    *err_count and sets the timeout word of the decode workspace.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_VERSION 1
#define PKV_BLOCK_SIZE 16

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_EINVAL = 1,        /* bad argument: NULL pointer, bad size, misaligned pointer, small workspace */
    PKV_EUNSUPPORTED = 2,  /* valid but not implemented: block_size, head_dim, dtype combination, group */
    PKV_ECUDA = 3,         /* a CUDA runtime/driver call failed (launch error, no device) */
    PKV_ENOMEM = 4,        /* block manager: not enough free blocks */
    PKV_ENOENT = 5,        /* block manager: no such sequence */
    PKV_ESWAPPED = 6       /* block manager: the sequence is swapped out to the host pool */
} pkv_status;

typedef enum pkv_dtype {
    PKV_F32 = 0,           /* IEEE binary32 */
    PKV_BF16 = 1,          /* bfloat16 */
    PKV_FP8_E4M3 = 2       /* OCP OFP8 E4M3 (bias 7, max 448, no infinities) */
} pkv_dtype;

/* Human-readable name of a pkv_status value (static string, never NULL). */
const char* pkv_status_string(int status);

/* PKV_VERSION of the loaded library. */
int pkv_version(void);

/* ------------------------------------------------------------------------
 * KV append ("reshape and cache"): store the K and V of new tokens.
 * Source: the KV cache keeps every token's K and V and each generation step
 * appends only the new token's ("Le cache KV et PagedAttention", section
 * "Qu'est-ce que le KV Cache ?"); slot addressing from the glossary entry's
 * worked example.
 *
 *   k, v          [num_tokens][num_kv_heads][head_dim] in src_dtype
 *   slot_mapping  int64 [num_tokens]; token i goes to pool row slot_mapping[i];
 *                 a negative slot is padding and is skipped; a slot
 *                 >= num_blocks * block_size is skipped and counted.
 *   k_pool, v_pool [num_blocks][block_size][num_kv_heads][head_dim] in cache_dtype
 *   k_scale, v_scale  host floats, used only for an FP8 cache: the stored
 *                 code is E4M3(x / scale) with IEEE fp32 division, round to
 *                 nearest even, saturating to +-448.
 * Supported (src_dtype, cache_dtype): (F32, F32), (BF16, BF16), (BF16, FP8_E4M3),
 * (F32, FP8_E4M3).  Same-dtype writes are byte copies.
 * Requirements: block_size == 16; num_kv_heads * head_dim * element size a
 * multiple of 16 bytes; all pointers 16-byte aligned; num_tokens >= 0
 * (0 launches nothing).  Two tokens with the same slot race (last writer
 * undefined).
 * ---------------------------------------------------------------------- */
int pkv_paged_kv_write(const void* k, const void* v, int src_dtype,
                       const int64_t* slot_mapping, int num_tokens,
                       void* k_pool, void* v_pool, int cache_dtype,
                       int num_blocks, int block_size, int num_kv_heads, int head_dim,
                       float k_scale, float v_scale,
                       int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Workspace bytes that pkv_paged_attention_decode needs for these bounds.
 * `max_context_len` bounds every context_lens entry; `partition_tokens` is
 * the value that will be passed to the decode (0 = automatic).  Returns 0 for
 * invalid arguments.  The workspace holds the partition plan, a work counter
 * and the per-partition partial results (fp32) of split contexts.
 * ---------------------------------------------------------------------- */
size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                  int max_context_len, int partition_tokens);

/* ------------------------------------------------------------------------
 * Single-query decode attention over a paged KV cache.
 * Source: the attention kernel reads a request's keys and values through its
 * block table, block by block, in logical order (glossary entry, section
 * "Como funciona la paginacion"; iplexlaw.co.kr, logical vs physical order);
 * FlashAttention-style tiling that never writes the full score matrix to HBM
 * (glossary entry, section "Tecnicas relacionadas"); grouped-query attention
 * (same section).  The formula is softmax(q K^T * scale) V.
 *
 *   out     [num_seqs][num_heads][head_dim] in q_dtype (written)
 *   q       [num_seqs][num_heads][head_dim] in q_dtype
 *   k_pool, v_pool  as for pkv_paged_kv_write, in cache_dtype
 *   block_tables int32 [num_seqs][max_blocks_per_seq]
 *   context_lens int32 [num_seqs]; a length 0 yields a zero output row.
 *   max_context_len  host-side upper bound of every context length (sizes the
 *           workspace; a larger device value is clamped and counted)
 *   scale   softmax scale (typically 1/sqrt(head_dim))
 *   k_scale, v_scale  per-tensor dequantisation scales of an FP8 cache
 *           (value = E4M3 code value * scale); ignored for F32/BF16 caches
 *   partition_tokens  0: the library splits long contexts into partitions of
 *           a size it picks on the device from the actual lengths; > 0: split
 *           every context into partitions of exactly this many tokens (a
 *           multiple of block_size).  Partitions are merged with a
 *           log-sum-exp weighted sum.  The result does not depend on which
 *           GPU thread processes which partition.
 *   workspace, workspace_bytes  device scratch of at least
 *           pkv_decode_workspace_bytes(...) bytes, 256-byte aligned.  Its
 *           contents need no initialisation and are overwritten; calls that
 *           share one workspace must be ordered on the GPU (same stream).
 * Supported (q_dtype, cache_dtype): (F32, F32), (BF16, BF16), (BF16, FP8_E4M3).
 * head_dim 64 or 128 (FP8: 128); num_heads % num_kv_heads == 0 and, for BF16
 * and FP8 caches, num_heads / num_kv_heads <= 16; block_size == 16.
 * Errors: PKV_EINVAL for NULL pointers (out, q, pools, tables, lens, workspace),
 * non-positive sizes, num_heads % num_kv_heads != 0, pointers not 16-byte
 * aligned, a bad partition size or a workspace that is too small;
 * PKV_EUNSUPPORTED outside the table above; PKV_ECUDA on a launch failure.
 * ---------------------------------------------------------------------- */
int pkv_paged_attention_decode(void* out, const void* q, int q_dtype,
                               const void* k_pool, const void* v_pool, int cache_dtype,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs, int max_context_len,
                               int num_blocks, int block_size, int num_heads, int num_kv_heads,
                               int head_dim, float scale, float k_scale, float v_scale,
                               int partition_tokens, void* workspace, size_t workspace_bytes,
                               int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Decode attention that allocates nothing and takes no workspace.
 * The pages have no counterpart to this call: it exists for callers that
 * cannot allocate device memory where they run the decode (a plug-in inside a
 * host program that owns all device memory, a loop that must not call
 * cudaMalloc/cudaFree because they synchronise the device, a latency budget
 * that allocation would break).
 *
 * Same arguments, layouts, computation and errors as
 * pkv_paged_attention_decode, without `workspace` / `workspace_bytes`: the
 * scratch is a device array of PKV_NOALLOC_SCRATCH_BYTES that the library
 * declares at file scope.  Every GPU that loads the library's kernels holds
 * that array until the process exits.
 *  - Checks: first every argument check of pkv_paged_attention_decode (same
 *    statuses: PKV_EUNSUPPORTED for an unsupported configuration whatever its
 *    size), then the limit: PKV_EINVAL, before any CUDA call, when the scratch
 *    these bounds need (pkv_decode_workspace_bytes(num_seqs, num_heads,
 *    head_dim, max_context_len, partition_tokens)) exceeds
 *    PKV_NOALLOC_SCRATCH_BYTES; a need of exactly that size is accepted.  A
 *    larger partition_tokens lowers the need.
 *  - The first call in a device's context looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it for later
 *    calls in the same context; a context that was destroyed and created again
 *    (cudaDeviceReset) is recognised by its driver context id and gets a new
 *    lookup.  Make the first call on each device before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents;
 *    nothing in it needs clearing (each call's first kernel rewrites what the
 *    others read).  Calls whose GPU work overlaps (different streams without
 *    ordering between them) race on it: order them on one stream.
 *  - Calls no cudaMalloc, cudaFree or allocating library routine.
 * ---------------------------------------------------------------------- */
#define PKV_NOALLOC_SCRATCH_BYTES (32u << 20)

int pkv_paged_attention_decode_noalloc(void* out, const void* q, int q_dtype,
                                       const void* k_pool, const void* v_pool, int cache_dtype,
                                       const int32_t* block_tables, int max_blocks_per_seq,
                                       const int32_t* context_lens, int num_seqs, int max_context_len,
                                       int num_blocks, int block_size, int num_heads, int num_kv_heads,
                                       int head_dim, float scale, float k_scale, float v_scale,
                                       int partition_tokens, int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Shared-prefix decode: the same attention as pkv_paged_attention_decode, but
 * sequences that begin with the same physical blocks read those blocks once
 * for all of them.  Source: block tables let several sequences point at the
 * same physical blocks -- parallel samples, beams, requests that start with the
 * same system prompt reuse one copy of the shared prefix (glossary entry
 * "PagedAttention", section "Compartir bloques entre secuencias"; full-block
 * hashing extends this across requests, same section).
 *
 * Extra arguments (device pointers, int32):
 *   group_offsets        [num_groups + 1]  group g is group_seqs[offsets[g] .. offsets[g+1])
 *   group_seqs           [num_group_seqs]  batch indices (0 .. num_seqs-1) of its members
 *   group_shared_blocks  [num_groups]      leading blocks the members are said to share
 * These are hints (pkv_bm_prefix_groups computes them): the plan keeps a
 * member only if it is in range and in no group claimed before (claim order
 * between groups is unspecified), and cuts a group's shared blocks to those
 * every kept member holds in full (16 tokens within its context); each work
 * item over shared blocks checks that its members' tables name the same
 * physical blocks and, where they do not, runs once per member.  A wrong hint
 * costs time, never correctness.  Up to 512 members per group are
 * considered.  The result equals pkv_paged_attention_decode's up to rounding
 * (partitions are cut differently: each sequence's shared and own blocks
 * separately).  Grouping applies to bf16 caches with head_dim 128 and at most 8
 * query heads per KV head (a member's heads and its group-mates' fill 16 score
 * columns); other configurations ignore the hints and run the plain decode.
 *
 * workspace: pkv_decode_workspace_bytes_shared(...) bytes (a little more than
 * the plain decode's).  num_groups == 0 runs the plain decode in that layout.
 * ---------------------------------------------------------------------- */
size_t pkv_decode_workspace_bytes_shared(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                         int partition_tokens);

int pkv_paged_attention_decode_shared(void* out, const void* q, int q_dtype,
                                      const void* k_pool, const void* v_pool, int cache_dtype,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int num_seqs, int max_context_len,
                                      int num_blocks, int block_size, int num_heads, int num_kv_heads,
                                      int head_dim, float scale, float k_scale, float v_scale,
                                      int partition_tokens,
                                      const int32_t* group_offsets, const int32_t* group_seqs,
                                      int num_group_seqs, const int32_t* group_shared_blocks, int num_groups,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Causal multi-token attention (the prompt pass) through block tables.
 * Source: a prompt's blocks are allocated first and its last block then
 * filled; attention reads the blocks through the table in logical order
 * (iplexlaw.co.kr, section on logical vs physical order); each token attends
 * to all the tokens before it (gyaansetu.com, what the KV cache holds).
 *
 * Sequence s has nq_s = query_start[s+1] - query_start[s] new query tokens:
 * the last nq_s of its context_lens[s] tokens, whose K/V are already in the
 * pools (pkv_paged_kv_write with the prompt's slots).  Query row
 * r = query_start[s] + i sits at position context_lens[s] - nq_s + i and
 * attends to tokens 0 .. that position.  A whole prompt, a prompt after a
 * cached prefix and a chunk of a long prompt are all this call.
 *   out, q          [total_query_tokens][num_heads][head_dim]
 *   block_tables    int32 [num_seqs][max_blocks_per_seq]
 *   context_lens    int32 [num_seqs]; query_start int32 [num_seqs + 1], query_start[0] = 0,
 *                   query_start[num_seqs] = total_query_tokens
 *   max_query_len   >= every nq_s (sizes the launch; rows past it are not computed)
 *   k_scale, v_scale  FP8 cache only (ignored for bf16): a stored code c stands
 *                   for c * k_scale (c * v_scale), as pkv_paged_kv_write quantised it
 * Supported: bf16 q, bf16 or FP8 E4M3 cache, head_dim 128, block_size 16, any
 * GQA group.  The product runs on the tcgen05 tensor cores (TMEM
 * accumulators).  With an FP8 cache the codes become f16 in shared memory
 * (exactly) and q is taken into f16 (exact inside the f16 range; entries past
 * +-65504 saturate there), so both operands of every product are f16.
 * Host errors, returned before any CUDA call: PKV_EINVAL for negative sizes,
 * max_blocks_per_seq <= 0, num_heads not a multiple of num_kv_heads, a null
 * pointer, a pointer not 16-byte (out, q, pools) or 4-byte (int32 arrays)
 * aligned, or a non-finite k_scale / v_scale with an FP8 cache;
 * PKV_EUNSUPPORTED for another dtype, head_dim or block_size, more than
 * 65,535 sequences or heads, or a max_query_len above 65,535 x 256 tokens.
 * No sequences or no queries: PKV_OK, nothing runs.
 * Device-data errors (a table entry out of range among the blocks a sequence
 * reads: its tokens are left out; nq_s > context_lens[s] or a context longer
 * than the table: the sequence's rows are zeroed) are counted into err_count.
 * ---------------------------------------------------------------------- */
int pkv_paged_attention_prefill(void* out, const void* q, int q_dtype,
                                const void* k_pool, const void* v_pool, int cache_dtype,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, const int32_t* query_start, int num_seqs,
                                int total_query_tokens, int max_query_len, int num_blocks, int block_size,
                                int num_heads, int num_kv_heads, int head_dim, float scale,
                                float k_scale, float v_scale, int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Copy-on-write block copy: for every pair (src, dst) copy the whole physical
 * block src over block dst, in both pools.
 * Source: before a sequence writes into a block that other sequences still
 * use, the engine first copies that block (glossary entry, section "Compartir
 * bloques entre secuencias"); full shared blocks stay shared and only the block
 * that must split is copied (iplexlaw.co.kr, "two answers to one request").
 *
 *   k_pool, v_pool  pools (any dtype), each num_blocks blocks of block_bytes
 *   block_bytes     bytes of one block of one pool
 *                   (block_size * num_kv_heads * head_dim * element size);
 *                   a multiple of 16
 *   src_dst_pairs   DEVICE int64 [num_pairs][2]
 * A pair with an id outside [0, num_blocks) is skipped and counted.  A dst that
 * repeats, or a dst that is also a src, gives an undefined result (the block
 * manager never emits such lists).  num_pairs == 0 launches nothing.
 * ---------------------------------------------------------------------- */
int pkv_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes,
                    const int64_t* src_dst_pairs, int num_pairs, int num_blocks,
                    int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Block swap between pools: for every pair (src, dst) copy the whole block src
 * of the source pools over block dst of the destination pools (K and V).
 * Source: when memory runs out, small pages are moved to the CPU instead of
 * whole sequences, and brought back later ("Le cache KV et PagedAttention",
 * gyaansetu.com, section "Comment PagedAttention resout ce probleme": fine-
 * grained eviction); with pkv_copy_blocks it is the copy of one page.
 *
 *   dst_k_pool, dst_v_pool  dst_num_blocks blocks of block_bytes each
 *   src_k_pool, src_v_pool  src_num_blocks blocks of block_bytes each
 *   src_dst_pairs           int64 [num_pairs][2], device-accessible
 * Any pointer may be device memory or page-locked host memory that the device
 * can address (cudaHostAlloc, torch pin_memory): the GPU moves the bytes over
 * the host link itself, so swap-out is (device pool -> host pool) and swap-in
 * (host pool -> device pool).  Pageable host memory is refused (PKV_EINVAL).
 * Pairs out of range are skipped and counted; a dst that repeats gives an
 * undefined result.  num_pairs == 0 launches nothing.
 * ---------------------------------------------------------------------- */
int pkv_swap_blocks(void* dst_k_pool, void* dst_v_pool, int dst_num_blocks,
                    const void* src_k_pool, const void* src_v_pool, int src_num_blocks,
                    size_t block_bytes, const int64_t* src_dst_pairs, int num_pairs,
                    int32_t* err_count, void* stream);

/* ------------------------------------------------------------------------
 * Host block manager (CPU only; no CUDA calls).  It decides where tokens go:
 * lazy allocation of a new block only when the last one is full, taken from
 * the front of a first-in first-out free list (glossary entry, worked example
 * and "Como funciona la paginacion"; iplexlaw.co.kr: allocate the prompt first,
 * then fill the last block); per-block reference counts, fork for parallel
 * sampling and copy-on-write of a partly filled shared last block; finished
 * sequences return their blocks at once (glossary entry, sections on sharing
 * and on continuous batching).  Freed blocks are appended to the back of the
 * free list in table order.  Not thread-safe: one manager per thread.
 * All pointers here are HOST pointers.
 * ---------------------------------------------------------------------- */
typedef struct pkv_block_manager pkv_block_manager;

/* free_order: optional order of the initial free list (NULL = 0..num_blocks-1);
 * it may name a subset of the blocks (the rest are owned elsewhere). */
int pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order, int free_count,
                  pkv_block_manager** out);
void pkv_bm_destroy(pkv_block_manager* bm);
/* New sequence holding num_tokens prompt tokens (ceil(n / block_size) blocks). */
int pkv_bm_alloc_seq(pkv_block_manager* bm, int num_tokens, int32_t* seq_out);
/* New sequence sharing every block of `parent` (reference counts + 1). */
int pkv_bm_fork(pkv_block_manager* bm, int32_t parent, int32_t* child_out);
/* Batched fork / free (one call for a whole step of beam search): fork_many
 * forks parents[i] into children_out[i] in order; free_many frees seqs[0..n)
 * in order (each at most once).  Arguments are checked before anything
 * changes. */
int pkv_bm_fork_many(pkv_block_manager* bm, const int32_t* parents, int n, int32_t* children_out);
int pkv_bm_free_many(pkv_block_manager* bm, const int32_t* seqs, int n);
/* Reserve one new token slot for each of seqs[0..n) in that order.  slots_out
 * [n] receives the slots; cow_pairs_out [n][2] receives the (src, dst) block
 * pairs to copy before writing (num_pairs_out of them).  On PKV_ENOMEM the
 * sequences before the failing one keep their new slots (reported through
 * *num_done_out when non-NULL) and the failing one is unchanged. */
int pkv_bm_append_tokens(pkv_block_manager* bm, const int32_t* seqs, int n, int64_t* slots_out,
                         int64_t* cow_pairs_out, int* num_pairs_out, int* num_done_out);
/* Drop a sequence; blocks whose count reaches 0 return to the free list. */
int pkv_bm_free_seq(pkv_block_manager* bm, int32_t seq);
int pkv_bm_num_free(const pkv_block_manager* bm);
int pkv_bm_seq_len(const pkv_block_manager* bm, int32_t seq, int32_t* len_out);
int pkv_bm_refcount(const pkv_block_manager* bm, int32_t block, int32_t* rc_out);
/* Copy a sequence's table (n_out entries) into out[0..cap). */
int pkv_bm_block_table(const pkv_block_manager* bm, int32_t seq, int32_t* out, int cap, int* n_out);
/* Slots of positions [start, start + count) of a sequence. */
int pkv_bm_slots(const pkv_block_manager* bm, int32_t seq, int start, int count, int64_t* out);
/* Padded tables [n][max_blocks] (pad value `pad`) and lengths [n] of seqs[0..n). */
int pkv_bm_tables(const pkv_block_manager* bm, const int32_t* seqs, int n, int32_t* tables,
                  int max_blocks, int32_t pad, int32_t* lens);
/* Current free list, front first (n_out entries). */
int pkv_bm_free_list(const pkv_block_manager* bm, int32_t* out, int cap, int* n_out);

/* Prefix caching across requests (full-block hashing: the glossary entry's
 * sharing section says hashing whole blocks extends sharing to separate
 * requests, which is how prompt caching is implemented).  With the cache on,
 * alloc_seq_tokens registers every full block of a prompt under the key
 * (parent block's registration, its block_size token ids); a later prompt
 * that begins with the same tokens gets the same physical blocks for its
 * longest run of matching leading full blocks (reference counts + 1) and
 * *num_cached_out = that run x block_size: the caller writes K/V only for
 * tokens [num_cached, num_tokens).  Keys hold the exact tokens (a hash picks
 * the bucket only), so different prefixes never collide.  A registered block
 * whose count drops to 0 keeps its contents and its key and goes to the back
 * of the free list; a hit takes it back out; when the free list hands it out
 * for new data its key is dropped.  Only prompt blocks are registered (tokens
 * appended later carry no ids here); registered blocks are always full, so
 * copy-on-write never touches them.  PKV_ENOMEM (nothing changed) if the
 * blocks that are not hits, plus the hits that must leave the free list, do
 * not fit.  With the cache off, alloc_seq_tokens is alloc_seq; turning it off
 * forgets every key. */
int pkv_bm_set_prefix_cache(pkv_block_manager* bm, int enable);
int pkv_bm_alloc_seq_tokens(pkv_block_manager* bm, const int32_t* tokens, int num_tokens, int32_t* seq_out,
                            int* num_cached_out);
int pkv_bm_num_cached_blocks(const pkv_block_manager* bm);

/* Shared-prefix hints for pkv_paged_attention_decode_shared, for the batch
 * seqs[0..n) (in that order: members are given as batch indices 0..n-1).
 * Resident sequences holding at least one full block are grouped by the
 * physical id of their first block, in order of first appearance; groups of at
 * least two members are emitted, members in batch order, and a group's shared
 * count is the number of leading table entries equal in all its members and
 * full (16 tokens) in every member.  Outputs: group_offsets [n + 1],
 * group_seqs [n], group_shared_blocks [n] (capacity n each),
 * *num_groups_out groups, group_offsets[*num_groups_out] = members written.
 * Unknown sequences return PKV_ENOENT, swapped ones PKV_ESWAPPED. */
int pkv_bm_prefix_groups(const pkv_block_manager* bm, const int32_t* seqs, int n, int32_t* group_offsets,
                         int32_t* group_seqs, int32_t* group_shared_blocks, int* num_groups_out);

/* Host pool for swapping (fine-grained eviction, see pkv_swap_blocks): give the
 * manager num_host_blocks host blocks (ids 0..n-1, free list in id order).
 * swap_out moves a resident sequence's pages to host blocks: it appends one
 * (device block, host block) pair per table entry to pairs_out (capacity =
 * table length), drops the sequence's references to its device blocks (a block
 * another sequence still uses stays on the device) and leaves the sequence
 * "swapped" (its table now holds host ids).  swap_in is the reverse: fresh
 * device blocks from the free list, (host block, device block) pairs, host
 * blocks freed.  Both return PKV_ENOMEM, with nothing changed, if the target
 * pool has too few free blocks, and PKV_EINVAL if cap is below the table
 * length.  A page shared with another sequence is copied out like any other,
 * and comes back as a private block: sharing is not restored.  A swapped
 * sequence can be swapped in, freed (its host blocks return to the host free
 * list) or queried (seq_len, block_table: host ids, is_swapped); fork,
 * append_tokens, slots and tables return PKV_ESWAPPED.  set_host_pool returns
 * PKV_EINVAL while any host block is in use. */
int pkv_bm_set_host_pool(pkv_block_manager* bm, int num_host_blocks);
int pkv_bm_swap_out(pkv_block_manager* bm, int32_t seq, int64_t* pairs_out, int cap, int* num_pairs_out);
int pkv_bm_swap_in(pkv_block_manager* bm, int32_t seq, int64_t* pairs_out, int cap, int* num_pairs_out);
int pkv_bm_is_swapped(const pkv_block_manager* bm, int32_t seq, int* swapped_out);
int pkv_bm_num_free_host(const pkv_block_manager* bm);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
