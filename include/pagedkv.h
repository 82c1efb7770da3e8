/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged KV-cache write and decode
 * attention on NVIDIA B200 (sm_100a), plus the host block allocator that
 * builds block tables.
 *
 * Sources (web pages describing vLLM's paged KV cache):
 *   [YK] "大模型推理框架 vLLM 源码解析 一" (ai.yueke.cloud), section 三
 *        "vLLM 源码关键路径解析": the cache shape
 *        [num_blocks, block_size, num_heads, head_dim]; paged_attention_v1
 *        takes (query, key_cache, value_cache, block_tables, context_lens);
 *        for token j of sequence i the physical block is
 *        block_tables[i][j // block_size] and the in-block offset is
 *        j % block_size.  Section 二: BlockAllocator.allocate() returns a
 *        list of physical block ids.  Section 四 step 4: --block-size
 *        defaults to 16; 32 reduces block-table lookups.
 *   [FC] "23.1 vLLM：高吞吐推理框架原理与部署" (r.flycode100.com), section 二
 *        "PagedAttention 的核心原理": parts 1-2 (fixed blocks of 16 tokens,
 *        one block allocated on arrival and one more every 16 tokens, a
 *        block table keeps the logical order, blocks return to a shared free
 *        pool when the request ends) and part 3 (prefix blocks are shared
 *        between parallel samples / beams and copied only when a sequence
 *        writes into a shared block: copy-on-write).
 *   [MH] "大模型推理框架VLLM-0.7.3源码" (mhpq.cn), sections 2.1 and 3.3: the
 *        model runner builds block_tables and slot_mapping; slot_mapping
 *        tells the operator into which cell each current token's K/V goes.
 *
 * Conventions for every call below:
 *   - Device pointers are caller-owned (the library never allocates or frees
 *     device memory and never synchronises the device inside compute calls).
 *     One exception: a fixed PKV_STATIC_WORKSPACE_BYTES (16 MiB) array in
 *     device memory on every GPU that loads the library, used only by
 *     pkv_paged_attention_decode_static_workspace (declared below).
 *     Tensors are dense and row-major in the shapes given; K/V/query/output
 *     pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Compute calls are asynchronous on it.  The returned status
 *     covers host-side validation and the launch; errors found while the
 *     kernels run (a slot, block id or context length outside its range,
 *     or a bounded wait that expired) set bits in a per-device flag word read
 *     by pkv_device_flags().  Kernels never trap.
 *   - Element types: PKV_F16 (IEEE binary16) or PKV_BF16 (bfloat16); the
 *     query, caches and output share one type.  Scores, softmax and
 *     accumulation are fp32; the output is rounded to nearest even.
 *   - Supported shapes: head_dim in {64, 128}; block_size in {16, 32};
 *     num_heads % num_kv_heads == 0 with group size 1..8;
 *     num_blocks * block_size < 2^31.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size */
    PKV_ERR_UNSUPPORTED = 2,   /* shape outside the compiled set (see above) */
    PKV_ERR_OUT_OF_RANGE = 3,  /* a host-visible index outside its pool */
    PKV_ERR_OOM = 4,           /* allocator: not enough free blocks (nothing taken) */
    PKV_ERR_CUDA = 5,          /* a CUDA runtime call failed; see pkv_last_error() */
    PKV_ERR_WORKSPACE = 6,     /* workspace missing or smaller than required */
    PKV_ERR_MISALIGNED = 7     /* a pointer is not 16-byte aligned */
} pkv_status;

typedef enum { PKV_F16 = 0, PKV_BF16 = 1 } pkv_dtype;

/* Device flag bits (pkv_device_flags). */
#define PKV_DEVFLAG_SLOT_RANGE    0x1u  /* write: slot >= num_blocks*block_size (token skipped) */
#define PKV_DEVFLAG_BLOCK_RANGE   0x2u  /* decode: table entry outside [0, num_blocks) (block 0 read instead) */
#define PKV_DEVFLAG_CONTEXT_RANGE 0x4u  /* decode: context_len < 0 or > max_blocks*block_size (clamped) */
#define PKV_DEVFLAG_WAIT_TIMEOUT  0x8u  /* decode: a shared-memory pipeline wait gave up (output invalid) */

/* Human-readable name of a status code (static string). */
const char *pkv_status_str(pkv_status s);

/* Detail of the last failing call on this host thread ("" if none). */
const char *pkv_last_error(void);

/* Library version string, e.g. "pagedkv 0.1.0 sm_100a". */
const char *pkv_version(void);

/*
 * Read (and with clear != 0, reset) the device flag word of `device`.
 * Synchronous: waits for all prior work on that device.
 */
pkv_status pkv_device_flags(int device, unsigned int *flags, int clear);

/*
 * Failure-detection self-test: launches one warp that waits, through the
 * decode kernel's bounded shared-memory pipeline wait, on a barrier phase
 * that nothing completes.  After limit_ns (0 < limit_ns <= 1e10) the wait
 * gives up, PKV_DEVFLAG_WAIT_TIMEOUT is set and the kernel returns; the
 * context stays usable.  Asynchronous on `stream`.
 */
pkv_status pkv_selftest_bounded_wait(int64_t limit_ns, void *stream);

/*
 * kv_cache_write -- store the current tokens' K/V into their cache cells
 * ([MH] 2.1, 3.3; cache shape [YK] 三).
 *
 *   key, value     [num_tokens, num_kv_heads, head_dim]   device, read
 *   slot_mapping   [num_tokens] int64                      device, read
 *   key_cache,
 *   value_cache    [num_blocks, block_size, num_kv_heads, head_dim]  device, written
 *
 * For token t with s = slot_mapping[t] >= 0 and every kv head h:
 *   key_cache[s / block_size, s % block_size, h, :] = key[t, h, :]   (bit copy)
 * and likewise for V.  s < 0 marks a padding token (skipped).  Slots must be
 * unique within a call (duplicates race).  A slot >= num_blocks*block_size
 * is skipped and sets PKV_DEVFLAG_SLOT_RANGE.  num_tokens == 0 is a no-op.
 */
pkv_status pkv_kv_cache_write(const void *key, const void *value,
                              const int64_t *slot_mapping, int64_t num_tokens,
                              int num_kv_heads, int head_dim,
                              void *key_cache, void *value_cache,
                              int64_t num_blocks, int block_size,
                              pkv_dtype dtype, void *stream);

/*
 * copy_blocks -- whole-block copies for copy-on-write and swapping ([FC] 二.3:
 * a shared block is copied before a sequence writes into it; [YK] 三: the
 * scheduler swaps a sequence's KV blocks out to CPU memory when the pool runs
 * short and back in later).
 *
 *   src_key_cache, src_value_cache   [src_num_blocks, block_bytes]   read
 *   dst_key_cache, dst_value_cache   [dst_num_blocks, block_bytes]   written
 *   block_mapping                    [num_pairs][2] int32 (src, dst)  read
 *
 * Pair i copies source block block_mapping[i][0] to destination block
 * block_mapping[i][1], K and V, bit for bit.  Caches and mapping are device
 * memory or pinned host memory (reached through unified addressing), so the
 * same call does copy-on-write inside one pool (source = destination caches),
 * swap-out to host and swap-in.  block_bytes = block_size * num_kv_heads *
 * head_dim * 2, a multiple of 16 (else PKV_ERR_UNSUPPORTED).  Destination
 * blocks must be distinct and not also sources in the same call.  num_pairs
 * is below 2^30 (two CTAs per pair, one for K and one for V, and a grid holds
 * fewer than 2^31; else PKV_ERR_UNSUPPORTED);
 * caches 16-byte aligned and the mapping 8-byte aligned (else
 * PKV_ERR_MISALIGNED).  Out-of-range pairs are skipped and set
 * PKV_DEVFLAG_BLOCK_RANGE.
 */
pkv_status pkv_copy_blocks(const void *src_key_cache, const void *src_value_cache,
                           void *dst_key_cache, void *dst_value_cache,
                           const int32_t *block_mapping, int num_pairs,
                           int64_t src_num_blocks, int64_t dst_num_blocks, int64_t block_bytes,
                           void *stream);

/*
 * Partition plan of a decode call: the partition length in tokens the call
 * will use (a multiple of block_size) and the number of partitions per
 * sequence (1 = single pass, no workspace).  partition_tokens: > 0 requests
 * that length (rounded up to a block multiple), 0 = automatic, < 0 = never
 * split.  Returns PKV_ERR_INVALID_ARG / PKV_ERR_UNSUPPORTED on bad shapes.
 */
pkv_status pkv_decode_plan(int batch, int num_heads, int num_kv_heads, int head_dim,
                           int max_blocks, int block_size, int partition_tokens,
                           int *plan_partition_tokens, int *plan_num_partitions);

/*
 * Bytes of device workspace pkv_paged_attention_decode needs for these
 * arguments (0 when the plan is a single pass).  The workspace holds, per
 * (sequence, query head, partition), the partition's running max, softmax
 * normaliser and normalised fp32 output row.
 */
size_t pkv_decode_workspace_bytes(int batch, int num_heads, int num_kv_heads, int head_dim,
                                  int max_blocks, int block_size, int partition_tokens);

/*
 * paged_attention_decode -- one query token per sequence attends over its
 * KV cache, scattered across fixed-size physical blocks located through the
 * block table ([YK] 三 paged_attention_v1; [FC] 二.2 step 3).
 *
 *   query          [batch, num_heads, head_dim]                      device, read
 *   key_cache,
 *   value_cache    [num_blocks, block_size, num_kv_heads, head_dim]  device, read
 *   block_tables   [batch, max_blocks] int32                         device, read
 *   context_lens   [batch] int32                                     device, read
 *   out            [batch, num_heads, head_dim]                      device, written
 *   workspace      pkv_decode_workspace_bytes(...) bytes             device, scratch
 *
 * For sequence b, query head h (kv head h / (num_heads/num_kv_heads)) and
 * L = context_lens[b]:
 *   s_j   = scale * <query[b,h,:], K_j>,   K_j = key_cache[block_tables[b][j / block_size],
 *                                                          j % block_size, kv_head, :]
 *   out[b,h,:] = sum_{j<L} softmax(s)_j * V_j          (V_j likewise)
 * Table entries past ceil(L / block_size) are never read.  L == 0 gives a
 * zero row.  partition_tokens as for pkv_decode_plan: a split plan computes
 * each partition's (max, normaliser, output) and merges them by log-sum-exp
 * in a second kernel.  workspace may be NULL when the plan needs none.
 */
pkv_status pkv_paged_attention_decode(const void *query, const void *key_cache,
                                      const void *value_cache,
                                      const int32_t *block_tables, int max_blocks,
                                      const int32_t *context_lens, int batch,
                                      int num_heads, int num_kv_heads, int head_dim,
                                      int block_size, int64_t num_blocks, float scale,
                                      int partition_tokens, void *workspace,
                                      size_t workspace_bytes, void *out,
                                      pkv_dtype dtype, void *stream);

/*
 * paged_attention_prefill -- chunked prefill over the paged cache: each
 * sequence brings a chunk of new query tokens whose K/V were already written
 * through pkv_kv_cache_write ([MH] 2.1/3.3: the model runner's slot_mapping
 * covers every token of the step; [YK] 三 for the block walk).
 *
 *   query          [num_tokens, num_heads, head_dim]                  device, read
 *   query_start    [batch + 1] int32, ascending, <= num_tokens: sequence b's
 *                  chunk is query rows query_start[b] .. query_start[b+1]-1
 *                  (C_b tokens, C_b <= max_query_len)                 device, read
 *   block_tables, context_lens (L_b >= C_b, the chunk included), caches as for
 *                  pkv_paged_attention_decode
 *   out            [T, num_heads, head_dim]                           device, written
 *
 * Query token i of sequence b sits at position L_b - C_b + i and attends
 * causally over the sequence's tokens 0 .. L_b - C_b + i.  One CTA per tile of
 * 128 (token, query head) rows of one sequence and kv head; its blocks are
 * streamed into shared memory (TMA) 64 keys at a time and both products
 * (Q K^T and P V) run on the tcgen05 tensor cores with f32 accumulators in
 * tensor memory.  The attention weights P are rounded to the cache dtype
 * before P V; the row sums are taken over those rounded weights.  The
 * group size (num_heads / num_kv_heads) is at most 8, as for decode.  A
 * chunk longer than
 * its context or than max_query_len, or outside the query rows, sets
 * PKV_DEVFLAG_CONTEXT_RANGE (such a chunk is clamped or skipped).
 */
pkv_status pkv_paged_attention_prefill(const void *query, int num_tokens, const int32_t *query_start,
                                       int max_query_len, const void *key_cache,
                                       const void *value_cache, const int32_t *block_tables,
                                       int max_blocks, const int32_t *context_lens, int batch,
                                       int num_heads, int num_kv_heads, int head_dim,
                                       int block_size, int64_t num_blocks, float scale, void *out,
                                       pkv_dtype dtype, void *stream);

/*
 * paged_attention_decode_cascade -- decode for sequences that share a prefix
 * ([FC] 二.3: parallel samples and beams share the prompt's blocks; [YK] 三
 * for the block walk).  The result equals pkv_paged_attention_decode over the
 * concatenated tables, but each shared prefix block is read from HBM once
 * per group instead of once per sequence.
 *
 *   prefix_tables  [num_groups, max_prefix_blocks] int32   device, read
 *   prefix_lens    [num_groups] int32, multiples of block_size, device, read
 *   group_start    [num_groups + 1] int32: group g owns sequences
 *                  group_start[g] .. group_start[g+1]-1 (ascending,
 *                  at most max_group_size each)          device, read
 *   suffix_tables  [batch, max_suffix_blocks] int32: each sequence's own
 *                  blocks, the tokens after its group's prefix    device, read
 *   suffix_lens    [batch] int32 (0 allowed)              device, read
 *   workspace      pkv_decode_cascade_workspace_bytes(...) bytes, 256-byte
 *                  aligned (partial records of prefix and suffix passes)
 *
 * Sequence b attends over prefix_tables[g] (prefix_lens[g] tokens) followed by
 * suffix_tables[b] (suffix_lens[b] tokens); sequences outside every group
 * attend over their suffix only.  Two plans, both on the tcgen05 tensor
 * cores for the group's query rows (128 per CTA):
 *   one pass   one kernel: a CTA per (kv head, chunk of 32/G members) reads
 *              its group's whole prefix once for all members' rows and then
 *              each member's own blocks for that member's rows, and writes
 *              the output; further CTAs take the sequences outside every
 *              group.  The workspace is not used.
 *   split      three kernels: the prefix in partitions (partial records per
 *              row), the regular decode over the suffixes (partial records),
 *              and a log-sum-exp merge of both.
 * partition_tokens < 0 asks for the one pass; > 0 for the split plan with
 * partitions of that many tokens (rounded up to a block multiple); 0 picks
 * the one pass when num_groups > 0 and its CTAs (num_groups x chunks of 32/G
 * members x num_kv_heads) number at least the SM count, else the split plan
 * with 512-token partitions.  pkv_decode_cascade_plan tells which.  Invalid
 * group bounds, prefix or suffix lengths set PKV_DEVFLAG_CONTEXT_RANGE.
 * num_groups x member chunks above 65535 is PKV_ERR_UNSUPPORTED.
 */
size_t pkv_decode_cascade_workspace_bytes(int batch, int num_heads, int num_kv_heads, int head_dim,
                                          int max_prefix_blocks, int max_suffix_blocks,
                                          int max_group_size, int block_size,
                                          int partition_tokens);
/* The plan pkv_paged_attention_decode_cascade will use for these sizes:
 * *one_pass = 1 for the one-pass kernel, else 0 and *prefix_partitions the
 * prefix partitions of the split plan (either output may be NULL).  The
 * workspace size above covers both plans. */
pkv_status pkv_decode_cascade_plan(int batch, int num_heads, int num_kv_heads, int head_dim,
                                   int max_prefix_blocks, int max_suffix_blocks, int max_group_size,
                                   int num_groups, int block_size, int partition_tokens,
                                   int *one_pass, int *prefix_partitions);
pkv_status pkv_paged_attention_decode_cascade(
    const void *query, const void *key_cache, const void *value_cache,
    const int32_t *prefix_tables, int max_prefix_blocks, const int32_t *prefix_lens,
    const int32_t *group_start, int num_groups, int max_group_size,
    const int32_t *suffix_tables, int max_suffix_blocks, const int32_t *suffix_lens, int batch,
    int num_heads, int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
    float scale, int partition_tokens, void *workspace, size_t workspace_bytes, void *out,
    pkv_dtype dtype, void *stream);

/*
 * hbm_read_probe -- measurement only (the pages have no counterpart): reads
 * `bytes` of device memory at `buf` once, with 16-byte loads that bypass L1,
 * and folds them into *sink (device memory, 4-byte aligned; its value has no
 * meaning).  A read-only stream is the bound of a kernel that mostly reads,
 * such as decode attention; the benchmark times this call to report the
 * decode kernels' fraction of it next to the copy peak.  `grid` CTAs of 512
 * threads.  buf 16-byte aligned and bytes a multiple of 16 (else
 * PKV_ERR_MISALIGNED / PKV_ERR_INVALID_ARG).  Asynchronous on `stream`.
 */
pkv_status pkv_hbm_read_probe(const void *buf, size_t bytes, unsigned int *sink, int grid,
                              void *stream);
/* hbm_gather_probe -- measurement only: reads a buffer of n_chunks chunks of
 * chunk_bytes each (a multiple of 16), whole chunks in the order order[0 ..
 * n_chunks) lists them (int32 chunk indices, device memory; an index outside
 * the buffer is skipped), one warp per chunk.  With a random order of 4 KiB
 * chunks this is the access pattern of a paged cache whose blocks are
 * scattered over the pool.  Same alignment rules and errors as above. */
pkv_status pkv_hbm_gather_probe(const void *buf, size_t chunk_bytes, const int32_t *order,
                                int64_t n_chunks, unsigned int *sink, int grid, void *stream);

/*
 * paged_attention_decode_static_workspace -- the same decode as
 * pkv_paged_attention_decode, for callers that cannot allocate device memory
 * at call time (an allocator that owns the whole pool, a serving runtime that
 * forbids cudaMalloc on its hot path, C code without an allocator).  The
 * pages have no counterpart: this is a convenience of this library.
 *
 * Arguments are those of pkv_paged_attention_decode without the workspace.
 * A split plan's workspace is taken from an array of
 * PKV_STATIC_WORKSPACE_BYTES bytes that the library reserves in device memory
 * on every GPU that loads it, until the process exits; nothing is allocated
 * per call.  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  The address is remembered per device and
 * context: after cudaDeviceReset (a new context, the module loaded again) the
 * next call looks it up again, so make that call before any capture as well.
 * All calls share the one array, which keeps the
 * last call's contents (no part of it needs to start at zero): calls whose
 * kernels overlap on the GPU race and must be serialised by the caller.  A
 * plan needing more than PKV_STATIC_WORKSPACE_BYTES returns
 * PKV_ERR_WORKSPACE without launching anything.
 */
#define PKV_STATIC_WORKSPACE_BYTES (16u << 20)   /* 16 MiB per device */
pkv_status pkv_paged_attention_decode_static_workspace(
    const void *query, const void *key_cache, const void *value_cache,
    const int32_t *block_tables, int max_blocks, const int32_t *context_lens, int batch,
    int num_heads, int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
    float scale, int partition_tokens, void *out, pkv_dtype dtype, void *stream);

/* ---- host block allocator ([YK] 二; [FC] 二.2 steps 1, 2, 4 and 二.3) ------
 *
 * A pool of num_blocks physical block ids with a free list and per-block
 * reference counts.  It runs on the host only and builds the int32 block
 * tables the decode call reads.  The free list starts as a permutation of
 * the ids drawn from `shuffle_seed` (0 = identity order), so a sequence's
 * blocks are scattered in the pool.  Not thread-safe: one allocator per
 * thread, or external locking.
 */
typedef struct pkv_alloc pkv_alloc;

/* NULL if num_blocks <= 0, block_size <= 0 or host memory is exhausted. */
pkv_alloc *pkv_alloc_create(int64_t num_blocks, int block_size, uint64_t shuffle_seed);
void pkv_alloc_destroy(pkv_alloc *a);

int64_t pkv_alloc_num_free(const pkv_alloc *a);
int pkv_alloc_block_size(const pkv_alloc *a);
/* Reference count of `block` (0 = free), or -1 if it is outside the pool. */
int32_t pkv_alloc_refcount(const pkv_alloc *a, int32_t block);

/*
 * New sequence of num_tokens tokens: takes ceil(num_tokens / block_size)
 * blocks (refcount 1) into out_blocks[0 .. *n).  PKV_ERR_OOM (nothing taken)
 * if the pool is short; PKV_ERR_INVALID_ARG if `capacity` is too small.
 */
pkv_status pkv_alloc_new_seq(pkv_alloc *a, int64_t num_tokens, int32_t *out_blocks,
                             int capacity, int *n);

/* Share a sequence's blocks with a forked sequence: refcount + 1 each. */
pkv_status pkv_alloc_fork(pkv_alloc *a, const int32_t *blocks, int n);

/*
 * Grow a sequence from old_len to new_len tokens.  blocks[0 .. *n) is its
 * table (capacity entries).  New blocks are appended as needed.  If old_len
 * is not a block multiple and the partly filled last block is shared
 * (refcount > 1), it is first replaced by a fresh block (copy-on-write): the
 * pair is reported as cow_src[0] -> cow_dst[0] with *n_cow = 1 so the caller
 * can copy the cells, and the shared block's refcount drops by one.  On
 * PKV_ERR_OOM nothing changes.
 */
pkv_status pkv_alloc_append(pkv_alloc *a, int32_t *blocks, int capacity, int *n,
                            int64_t old_len, int64_t new_len,
                            int32_t *cow_src, int32_t *cow_dst, int *n_cow);

/* Release a sequence's blocks: refcount - 1 each; a block reaching 0 returns
 * to the free list.  PKV_ERR_OUT_OF_RANGE (nothing changed) if an id is
 * outside the pool or already free. */
pkv_status pkv_alloc_free(pkv_alloc *a, const int32_t *blocks, int n);

/* ---- automatic prefix caching ([FC] 五.4; [MH] 2.3) --------------------
 *
 * Full blocks can be registered under a hash of their tokens chained with
 * the previous block's hash, so a new request whose prompt starts with the
 * same tokens reuses those blocks (and skips recomputing their K/V).  A
 * registered block whose reference count drops to zero stays findable: it
 * is "evictable" and is reused by a later lookup, or given out (and
 * forgotten) by new_seq / append only when the free list is empty, least
 * recently released first.  pkv_alloc_num_free counts free and evictable
 * blocks.
 */

/* Hash of a block's n tokens chained to the previous block's hash (0 for the
 * first block); never returns 0. */
uint64_t pkv_block_hash(uint64_t parent_hash, const int32_t *tokens, int n);

/* Register an in-use block (refcount > 0) under `hash`.  No-op if the block
 * is already registered or another block holds that hash. */
pkv_status pkv_alloc_cache_insert(pkv_alloc *a, uint64_t hash, int32_t block);

/* Block registered under `hash` with its refcount raised by one (a released
 * block is revived), or -1 if none. */
int32_t pkv_alloc_cache_lookup(pkv_alloc *a, uint64_t hash);

/*
 * New sequence of num_tokens tokens whose first num_hashes full blocks have
 * the given chained hashes: the longest run of leading blocks found in the
 * cache is reused (*num_hits of them, refcount + 1 each), the rest are taken
 * fresh.  PKV_ERR_OOM (nothing taken) if the pool is short.
 */
pkv_status pkv_alloc_new_seq_cached(pkv_alloc *a, const uint64_t *block_hashes, int num_hashes,
                                    int64_t num_tokens, int32_t *out_blocks, int capacity, int *n,
                                    int *num_hits);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
