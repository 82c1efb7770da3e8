// pkv_allocator.cpp -- host-side block allocator for the paged KV cache.
//
// Behaviour follows the block lifecycle the pages describe:
//   "大模型推理框架 vLLM 源码解析 一" (ai.yueke.cloud), section 二:
//     allocate() hands out a list of physical block ids;
//   "23.1 vLLM：高吞吐推理框架原理与部署" (r.flycode100.com), section 二.2:
//     the first block is taken when a request arrives and one more every
//     block_size tokens (step 2); blocks return to the shared pool when the
//     request finishes (step 4); section 二.3: prefix blocks are shared by
//     parallel samples and a shared block is copied only when one sequence
//     writes into it (copy-on-write).
// Every call either succeeds completely or leaves the allocator unchanged.

#include "pagedkv.h"

#include <cstdint>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

// Records the detail string returned by pkv_last_error() (pagedkv.cu).
void pkv_set_last_error(const char *msg);

struct pkv_alloc {
    int block_size;
    std::vector<int32_t> free_list;   // popped from the back
    std::vector<int32_t> refcount;    // 0 = free or cached-evictable
    // prefix cache: full blocks registered under the hash of their tokens
    std::unordered_map<uint64_t, int32_t> by_hash;
    std::vector<uint64_t> hash_of;     // per block; valid when cached[block]
    std::vector<uint8_t> cached;
    std::list<int32_t> evictable;      // cached blocks with refcount 0, oldest first
    std::vector<std::list<int32_t>::iterator> lru_pos;
};

namespace {

// SplitMix64 (Steele, Lea, Flood 2014): a counter-based 64-bit generator.
uint64_t splitmix64(uint64_t &state)
{
    uint64_t z = (state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

pkv_status err(pkv_status s, const char *msg)
{
    pkv_set_last_error(msg);
    return s;
}

int64_t blocks_for(int64_t tokens, int bs) { return tokens <= 0 ? 0 : (tokens + bs - 1) / bs; }

// Blocks a caller can take right now: free ones plus cached ones nobody uses.
int64_t available(const pkv_alloc *a) { return (int64_t)a->free_list.size() + (int64_t)a->evictable.size(); }

void uncache(pkv_alloc *a, int32_t id)
{
    if (!a->cached[(size_t)id])
        return;
    a->by_hash.erase(a->hash_of[(size_t)id]);
    a->cached[(size_t)id] = 0;
}

// Take one block with refcount 1: from the free list, else the least recently
// released cached block (its hash entry is dropped).  Caller checked available().
int32_t take_block(pkv_alloc *a)
{
    int32_t id;
    if (!a->free_list.empty()) {
        id = a->free_list.back();
        a->free_list.pop_back();
    } else {
        id = a->evictable.front();
        a->evictable.pop_front();
        uncache(a, id);
    }
    a->refcount[(size_t)id] = 1;
    return id;
}

// Reference drops to zero: cached blocks stay findable (evictable), others are free.
void release_block(pkv_alloc *a, int32_t id)
{
    if (a->cached[(size_t)id]) {
        a->evictable.push_back(id);
        a->lru_pos[(size_t)id] = std::prev(a->evictable.end());
    } else {
        a->free_list.push_back(id);
    }
}

}  // namespace

extern "C" {

pkv_alloc *pkv_alloc_create(int64_t num_blocks, int block_size, uint64_t shuffle_seed)
{
    if (num_blocks <= 0 || block_size <= 0 || num_blocks > INT32_MAX)
        return nullptr;
    pkv_alloc *a = new (std::nothrow) pkv_alloc;
    if (!a)
        return nullptr;
    try {
        a->block_size = block_size;
        a->refcount.assign((size_t)num_blocks, 0);
        a->hash_of.assign((size_t)num_blocks, 0);
        a->cached.assign((size_t)num_blocks, 0);
        a->lru_pos.resize((size_t)num_blocks);
        a->free_list.resize((size_t)num_blocks);
        for (int64_t i = 0; i < num_blocks; ++i)
            a->free_list[(size_t)i] = (int32_t)i;
        if (shuffle_seed != 0) {   // Fisher-Yates with SplitMix64 draws
            uint64_t st = shuffle_seed;
            for (int64_t i = num_blocks - 1; i > 0; --i) {
                int64_t j = (int64_t)(splitmix64(st) % (uint64_t)(i + 1));
                int32_t t = a->free_list[(size_t)i];
                a->free_list[(size_t)i] = a->free_list[(size_t)j];
                a->free_list[(size_t)j] = t;
            }
        }
        // pop from the back: reverse so the first id handed out is free_list[0]
        for (size_t i = 0, j = a->free_list.size() - 1; i < j; ++i, --j) {
            int32_t t = a->free_list[i];
            a->free_list[i] = a->free_list[j];
            a->free_list[j] = t;
        }
    } catch (...) {
        delete a;
        return nullptr;
    }
    return a;
}

void pkv_alloc_destroy(pkv_alloc *a) { delete a; }

int64_t pkv_alloc_num_free(const pkv_alloc *a) { return a ? available(a) : -1; }

int pkv_alloc_block_size(const pkv_alloc *a) { return a ? a->block_size : -1; }

int32_t pkv_alloc_refcount(const pkv_alloc *a, int32_t block)
{
    if (!a || block < 0 || (size_t)block >= a->refcount.size())
        return -1;
    return a->refcount[(size_t)block];
}

pkv_status pkv_alloc_new_seq(pkv_alloc *a, int64_t num_tokens, int32_t *out_blocks,
                             int capacity, int *n)
{
    if (!a || !n || num_tokens < 0 || capacity < 0)
        return err(PKV_ERR_INVALID_ARG, "new_seq: bad handle, count or output pointer");
    int64_t need = blocks_for(num_tokens, a->block_size);
    if (need > capacity || (need > 0 && !out_blocks))
        return err(PKV_ERR_INVALID_ARG, "new_seq: output capacity too small");
    if (need > available(a))
        return err(PKV_ERR_OOM, "new_seq: not enough free blocks");
    for (int64_t i = 0; i < need; ++i)
        out_blocks[i] = take_block(a);
    *n = (int)need;
    return PKV_OK;
}

pkv_status pkv_alloc_fork(pkv_alloc *a, const int32_t *blocks, int n)
{
    if (!a || n < 0 || (n > 0 && !blocks))
        return err(PKV_ERR_INVALID_ARG, "fork: bad handle or block list");
    for (int i = 0; i < n; ++i) {
        int32_t id = blocks[i];
        if (id < 0 || (size_t)id >= a->refcount.size() || a->refcount[(size_t)id] <= 0)
            return err(PKV_ERR_OUT_OF_RANGE, "fork: block id outside the pool or free");
    }
    for (int i = 0; i < n; ++i)
        a->refcount[(size_t)blocks[i]] += 1;
    return PKV_OK;
}

pkv_status pkv_alloc_append(pkv_alloc *a, int32_t *blocks, int capacity, int *n,
                            int64_t old_len, int64_t new_len,
                            int32_t *cow_src, int32_t *cow_dst, int *n_cow)
{
    if (!a || !blocks || !n || !n_cow || old_len < 0 || new_len < old_len || capacity < 0)
        return err(PKV_ERR_INVALID_ARG, "append: bad handle, pointer or lengths");
    const int bs = a->block_size;
    const int have = *n;
    if (have != blocks_for(old_len, bs))
        return err(PKV_ERR_INVALID_ARG, "append: block count does not match old_len");
    for (int i = 0; i < have; ++i) {
        int32_t id = blocks[i];
        if (id < 0 || (size_t)id >= a->refcount.size() || a->refcount[(size_t)id] <= 0)
            return err(PKV_ERR_OUT_OF_RANGE, "append: block id outside the pool or free");
    }
    const int64_t want = blocks_for(new_len, bs);
    if (want > capacity)
        return err(PKV_ERR_INVALID_ARG, "append: table capacity too small");
    // copy-on-write: new tokens land in the partly filled last block
    const bool partial_tail = (old_len % bs) != 0 && new_len > old_len;
    const bool cow = partial_tail && a->refcount[(size_t)blocks[have - 1]] > 1;
    if (cow && (!cow_src || !cow_dst))
        return err(PKV_ERR_INVALID_ARG, "append: copy-on-write outputs missing");
    const int64_t fresh = (want - have) + (cow ? 1 : 0);
    if (fresh > available(a))
        return err(PKV_ERR_OOM, "append: not enough free blocks");

    *n_cow = 0;
    if (cow) {
        int32_t src = blocks[have - 1];
        int32_t dst = take_block(a);
        a->refcount[(size_t)src] -= 1;
        blocks[have - 1] = dst;
        cow_src[0] = src;
        cow_dst[0] = dst;
        *n_cow = 1;
    }
    for (int64_t i = have; i < want; ++i)
        blocks[i] = take_block(a);
    *n = (int)want;
    return PKV_OK;
}

pkv_status pkv_alloc_free(pkv_alloc *a, const int32_t *blocks, int n)
{
    if (!a || n < 0 || (n > 0 && !blocks))
        return err(PKV_ERR_INVALID_ARG, "free: bad handle or block list");
    // validate first (counting repeats) so a failing call changes nothing
    std::vector<int32_t> dec;
    try {
        dec.assign(a->refcount.size(), 0);
    } catch (...) {
        return err(PKV_ERR_OOM, "free: host memory exhausted");
    }
    for (int i = 0; i < n; ++i) {
        int32_t id = blocks[i];
        if (id < 0 || (size_t)id >= a->refcount.size())
            return err(PKV_ERR_OUT_OF_RANGE, "free: block id outside the pool");
        if (++dec[(size_t)id] > a->refcount[(size_t)id])
            return err(PKV_ERR_OUT_OF_RANGE, "free: block released more often than referenced");
    }
    for (int i = 0; i < n; ++i) {
        int32_t id = blocks[i];
        if (--a->refcount[(size_t)id] == 0)
            release_block(a, id);
    }
    return PKV_OK;
}

// ---- automatic prefix caching -------------------------------------------
// A full block is named by a hash of its tokens chained with the previous
// block's hash, so equal hashes mean equal token prefixes up to the block's
// end ("23.1 vLLM：高吞吐推理框架原理与部署", section 五.4: requests with the same
// system prompt reuse its KV; "大模型推理框架VLLM-0.7.3源码", section 2.3: the
// sequence hashes token prefixes and the block manager keeps cached blocks).

uint64_t pkv_block_hash(uint64_t parent_hash, const int32_t *tokens, int n)
{
    // SplitMix64 finaliser over (state, token) pairs, seeded by the parent's
    // hash and the token count
    uint64_t st = parent_hash ^ (0xD6E8FEB86659FD93ull * (uint64_t)(n + 1));
    uint64_t h = splitmix64(st);
    for (int i = 0; i < n; ++i) {
        st ^= (uint64_t)(uint32_t)tokens[i] + 0x9E3779B97F4A7C15ull * (uint64_t)(i + 1);
        h ^= splitmix64(st);
        h *= 0xBF58476D1CE4E5B9ull;
    }
    return h == 0 ? 1 : h;   // 0 is reserved for "not cached"
}

pkv_status pkv_alloc_cache_insert(pkv_alloc *a, uint64_t hash, int32_t block)
{
    if (!a || hash == 0)
        return err(PKV_ERR_INVALID_ARG, "cache_insert: bad handle or zero hash");
    if (block < 0 || (size_t)block >= a->refcount.size() || a->refcount[(size_t)block] <= 0)
        return err(PKV_ERR_OUT_OF_RANGE, "cache_insert: block outside the pool or free");
    if (a->cached[(size_t)block] || a->by_hash.count(hash))
        return PKV_OK;   // already named, or another block holds these tokens
    try {
        a->by_hash.emplace(hash, block);
    } catch (...) {
        return err(PKV_ERR_OOM, "cache_insert: host memory exhausted");
    }
    a->hash_of[(size_t)block] = hash;
    a->cached[(size_t)block] = 1;
    return PKV_OK;
}

int32_t pkv_alloc_cache_lookup(pkv_alloc *a, uint64_t hash)
{
    if (!a || hash == 0)
        return -1;
    auto it = a->by_hash.find(hash);
    if (it == a->by_hash.end())
        return -1;
    const int32_t id = it->second;
    if (a->refcount[(size_t)id] == 0)
        a->evictable.erase(a->lru_pos[(size_t)id]);   // revive a released block
    a->refcount[(size_t)id] += 1;
    return id;
}

pkv_status pkv_alloc_new_seq_cached(pkv_alloc *a, const uint64_t *block_hashes, int num_hashes,
                                    int64_t num_tokens, int32_t *out_blocks, int capacity, int *n,
                                    int *num_hits)
{
    if (!a || !n || !num_hits || num_tokens < 0 || capacity < 0 || num_hashes < 0 ||
        (num_hashes > 0 && !block_hashes))
        return err(PKV_ERR_INVALID_ARG, "new_seq_cached: bad handle, counts or pointers");
    const int64_t need = blocks_for(num_tokens, a->block_size);
    if (need > capacity || (need > 0 && !out_blocks) || num_hashes > need)
        return err(PKV_ERR_INVALID_ARG, "new_seq_cached: capacity too small or too many hashes");
    // longest run of cached leading blocks
    int hits = 0;
    while (hits < num_hashes && a->by_hash.count(block_hashes[hits]))
        ++hits;
    // blocks that would be revived from the evictable list are not available
    int64_t revive = 0;
    for (int i = 0; i < hits; ++i)
        if (a->refcount[(size_t)a->by_hash[block_hashes[i]]] == 0)
            ++revive;
    if (need - hits > available(a) - revive)
        return err(PKV_ERR_OOM, "new_seq_cached: not enough free blocks");
    for (int i = 0; i < hits; ++i)
        out_blocks[i] = pkv_alloc_cache_lookup(a, block_hashes[i]);
    for (int64_t i = hits; i < need; ++i)
        out_blocks[i] = take_block(a);
    *n = (int)need;
    *num_hits = hits;
    return PKV_OK;
}

}  // extern "C"
