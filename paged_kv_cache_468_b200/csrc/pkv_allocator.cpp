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
#include <new>
#include <vector>

// Records the detail string returned by pkv_last_error() (pagedkv.cu).
void pkv_set_last_error(const char *msg);

struct pkv_alloc {
    int block_size;
    std::vector<int32_t> free_list;   // popped from the back
    std::vector<int32_t> refcount;    // 0 = free
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

int64_t pkv_alloc_num_free(const pkv_alloc *a) { return a ? (int64_t)a->free_list.size() : -1; }

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
    if (need > (int64_t)a->free_list.size())
        return err(PKV_ERR_OOM, "new_seq: not enough free blocks");
    for (int64_t i = 0; i < need; ++i) {
        int32_t id = a->free_list.back();
        a->free_list.pop_back();
        a->refcount[(size_t)id] = 1;
        out_blocks[i] = id;
    }
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
    if (fresh > (int64_t)a->free_list.size())
        return err(PKV_ERR_OOM, "append: not enough free blocks");

    *n_cow = 0;
    if (cow) {
        int32_t src = blocks[have - 1];
        int32_t dst = a->free_list.back();
        a->free_list.pop_back();
        a->refcount[(size_t)dst] = 1;
        a->refcount[(size_t)src] -= 1;
        blocks[have - 1] = dst;
        cow_src[0] = src;
        cow_dst[0] = dst;
        *n_cow = 1;
    }
    for (int64_t i = have; i < want; ++i) {
        int32_t id = a->free_list.back();
        a->free_list.pop_back();
        a->refcount[(size_t)id] = 1;
        blocks[i] = id;
    }
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
            a->free_list.push_back(id);
    }
    return PKV_OK;
}

}  // extern "C"
