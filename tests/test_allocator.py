"""Host block allocator: free list, refcounts, fork, copy-on-write (CPU only).

Invariants follow the block lifecycle on the pages: blocks are taken on
demand, one per block_size tokens, need not be contiguous, return to the
shared pool at the end ("23.1 vLLM：高吞吐推理框架原理与部署", section 二.2),
prefix blocks are shared by forked samples and copied only on a write into a
shared block (section 二.3), and only the last block of a sequence is partly
empty (section 二.1 table)."""
import random

import pytest

from paged_kv_cache_468_b200 import BlockAllocator, PagedKVError, pagedkv


def conservation(a, tables):
    live = set()
    refs = {}
    for t in tables:
        for b in t:
            live.add(b)
            refs[b] = refs.get(b, 0) + 1
    assert a.num_free + len(live) == a.num_blocks
    for b, r in refs.items():
        assert a.refcount(b) == r


def test_new_seq_takes_ceil_blocks_and_scatters():
    a = BlockAllocator(100, 16, shuffle_seed=5)
    s = a.new_seq(33)
    assert len(s) == 3 and len(set(s)) == 3
    assert a.new_seq(0) == []
    t = a.new_seq(16)
    assert len(t) == 1
    conservation(a, [s, t])
    # a seeded shuffle scatters ids; seed 0 hands them out in order
    b = BlockAllocator(100, 16, shuffle_seed=0)
    assert b.new_seq(64) == [0, 1, 2, 3]
    assert sorted(a.new_seq(16 * 90)) != list(range(90))


def test_internal_fragmentation_only_in_last_block():
    a = BlockAllocator(1000, 16, shuffle_seed=1)
    rng = random.Random(0)
    for _ in range(200):
        n = rng.randint(1, 500)
        s = a.new_seq(n)
        assert len(s) * 16 - n < 16          # at most block_size-1 empty slots
        a.free(s)
    assert a.num_free == 1000


def test_oom_takes_nothing():
    a = BlockAllocator(5, 16, shuffle_seed=2)
    s = a.new_seq(48)
    with pytest.raises(PagedKVError) as e:
        a.new_seq(48)
    assert e.value.status == pagedkv.ERR_OOM
    assert a.num_free == 2
    with pytest.raises(PagedKVError):
        a.append(s, 48, 48 + 16 * 3)
    assert a.num_free == 2 and len(s) == 3
    conservation(a, [s])


def test_fork_shares_and_free_returns_on_zero():
    a = BlockAllocator(50, 16, shuffle_seed=3)
    p = a.new_seq(64)
    kids = [a.fork(list(p)) for _ in range(7)]
    for b in p:
        assert a.refcount(b) == 8
    conservation(a, [p] + kids)
    a.free(p)
    for k in kids[:-1]:
        a.free(k)
    for b in p:
        assert a.refcount(b) == 1
    a.free(kids[-1])
    assert a.num_free == 50
    for b in p:
        assert a.refcount(b) == 0


def test_copy_on_write_on_shared_partial_block():
    a = BlockAllocator(300, 16, shuffle_seed=4)
    p = a.new_seq(2001)                       # 126 blocks, last one holds 1 token
    assert len(p) == 126
    q = a.fork(list(p))
    cow = a.append(q, 2001, 2002)             # writes into the shared partial block
    assert cow is not None
    src, dst = cow
    assert src == p[-1] and dst == q[-1] and dst != src
    assert a.refcount(src) == 1 and a.refcount(dst) == 1
    assert q[:-1] == p[:-1]
    for b in p[:-1]:
        assert a.refcount(b) == 2
    conservation(a, [p, q])
    # the owner of the now-private block appends without a copy
    assert a.append(p, 2001, 2003) is None
    # full prefix blocks: appending starts a new block, no copy
    r = a.new_seq(32)
    r2 = a.fork(list(r))
    assert a.append(r2, 32, 33) is None and len(r2) == 3 and r2[:2] == r


def test_free_validates_before_changing_anything():
    a = BlockAllocator(10, 16, shuffle_seed=6)
    s = a.new_seq(32)
    with pytest.raises(PagedKVError):
        a.free([s[0], s[0]])                  # second release of a refcount-1 block
    assert a.refcount(s[0]) == 1
    with pytest.raises(PagedKVError):
        a.free([99])
    with pytest.raises(PagedKVError):
        a.fork([s[0], 99])
    assert a.refcount(s[0]) == 1
    a.free(s)
    with pytest.raises(PagedKVError):
        a.free(s)                             # already free


def test_random_lifecycle_conserves_blocks():
    rng = random.Random(7)
    a = BlockAllocator(400, 16, shuffle_seed=7)
    seqs = {}                                 # id -> (blocks, length)
    nxt = 0
    for step in range(2000):
        op = rng.random()
        try:
            if op < 0.3 or not seqs:
                n = rng.randint(1, 200)
                seqs[nxt] = (a.new_seq(n), n)
                nxt += 1
            elif op < 0.45:
                k = rng.choice(list(seqs))
                blocks, n = seqs[k]
                seqs[nxt] = (a.fork(list(blocks)), n)
                nxt += 1
            elif op < 0.8:
                k = rng.choice(list(seqs))
                blocks, n = seqs[k]
                m = n + rng.randint(1, 40)
                a.append(blocks, n, m)
                seqs[k] = (blocks, m)
            else:
                k = rng.choice(list(seqs))
                a.free(seqs.pop(k)[0])
        except PagedKVError as e:
            assert e.status == pagedkv.ERR_OOM
        for blocks, n in seqs.values():
            assert len(blocks) == -(-n // 16)
        if step % 100 == 0:
            conservation(a, [b for b, _ in seqs.values()])
    conservation(a, [b for b, _ in seqs.values()])


# ---- automatic prefix caching ------------------------------------------------

def _register(a, blocks, tokens):
    for h, b in zip(a.block_hashes(tokens), blocks):
        a.cache_insert(h, b)


def test_block_hash_chains_the_prefix():
    a = BlockAllocator(8, 4)
    h1 = a.block_hashes([1, 2, 3, 4, 5, 6, 7, 8])
    h2 = a.block_hashes([9, 9, 9, 9, 5, 6, 7, 8])     # same 2nd block, different prefix
    h3 = a.block_hashes([1, 2, 3, 4, 5, 6, 7, 8, 0])  # trailing partial block not hashed
    assert len(h1) == 2 and h1 == h3
    assert h1[1] != h2[1] and h1[0] != h2[0]
    assert all(h != 0 for h in h1 + h2)


def test_same_prompt_reuses_cached_blocks():
    a = BlockAllocator(64, 16, shuffle_seed=3)
    prompt = list(range(1000, 1000 + 50))             # 3 full blocks + 2 tokens
    s1, hits1 = a.new_seq_cached(prompt)
    assert hits1 == 0 and len(s1) == 4
    _register(a, s1, prompt)                          # after its K/V are written
    s2, hits2 = a.new_seq_cached(prompt)
    assert hits2 == 3 and s2[:3] == s1[:3] and s2[3] != s1[3]
    for b in s1[:3]:
        assert a.refcount(b) == 2
    other = prompt[:20] + [7] * 30                    # shares only the first block
    s3, hits3 = a.new_seq_cached(other)
    assert hits3 == 1 and s3[0] == s1[0] and s3[1] not in s1
    conservation(a, [s1, s2, s3])


def test_released_cached_blocks_are_revived_or_evicted_lru():
    a = BlockAllocator(6, 4, shuffle_seed=5)
    p = [1] * 8                                       # 2 full blocks
    q = [2] * 8
    sp, _ = a.new_seq_cached(p)
    _register(a, sp, p)
    sq, _ = a.new_seq_cached(q)
    _register(a, sq, q)
    a.free(sp)                                        # released first
    a.free(sq)
    assert a.num_free == 6                            # free + evictable
    for b in sp + sq:
        assert a.refcount(b) == 0
    again, hits = a.new_seq_cached(q)                 # revived, not recomputed
    assert hits == 2 and again == sq
    fresh = a.new_seq(16)                             # needs 4: 2 free + 2 evicted (p's)
    assert sorted(set(fresh) & set(sp)) == sorted(sp)
    assert a.cache_lookup(a.block_hashes(p)[0]) == -1  # p's entries were dropped
    with pytest.raises(PagedKVError) as e:
        a.new_seq(4)
    assert e.value.status == pagedkv.ERR_OOM
    conservation(a, [again, fresh])


def test_cache_random_workload_conserves_blocks():
    rng = random.Random(11)
    a = BlockAllocator(200, 8, shuffle_seed=11)
    prompts = [[rng.randrange(50) for _ in range(rng.randrange(8, 80))] for _ in range(12)]
    live = []
    for step in range(600):
        if live and rng.random() < 0.45:
            a.free(live.pop(rng.randrange(len(live))))
        else:
            base = rng.choice(prompts)
            toks = base[:rng.randrange(1, len(base) + 1)] + [rng.randrange(50) for _ in range(rng.randrange(0, 9))]
            try:
                blocks, hits = a.new_seq_cached(toks)
            except PagedKVError as e:
                assert e.status == pagedkv.ERR_OOM
                continue
            _register(a, blocks, toks)
            assert len(blocks) == -(-len(toks) // 8)
            live.append(blocks)
        refs = {}
        for t in live:
            for b in t:
                refs[b] = refs.get(b, 0) + 1
        for b, r in refs.items():
            assert a.refcount(b) == r
        assert a.num_free + len(refs) == 200
