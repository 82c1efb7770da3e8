"""Automatic prefix caching end to end on the GPU.

Prompts that begin with the same tokens reuse the cached KV blocks of that
prefix instead of computing and storing them again ("大模型推理框架VLLM-0.7.3源码",
section 2.3; "23.1 vLLM：高吞吐推理框架原理与部署", section 五.4).  Here the
host allocator builds every block table through new_seq_cached (full blocks
named by chained token hashes), only the positions it did not find cached are
written through kv_cache_write, and the decode over those tables -- whose
leading blocks are physically shared -- is compared with the fp64 oracle run
on a private, unshared layout of the same sequences.

A token's K/V depends on every token up to it (as in a transformer): the test
draws the rows of position p from a generator seeded by a hash of the tokens
0..p, so equal prefixes have equal K/V and any divergence changes every later
row.
"""
import hashlib

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import BlockAllocator
from tests.parity_util import NTHREADS, TOL, max_abs_err, u16

pytestmark = pytest.mark.gpu

BS, HQ, HKV, D = 16, 8, 2, 128
DT = torch.bfloat16


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield
    assert pkv.device_flags() == 0


def _kv_rows(tokens):
    """K and V rows [len(tokens), HKV, D] of a token sequence (row p from tokens 0..p)."""
    ks, vs = [], []
    h = hashlib.sha256()
    for t in tokens:
        h.update(int(t).to_bytes(4, "little", signed=True))
        g = torch.Generator().manual_seed(int.from_bytes(h.digest()[:8], "little") >> 1)
        kv = torch.randn(2, HKV, D, generator=g).to(DT)
        ks.append(kv[0])
        vs.append(kv[1])
    return torch.stack(ks), torch.stack(vs)


def _write(kc, vc, k, v, blocks, positions, host_k, host_v):
    """kv_cache_write of the given positions on the GPU, and the oracle's write
    of the same rows into the host mirror of the pool."""
    pos = torch.tensor(positions, dtype=torch.int64)
    slots = torch.tensor([blocks[p // BS] * BS + p % BS for p in positions], dtype=torch.int64)
    kk, vv = k[pos].contiguous(), v[pos].contiguous()
    pkv.kv_cache_write(kk.cuda(), vv.cuda(), slots.cuda(), kc, vc)
    oracle.kv_cache_write(u16(kk), u16(vv), slots.numpy(), host_k, host_v, BS)


def test_prefix_cache_hits_decode_like_private_blocks():
    rng = np.random.default_rng(468)
    NB = 64
    alloc = BlockAllocator(NB, BS, shuffle_seed=17)
    g = torch.Generator().manual_seed(3)
    kc = torch.randn(NB, BS, HKV, D, generator=g).to(DT)     # garbage in unused cells
    vc = torch.randn(NB, BS, HKV, D, generator=g).to(DT)
    host_k, host_v = u16(kc).copy(), u16(vc).copy()
    kc, vc = kc.cuda(), vc.cuda()

    def tokens(n):
        return [int(x) for x in rng.integers(0, 32000, size=n)]

    A = tokens(100)                                        # 6 full blocks + 4 tokens
    B = A[:64] + tokens(26)                                # shares 4 full blocks with A
    C = A[:16] + tokens(47)                                # shares 1 block
    D_ = A + tokens(5)                                     # A again, after A is released

    def admit(toks, expect_hits):
        blocks, hits = alloc.new_seq_cached(toks)
        assert hits == expect_hits, (hits, expect_hits)
        k, v = _kv_rows(toks)
        _write(kc, vc, k, v, blocks, list(range(hits * BS, len(toks))), host_k, host_v)
        for h, b in zip(alloc.block_hashes(toks), blocks):   # full blocks, once written
            alloc.cache_insert(h, b)
        return blocks

    bA = admit(A, 0)
    bB = admit(B, 4)
    assert bB[:4] == bA[:4] and bB[4] not in bA
    for blk in bA[:4]:
        assert alloc.refcount(blk) == 2                   # A and B
    bC = admit(C, 1)
    assert bC[0] == bA[0] and alloc.refcount(bA[0]) == 3
    alloc.free(bA)                                         # A leaves; its full blocks stay cached
    bD = admit(D_, 6)                                      # revived: nothing recomputed but the tail
    assert bD[:6] == bA[:6]

    # the GPU pool holds exactly what the oracle's writes put in its mirror
    assert np.array_equal(u16(kc), host_k) and np.array_equal(u16(vc), host_v)

    # decode B, C and D over the allocator's (shared) tables
    seqs = [(B, bB), (C, bC), (D_, bD)]
    mb = max(len(b) for _, b in seqs)
    tables = torch.full((len(seqs), mb), -1, dtype=torch.int32)
    for i, (_, b) in enumerate(seqs):
        tables[i, :len(b)] = torch.tensor(b, dtype=torch.int32)
    lens = torch.tensor([len(t) for t, _ in seqs], dtype=torch.int32)
    q = torch.randn(len(seqs), HQ, D, generator=g).to(DT)
    scale = 1.0 / np.sqrt(D)
    out = pkv.paged_attention_decode(q.cuda(), kc, vc, tables.cuda(), lens.cuda(), scale)

    # expected: the same sequences with private blocks, nothing shared
    pk = np.zeros((sum(-(-len(t) // BS) for t, _ in seqs), BS, HKV, D), dtype=np.uint16)
    pv = np.zeros_like(pk)
    ptab = np.full((len(seqs), mb), -1, dtype=np.int32)
    nxt = 0
    for i, (toks, _) in enumerate(seqs):
        nblk = -(-len(toks) // BS)
        ptab[i, :nblk] = np.arange(nxt, nxt + nblk)
        k, v = _kv_rows(toks)
        slots = np.array([ptab[i, p // BS] * BS + p % BS for p in range(len(toks))], dtype=np.int64)
        oracle.kv_cache_write(u16(k), u16(v), slots, pk, pv, BS)
        nxt += nblk
    ref = oracle.paged_attention_decode(u16(q), pk, pv, ptab, lens.numpy(), scale, "bf16",
                                        nthreads=NTHREADS)
    err, idx, finite = max_abs_err(out, ref)
    assert finite and err <= TOL["bf16"], (err, idx)
