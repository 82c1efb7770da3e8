"""Whole-block copies on the GPU vs the oracle (bit-exact): copy-on-write in one
pool, swap-out to pinned host memory and swap-in, and the allocator's
copy-on-write pair materialised before a decode reads the new block."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import pagedkv
from tests.parity_util import TOL, max_abs_err, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield


def _pool(NB, seed, shape=(16, 8, 128), dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(NB, *shape, generator=g).to(dtype)


def test_copy_on_write_in_device_pool_bit_exact():
    k, v = _pool(300, 1), _pool(300, 2)
    mapping = torch.tensor([[5, 17], [250, 3], [5, 299], [0, 1]], dtype=torch.int32)
    kd, vd = k.cuda(), v.cuda()
    pkv.copy_blocks(kd, vd, kd, vd, mapping.cuda())
    ek, ev = u16(k).copy(), u16(v).copy()
    oracle.copy_blocks(ek.copy(), ek, mapping.numpy())
    oracle.copy_blocks(ev.copy(), ev, mapping.numpy())
    assert np.array_equal(u16(kd), ek) and np.array_equal(u16(vd), ev)
    assert pkv.device_flags() == 0


def test_swap_out_to_pinned_host_and_back():
    k, v = _pool(64, 3, (32, 4, 64), torch.float16), _pool(64, 4, (32, 4, 64), torch.float16)
    kd, vd = k.cuda(), v.cuda()
    hk = torch.zeros(10, 32, 4, 64, dtype=torch.float16).pin_memory()
    hv = torch.zeros(10, 32, 4, 64, dtype=torch.float16).pin_memory()
    out_map = torch.tensor([[7, 0], [63, 9], [12, 4]], dtype=torch.int32).cuda()
    pkv.copy_blocks(kd, vd, hk, hv, out_map)                 # swap out
    torch.cuda.synchronize()
    assert torch.equal(hk[0], k[7]) and torch.equal(hv[9], v[63]) and torch.equal(hk[4], k[12])
    assert torch.count_nonzero(hk[1]) == 0
    back = torch.zeros_like(kd), torch.zeros_like(vd)
    in_map = torch.tensor([[0, 40], [9, 41], [4, 42]], dtype=torch.int32).cuda()
    pkv.copy_blocks(hk, hv, back[0], back[1], in_map)         # swap in elsewhere
    assert torch.equal(back[0][40], kd[7]) and torch.equal(back[1][41], vd[63])
    assert torch.equal(back[1][42], vd[12])
    assert pkv.device_flags() == 0


def test_out_of_range_pair_is_skipped_and_flagged():
    k, v = _pool(8, 5).cuda(), _pool(8, 6).cuda()
    before = k.clone()
    pkv.copy_blocks(k, v, k, v, torch.tensor([[1, 8], [2, 3]], dtype=torch.int32).cuda())
    assert pkv.device_flags() & pagedkv.DEVFLAG_BLOCK_RANGE
    assert torch.equal(k[3], before[2]) and torch.equal(k[:3], before[:3])


def test_allocator_copy_on_write_then_decode():
    bs, Hkv, Hq, D = 16, 2, 8, 128
    alloc = pkv.BlockAllocator(64, bs, shuffle_seed=9)
    parent = alloc.new_seq(37)                                # last block holds 5 tokens
    child = alloc.fork(list(parent))
    src_dst = alloc.append(child, 37, 38)                     # write into the shared block
    assert src_dst is not None
    k, v = _pool(64, 7, (bs, Hkv, D)), _pool(64, 8, (bs, Hkv, D))
    kd, vd = k.cuda(), v.cuda()
    pkv.copy_blocks(kd, vd, kd, vd, torch.tensor([src_dst], dtype=torch.int32).cuda())
    # the child's new token: written into the copied block at offset 37 % 16
    g = torch.Generator().manual_seed(10)
    nk = torch.randn(1, Hkv, D, generator=g).bfloat16().cuda()
    nv = torch.randn(1, Hkv, D, generator=g).bfloat16().cuda()
    slot = torch.tensor([child[37 // bs] * bs + 37 % bs], dtype=torch.int64).cuda()
    pkv.kv_cache_write(nk, nv, slot, kd, vd)
    q = torch.randn(2, Hq, D, generator=g).bfloat16().cuda()
    tables = torch.full((2, 3), -1, dtype=torch.int32)
    tables[0, :3] = torch.tensor(parent, dtype=torch.int32)
    tables[1, :3] = torch.tensor(child, dtype=torch.int32)
    lens = torch.tensor([37, 38], dtype=torch.int32)
    out = pkv.paged_attention_decode(q, kd, vd, tables.cuda(), lens.cuda(), 1 / np.sqrt(D),
                                     partition_tokens=-1)
    # oracle: copy, write and decode on the host copies
    ek, ev = u16(k).copy(), u16(v).copy()
    oracle.copy_blocks(ek.copy(), ek, np.array([src_dst], np.int32))
    oracle.copy_blocks(ev.copy(), ev, np.array([src_dst], np.int32))
    oracle.kv_cache_write(u16(nk), u16(nv), slot.cpu().numpy(), ek, ev, bs)
    ref = oracle.paged_attention_decode(u16(q), ek, ev, tables.numpy(), lens.numpy(),
                                        1 / np.sqrt(D), "bf16")
    err, idx, finite = max_abs_err(out, ref)
    assert finite and err <= TOL["bf16"], (err, idx)
    # the parent's shared block was not touched by the child's write
    assert np.array_equal(u16(kd)[parent[2]], u16(k)[parent[2]])
    assert pkv.device_flags() == 0
