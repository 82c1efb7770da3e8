"""paged_attention_decode on the GPU vs the fp64 oracle.

Bar: max-abs error <= 2e-3 (fp16) / 1e-2 (bf16) against the unrounded oracle,
fp32 accumulation, on every workload at full size (the configuration the
benchmark times), on edge cases (context lengths around block and partition
boundaries, group sizes 1..8, both head dims and block sizes), and on the
invariants the pages state (physical placement does not matter; split and
single-pass plans agree)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import pagedkv, workloads
from tests.parity_util import TOL, custom, gpu_step, max_abs_err, oracle_step, to_device, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield


def _parity(step, write=True, partition_tokens=None, flags_ok=0):
    ref, _, _ = oracle_step(step, write=write)
    d = to_device(step)
    out = gpu_step(d, write=write, partition_tokens=partition_tokens)
    err, idx, finite = max_abs_err(out, ref)
    assert finite
    assert err <= TOL[step["dtype"]], f"max-abs error {err:.3e} at {idx}"
    assert pkv.device_flags() == flags_ok
    return out, err


@pytest.mark.parametrize("name", sorted(workloads.CONFIGS))
def test_full_config_write_then_decode(name):
    step = workloads.make_decode_step(workloads.CONFIGS[name])
    _parity(step)


@pytest.mark.parametrize("name", sorted(workloads.CONFIGS))
def test_small_config_single_pass_and_split(name):
    cfg = workloads.CONFIGS[name]
    B = 8 if cfg.shared_prefix else min(cfg.batch, 6)
    step = workloads.make_decode_step(cfg, batch=B)
    for pt in (-1, 64, 256):
        _parity(step, partition_tokens=pt)


EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 511, 512, 513, 1000]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_edge_lengths(D, bs, dtype):
    step = custom("edge", len(EDGE_LENS), 8, 2, D, bs, dtype, EDGE_LENS, seed=D + bs)
    for pt in (-1, 0, 128):
        _parity(step, partition_tokens=pt)


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 6, 7, 8])
def test_group_sizes(G):
    Hkv = 3
    step = custom("grp", 5, G * Hkv, Hkv, 128, 16, "bf16", [7, 100, 257, 16, 600], seed=G)
    _parity(step, partition_tokens=-1)
    _parity(step, partition_tokens=96)


def test_split_matches_single_pass():
    step = workloads.make_decode_step(workloads.CONFIGS["long_split"], batch=3)
    ref, _, _ = oracle_step(step)
    outs = []
    for pt in (-1, 512, 2048):
        d = to_device(step)
        o = gpu_step(d, partition_tokens=pt)
        err, idx, _ = max_abs_err(o, ref)
        assert err <= TOL["bf16"], (pt, err, idx)
        outs.append(o.float())
    assert (outs[0] - outs[1]).abs().max().item() <= TOL["bf16"]
    assert (outs[0] - outs[2]).abs().max().item() <= TOL["bf16"]


def test_physical_permutation_is_bitwise_invariant():
    step = workloads.make_decode_step(workloads.CONFIGS["llama3_8b_gqa"], batch=16)
    d = to_device(step)
    a = gpu_step(d, write=False)
    NB = d["key_cache"].shape[0]
    perm = torch.randperm(NB, generator=torch.Generator().manual_seed(3)).cuda()
    kc2 = torch.empty_like(d["key_cache"])
    vc2 = torch.empty_like(d["value_cache"])
    kc2[perm] = d["key_cache"]
    vc2[perm] = d["value_cache"]
    t2 = d["block_tables"].clone()
    used = t2 >= 0
    t2[used] = perm[t2[used].long()].int()
    d2 = dict(d, key_cache=kc2, value_cache=vc2, block_tables=t2)
    for pt in (-1, 128):
        x = gpu_step(d, write=False, partition_tokens=pt)
        y = gpu_step(d2, write=False, partition_tokens=pt)
        assert torch.equal(x, y)
    assert torch.equal(a, gpu_step(d2, write=False))


def test_garbage_past_context_end_is_ignored():
    """Cells past context_len in the last block hold NaN / inf: output unaffected."""
    lens = [1, 17, 30, 45]
    step = custom("nan", 4, 8, 2, 128, 16, "f16", lens, seed=11)
    ref, _, _ = oracle_step(step, write=False)
    d = to_device(step)
    bs = 16
    for b, L in enumerate(lens):
        last = int(step["block_tables"][b, (L - 1) // bs])
        off = L % bs
        if off:
            d["key_cache"][last, off:] = float("nan")
            d["value_cache"][last, off:] = float("inf")
    for pt in (-1, 16):
        out = gpu_step(d, write=False, partition_tokens=pt)
        err, idx, finite = max_abs_err(out, ref)
        assert finite and err <= TOL["f16"], (pt, err, idx)


def test_empty_context_gives_zeros():
    step = custom("empty", 3, 8, 8, 64, 16, "f16", [0, 5, 0], seed=12)
    step["slot_mapping"][:] = -1
    out, _ = _parity(step, write=False, partition_tokens=-1)
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    out, _ = _parity(step, write=False, partition_tokens=16)
    assert torch.count_nonzero(out[0]) == 0


@pytest.mark.parametrize("D", [64, 128])
def test_empty_context_many_partitions(D):
    """13 partitions per row (the merge that gives each row a CTA): rows
    without tokens still come out as zeros, next to a row that has them."""
    step = custom("empty_wide", 3, 8, 8, D, 16, "bf16", [0, 200, 0], seed=13)
    step["slot_mapping"][:] = -1
    out, _ = _parity(step, write=False, partition_tokens=16)
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0


def test_shared_prefix_tables_from_allocator():
    """Forked samples share the prefix blocks (refcounted, read-only); the
    decode equals the oracle on the allocator's tables."""
    B, samples, prefix, bs = 8, 4, 2001, 16
    alloc = pkv.BlockAllocator(2 * (prefix // bs + 1) + 64, bs, shuffle_seed=21)
    tables, lens, cows = [], [], []
    for p in range(B // samples):
        base = alloc.new_seq(prefix)
        for s in range(samples):
            t = alloc.fork(list(base)) if s else base
            n = prefix + 1 + 3 * s
            cow = alloc.append(t, prefix, n)
            if cow:
                cows.append(cow)
            tables.append(t)
            lens.append(n)
    assert cows, "a 2001-token prefix leaves a shared partial block: copy-on-write expected"
    step = custom("fork", B, 8, 2, 128, bs, "bf16", lens, seed=13)
    NB = alloc.num_blocks
    g = torch.Generator().manual_seed(14)
    step["key_cache"] = torch.randn(NB, bs, 2, 128, generator=g).bfloat16()
    step["value_cache"] = torch.randn(NB, bs, 2, 128, generator=g).bfloat16()
    for src, dst in cows:                               # materialise the copies
        step["key_cache"][dst] = step["key_cache"][src]
        step["value_cache"][dst] = step["value_cache"][src]
    MB = max(len(t) for t in tables)
    bt = torch.full((B, MB), -1, dtype=torch.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
    step["block_tables"] = bt
    step["slot_mapping"][:] = -1
    for pt in (-1, 0, 512):
        _parity(step, write=False, partition_tokens=pt)


def test_bad_block_id_sets_flag_without_fault():
    step = custom("bad", 2, 8, 8, 64, 16, "f16", [20, 20], seed=15)
    step["block_tables"][0, 1] = 10 ** 6
    d = to_device(step)
    gpu_step(d, write=False, partition_tokens=-1)
    assert pkv.device_flags() & pagedkv.DEVFLAG_BLOCK_RANGE


def test_context_beyond_table_sets_flag():
    step = custom("ctx", 2, 8, 8, 64, 16, "f16", [20, 20], seed=16)
    d = to_device(step)
    d["context_lens"][1] = 10 ** 6
    gpu_step(d, write=False, partition_tokens=-1)
    assert pkv.device_flags() & pagedkv.DEVFLAG_CONTEXT_RANGE


def test_caller_workspace_and_out_are_used():
    step = workloads.make_decode_step(workloads.CONFIGS["long_split"], batch=2)
    ref, _, _ = oracle_step(step)
    d = to_device(step)
    pkv.kv_cache_write(d["new_key"], d["new_value"], d["slot_mapping"], d["key_cache"],
                       d["value_cache"])
    B, Hq, D = d["query"].shape
    NB, bs, Hkv, _ = d["key_cache"].shape
    nbytes = pkv.decode_workspace_bytes(B, Hq, Hkv, D, d["block_tables"].shape[1], bs, 512)
    ws = torch.empty(nbytes // 4, dtype=torch.float32, device="cuda")
    out = torch.empty_like(d["query"])
    r = pkv.paged_attention_decode(d["query"], d["key_cache"], d["value_cache"], d["block_tables"],
                                   d["context_lens"], d["scale"], partition_tokens=512, out=out,
                                   workspace=ws)
    assert r.data_ptr() == out.data_ptr()
    err, idx, _ = max_abs_err(out, ref)
    assert err <= TOL["bf16"]
    with pytest.raises(pagedkv.PagedKVError) as e:
        pkv.paged_attention_decode(d["query"], d["key_cache"], d["value_cache"], d["block_tables"],
                                   d["context_lens"], d["scale"], partition_tokens=512,
                                   workspace=ws[: nbytes // 8])
    assert e.value.status == pagedkv.ERR_WORKSPACE


def test_nonblocking_stream():
    step = workloads.make_decode_step(workloads.CONFIGS["tiny_mha"])
    ref, _, _ = oracle_step(step)
    d = to_device(step)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = gpu_step(d)
    s.synchronize()
    err, _, _ = max_abs_err(out, ref)
    assert err <= TOL["f16"]
