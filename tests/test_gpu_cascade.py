"""Cascade (shared-prefix) decode on the GPU vs the fp64 oracle.

The cascade computes exactly the decode over each sequence's full table
(group prefix followed by its own blocks): the oracle runs the plain
definition on the concatenated tables ("23.1 vLLM：高吞吐推理框架原理与部署",
section 二.3: parallel samples share the prompt's blocks).

Both plans are covered: the split plan (prefix partitions as records, the
suffix decode, a merge; partition_tokens > 0) and the one pass (a CTA per
group chunk reads the prefix and then each member's own blocks;
partition_tokens < 0); partition_tokens = 0 picks by size."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import workloads
from tests.parity_util import NTHREADS, TOL, max_abs_err, u16

pytestmark = pytest.mark.gpu

_DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _cascade_case(groups, prefix_blocks, suffix_tokens, Hq, Hkv, D, bs, dtype, seed, before=0,
                  after=0):
    """groups: sizes of consecutive groups (0-prefix groups allowed);
    prefix_blocks[g]: shared blocks; suffix_tokens[b]: own tokens;
    `before` / `after` sequences outside every group (own tokens only)."""
    g = torch.Generator().manual_seed(seed)
    B = before + sum(groups) + after
    assert len(suffix_tokens) == B
    sfx_blocks = [-(-t // bs) for t in suffix_tokens]
    need = sum(prefix_blocks) + sum(sfx_blocks)
    NB = need + 7
    perm = torch.randperm(NB, generator=g).tolist()
    cur = 0
    prefix_tables = torch.full((len(groups), max(1, max(prefix_blocks))), -1, dtype=torch.int32)
    for i, n in enumerate(prefix_blocks):
        prefix_tables[i, :n] = torch.tensor(perm[cur:cur + n], dtype=torch.int32)
        cur += n
    msb = max(1, max(sfx_blocks))
    suffix_tables = torch.full((B, msb), -1, dtype=torch.int32)
    for b, n in enumerate(sfx_blocks):
        suffix_tables[b, :n] = torch.tensor(perm[cur:cur + n], dtype=torch.int32)
        cur += n
    group_start = torch.tensor(before + np.concatenate([[0], np.cumsum(groups)]), dtype=torch.int32)
    prefix_lens = torch.tensor([n * bs for n in prefix_blocks], dtype=torch.int32)
    suffix_lens = torch.tensor(suffix_tokens, dtype=torch.int32)
    # full tables for the oracle: prefix blocks, then own blocks
    full_lens, rows = [], []
    owner = [None] * B
    for gi, size in enumerate(groups):
        for m in range(size):
            owner[int(group_start[gi]) + m] = gi
    for b in range(B):
        gi = owner[b]
        pre = prefix_tables[gi, :prefix_blocks[gi]].tolist() if gi is not None else []
        rows.append(pre + suffix_tables[b, :sfx_blocks[b]].tolist())
        full_lens.append((prefix_blocks[gi] * bs if gi is not None else 0) + suffix_tokens[b])
    mb = max(1, max(len(r) for r in rows))
    full = torch.full((B, mb), -1, dtype=torch.int32)
    for b, r in enumerate(rows):
        if r:
            full[b, :len(r)] = torch.tensor(r, dtype=torch.int32)
    kc = torch.randn(NB, bs, Hkv, D, generator=g).to(_DT[dtype])
    vc = torch.randn(NB, bs, Hkv, D, generator=g).to(_DT[dtype])
    q = torch.randn(B, Hq, D, generator=g).to(_DT[dtype])
    return dict(query=q, key_cache=kc, value_cache=vc, prefix_tables=prefix_tables,
                prefix_lens=prefix_lens, group_start=group_start, suffix_tables=suffix_tables,
                suffix_lens=suffix_lens, full_tables=full,
                full_lens=torch.tensor(full_lens, dtype=torch.int32),
                max_group_size=max(groups), scale=1.0 / np.sqrt(D), dtype=dtype)


def _run(case, pt=0):
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    return pkv.paged_attention_decode_cascade(
        d["query"], d["key_cache"], d["value_cache"], d["prefix_tables"], d["prefix_lens"],
        d["group_start"], d["suffix_tables"], d["suffix_lens"], d["scale"],
        max_group_size=d["max_group_size"], partition_tokens=pt)


def _oracle(case):
    return oracle.paged_attention_decode(u16(case["query"]), u16(case["key_cache"]),
                                         u16(case["value_cache"]), case["full_tables"].numpy(),
                                         case["full_lens"].numpy(), case["scale"], case["dtype"],
                                         nthreads=NTHREADS)


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield
    assert pkv.device_flags() == 0


def test_cascade_full_shared_prefix_workload():
    cfg = workloads.CONFIGS["shared_prefix"]
    step = workloads.make_decode_step(cfg)
    cas = workloads.cascade_inputs(step, cfg.shared_prefix, cfg.samples)
    case = dict(query=step["query"], key_cache=step["key_cache"], value_cache=step["value_cache"],
                full_tables=step["block_tables"], full_lens=step["context_lens"], scale=cfg.scale,
                dtype=cfg.dtype, **cas)
    ref = _oracle(case)
    out = _run(case)
    err, idx, finite = max_abs_err(out, ref)
    assert finite and err <= TOL[cfg.dtype], (err, idx)
    # and it agrees with the plain decode over the full tables
    d = {k: v.cuda() for k, v in step.items() if isinstance(v, torch.Tensor)}
    plain = pkv.paged_attention_decode(d["query"], d["key_cache"], d["value_cache"],
                                       d["block_tables"], d["context_lens"], cfg.scale)
    assert (plain.float() - out.float()).abs().max().item() <= TOL[cfg.dtype]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_cascade_irregular_groups(D, bs, dtype):
    groups = [3, 1, 3]
    prefix_blocks = [5, 0, 40]
    suffix_tokens = [7, 0, 33, 100, 1, 16, 0]
    case = _cascade_case(groups, prefix_blocks, suffix_tokens, 8, 2, D, bs, dtype, seed=D + bs)
    ref = _oracle(case)
    for pt in (0, 64, -1):                  # auto (split here), split, one pass
        err, idx, finite = max_abs_err(_run(case, pt), ref)
        assert finite and err <= TOL[dtype], (pt, err, idx)


# a prefix CTA takes 128 query rows: 128/G members; the last three shapes
# split a group over several CTAs (G = 3 leaves 2 rows of each CTA unused)
@pytest.mark.parametrize("G,size", [(1, 8), (4, 8), (8, 16), (4, 32), (8, 40), (3, 50), (1, 130)])
def test_cascade_group_shapes(G, size):
    Hkv = 2
    groups = [size, size]
    case = _cascade_case(groups, [12, 20], list(range(1, 2 * size + 1)), G * Hkv, Hkv, 128, 16,
                         "bf16", seed=G * 100 + size)
    ref = _oracle(case)
    for pt in (0, -1):
        err, idx, finite = max_abs_err(_run(case, pt), ref)
        assert finite and err <= TOL["bf16"], (pt, err, idx)


@pytest.mark.parametrize("D,bs,dtype", [(128, 16, "bf16"), (64, 32, "f16"), (128, 32, "f16"),
                                        (64, 16, "bf16")])
def test_cascade_sequences_outside_groups(D, bs, dtype):
    """Sequences before and after the groups attend over their own blocks only."""
    groups = [4, 2]
    before, after = 3, 5
    B = before + sum(groups) + after
    suffix = [1, 0, 40, 17, 16, 15, 64, 65, 0, 3, 100, 33, 2, 129][:B]
    case = _cascade_case(groups, [6, 3], suffix, 8, 2, D, bs, dtype, seed=D * 3 + bs, before=before,
                         after=after)
    ref = _oracle(case)
    for pt in (64, -1):
        err, idx, finite = max_abs_err(_run(case, pt), ref)
        assert finite and err <= TOL[dtype], (pt, err, idx)


@pytest.mark.parametrize("bs", [16, 32])
def test_cascade_one_pass_long_and_edge_suffixes(bs):
    """Own-block lengths around block and tile edges, and own blocks beyond one
    32-entry window of block ids (more than 512 tokens at 16 per block)."""
    suffix = [0, 1, bs - 1, bs, bs + 1, 63, 64, 65, 127, 128, 129, 700, 1100, 2, 0, 513]
    groups = [8, 8]
    case = _cascade_case(groups, [9, 1], suffix, 16, 4, 128, bs, "bf16", seed=bs + 5)
    ref = _oracle(case)
    for pt in (0, -1, 128):
        err, idx, finite = max_abs_err(_run(case, pt), ref)
        assert finite and err <= TOL["bf16"], (pt, err, idx)


def test_cascade_one_pass_garbage_past_the_end():
    """Cells past each sequence's last token (in its last block) hold NaN: they
    are never weighted, so the output stays finite and within tolerance."""
    groups = [5, 3]
    suffix = [3, 17, 30, 1, 9, 40, 2, 33]
    case = _cascade_case(groups, [4, 2], suffix, 16, 4, 128, 16, "bf16", seed=91)
    ref = _oracle(case)
    bs = 16
    for b, n in enumerate(suffix):
        nb = -(-n // bs)
        if n % bs:
            blk = int(case["suffix_tables"][b, nb - 1])
            case["key_cache"][blk, n % bs:] = float("nan")
            case["value_cache"][blk, n % bs:] = float("nan")
    for pt in (64, -1):
        err, idx, finite = max_abs_err(_run(case, pt), ref)
        assert finite and err <= TOL["bf16"], (pt, err, idx)
