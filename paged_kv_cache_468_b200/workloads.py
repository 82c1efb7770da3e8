"""Seeded synthetic workloads for paged decode (shared by tests, bench and smoke).

This module only *draws inputs*: sizes, N(0,1) values, context lengths and
the random physical placement of KV blocks.  It holds none of the method's
arithmetic and imports neither the CUDA library nor the oracle, so both
sides of a parity check can consume the same tensors.

Shapes follow the pages' statement of the problem: the caches are
``[num_blocks, block_size, num_kv_heads, head_dim]``, ``block_tables`` is
``[batch, max_blocks]`` with one row of physical block ids per sequence, and
``context_lens`` holds each sequence's token count ("大模型推理框架 vLLM 源码
解析 一", section 三).  Blocks are scattered in a shared pool and need not be
contiguous ("23.1 vLLM：高吞吐推理框架原理与部署", section 二.2).

Every workload is one decode step: each sequence's newest token (logical
position ``context_len - 1``) has its K/V written through ``slot_mapping``
("大模型推理框架VLLM-0.7.3源码", sections 2.1 / 3.3), then every sequence's
single query token attends over its first ``context_len`` tokens.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

_TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                      # "f16" | "bf16"
    ctx_lo: int                     # context length ~ U{ctx_lo .. ctx_hi}
    ctx_hi: int
    seed: int
    pool_factor: float = 1.1        # pool = ceil(pool_factor * blocks needed)
    pool_blocks: Optional[int] = None   # fixed pool size (overrides pool_factor)
    shared_prefix: int = 0          # tokens of a prefix shared by `samples` rows
    samples: int = 1                # sequences per prompt that share the prefix
    partition_tokens: int = 0       # 0 = library's automatic choice
    description: str = ""

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def max_context(self) -> int:
        return self.shared_prefix + self.ctx_hi if self.shared_prefix else self.ctx_hi

    @property
    def max_blocks(self) -> int:
        return -(-self.max_context // self.block_size)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


# The five workloads, with the sizes, distributions and structure stated for them.
CONFIGS = {
    "tiny_mha": DecodeConfig(
        "tiny_mha", batch=4, num_heads=8, num_kv_heads=8, head_dim=64, block_size=16,
        dtype="f16", ctx_lo=1, ctx_hi=200, seed=0, pool_blocks=64,
        description="batch 4, 8/8 heads, D 64, bs 16, fp16, L~U[1,200], 64-block pool"),
    "llama3_8b_gqa": DecodeConfig(
        "llama3_8b_gqa", batch=256, num_heads=32, num_kv_heads=8, head_dim=128,
        block_size=16, dtype="bf16", ctx_lo=512, ctx_hi=640, seed=1,
        description="Llama-3-8B-shaped GQA: batch 256, 32/8 heads, D 128, bs 16, bf16, "
                    "L~U[512,640], pool 1.1x need"),
    "llama13b_mha": DecodeConfig(
        "llama13b_mha", batch=50, num_heads=40, num_kv_heads=40, head_dim=128,
        block_size=16, dtype="f16", ctx_lo=64, ctx_hi=2048, seed=2,
        description="Llama-13B-shaped MHA: batch 50, 40 heads, D 128, bs 16, fp16, "
                    "L~U[64,2048], pool 1.1x need, 50-token slot_mapping write"),
    "shared_prefix": DecodeConfig(
        "shared_prefix", batch=256, num_heads=32, num_kv_heads=8, head_dim=128,
        block_size=16, dtype="bf16", ctx_lo=1, ctx_hi=256, seed=3,
        shared_prefix=2000, samples=8,
        description="32 prompts x 8 samples, 32/8 heads, D 128, bs 16, bf16, 2000-token "
                    "shared prefix + U[1,256] private tokens, pool 1.1x unique need"),
    "long_split": DecodeConfig(
        "long_split", batch=8, num_heads=32, num_kv_heads=8, head_dim=128, block_size=32,
        dtype="bf16", ctx_lo=16384, ctx_hi=32768, seed=4, partition_tokens=512,
        description="long context: batch 8, 32/8 heads, D 128, bs 32, bf16, "
                    "L~U[16384,32768], 512-token partitions + LSE merge"),
}
HEADLINE = "llama3_8b_gqa"


def _randn(shape, gen, dtype, chunk_rows: int = 1024) -> torch.Tensor:
    """N(0,1) in fp32, rounded to `dtype` (round-to-nearest-even), drawn in
    row chunks so a multi-GB pool never needs a full fp32 copy."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        flat[r0:r1] = torch.randn((r1 - r0, flat.shape[1]), generator=gen,
                                  dtype=torch.float32).to(dtype)
    return out


def make_decode_step(cfg: DecodeConfig, batch: Optional[int] = None,
                     context_lens: Optional[list] = None) -> dict:
    """Draw one decode step of `cfg` on the CPU.

    Returns a dict of CPU tensors:
      query        [B, Hq, D]            dtype
      key_cache    [NB, bs, Hkv, D]      dtype (every slot N(0,1), used or not)
      value_cache  [NB, bs, Hkv, D]
      block_tables [B, max_blocks]       int32 (unused entries -1)
      context_lens [B]                   int32
      new_key      [B, Hkv, D]           the newest token's K, written before decode
      new_value    [B, Hkv, D]
      slot_mapping [B]                   int64, the cell of position context_len-1
    plus python scalars `scale`, `dtype`, `block_size`, `partition_tokens`.
    `batch` / `context_lens` override the config (for small or edge cases).
    """
    g = torch.Generator().manual_seed(cfg.seed)
    tdt = _TORCH_DTYPE[cfg.dtype]
    B = batch if batch is not None else cfg.batch
    bs, Hkv, D = cfg.block_size, cfg.num_kv_heads, cfg.head_dim

    # context lengths
    if context_lens is not None:
        lens = torch.tensor(context_lens, dtype=torch.int64)
        B = len(context_lens)
        prefix = 0
        samples = 1
    elif cfg.shared_prefix:
        prefix, samples = cfg.shared_prefix, cfg.samples
        assert B % samples == 0
        tails = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (B,), generator=g)
        lens = prefix + tails
    else:
        prefix, samples = 0, 1
        lens = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (B,), generator=g)
    max_len = int(lens.max()) if B else 0
    if context_lens is None:
        max_blocks = cfg.max_blocks
    else:
        max_blocks = max(1, -(-max_len // bs))

    # block demand: the shared prefix's full blocks are stored once per prompt
    shared_full = prefix // bs
    need = 0
    for b in range(B):
        nblk = -(-int(lens[b]) // bs)
        need += nblk - (shared_full if (samples > 1 and b % samples != 0) else 0)
    if cfg.pool_blocks is not None and context_lens is None:
        nb = cfg.pool_blocks
    else:
        nb = max(1, math.ceil(cfg.pool_factor * need))
    assert nb >= need, (nb, need)

    # random physical placement: a seeded permutation of the pool, handed out in order
    perm = torch.randperm(nb, generator=g).tolist()
    tables = torch.full((B, max_blocks), -1, dtype=torch.int32)
    cursor = 0
    prompt_prefix = None
    for b in range(B):
        nblk = -(-int(lens[b]) // bs)
        row = []
        if samples > 1:
            if b % samples == 0:
                prompt_prefix = perm[cursor:cursor + shared_full]
                cursor += shared_full
            row.extend(prompt_prefix)
        rest = nblk - len(row)
        row.extend(perm[cursor:cursor + rest])
        cursor += rest
        tables[b, :nblk] = torch.tensor(row, dtype=torch.int32)

    query = _randn((B, cfg.num_heads, D), g, tdt)
    key_cache = _randn((nb, bs, Hkv, D), g, tdt)
    value_cache = _randn((nb, bs, Hkv, D), g, tdt)
    new_key = _randn((B, Hkv, D), g, tdt)
    new_value = _randn((B, Hkv, D), g, tdt)

    # the newest token of each sequence sits at logical position L-1
    slots = torch.empty(B, dtype=torch.int64)
    for b in range(B):
        pos = int(lens[b]) - 1
        if pos < 0:
            slots[b] = -1
        else:
            slots[b] = int(tables[b, pos // bs]) * bs + pos % bs

    return dict(query=query, key_cache=key_cache, value_cache=value_cache,
                block_tables=tables, context_lens=lens.to(torch.int32),
                new_key=new_key, new_value=new_value, slot_mapping=slots,
                scale=cfg.scale, dtype=cfg.dtype, block_size=bs,
                partition_tokens=cfg.partition_tokens)


def kv_bytes(context_lens, num_kv_heads: int, head_dim: int, esize: int) -> int:
    """K+V bytes one decode step reads: every cached token row, for K and V."""
    return int(sum(int(x) for x in context_lens)) * num_kv_heads * head_dim * esize * 2


def cascade_inputs(step: dict, prefix_tokens: int, samples: int) -> dict:
    """Shared-prefix description of a step whose consecutive groups of
    `samples` sequences share their first `prefix_tokens` tokens' blocks (as
    make_decode_step builds them): one prefix table per group (the group's
    first sequence's leading blocks) and each sequence's remaining blocks.
    Only whole blocks are shared, so the prefix is rounded down to a block
    multiple and the rest of a partly shared block stays in the suffix."""
    bs = step["block_size"]
    tables, lens = step["block_tables"], step["context_lens"]
    B = tables.shape[0]
    assert B % samples == 0
    pb = prefix_tokens // bs
    groups = B // samples
    prefix_tables = tables[::samples, :max(pb, 1)].clone().contiguous()
    prefix_lens = torch.full((groups,), pb * bs, dtype=torch.int32)
    group_start = torch.arange(0, B + 1, samples, dtype=torch.int32)
    msb = max(1, tables.shape[1] - pb)
    suffix_tables = torch.full((B, msb), -1, dtype=torch.int32)
    suffix_tables[:, :tables.shape[1] - pb] = tables[:, pb:]
    suffix_lens = (lens - pb * bs).clamp(min=0).to(torch.int32)
    return dict(prefix_tables=prefix_tables, prefix_lens=prefix_lens, group_start=group_start,
                suffix_tables=suffix_tables, suffix_lens=suffix_lens, max_group_size=samples)
