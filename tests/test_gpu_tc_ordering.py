"""Repeated runs of the tcgen05 attention pipeline (chunked prefill and the
shared-prefix pass of cascade decode) against the fp64 oracle.

The pipeline hands scores, weights and the output accumulator between the
tensor core and the softmax warps through tensor memory and mbarriers; an
ordering mistake there shows up as intermittently wrong rows, not as a
failure of any single run.  Each case runs many times on a full GPU (many
CTAs in flight at once) and checks that

  * every run is bit-identical to the first (the kernels are deterministic:
    no atomics, a fixed order of operations per row), and
  * the first run matches the oracle within the parity tolerance,

with the device flag word clear afterwards (no bounded wait expired).

The prefill case is the shape that exposed an ordering fault before: chunks
of 7 tokens over 520 cached keys, group size 4, bf16 (9 key tiles, so the
last P V phases are still open when the softmax warps finish).  The cascade
cases are the shared-prefix workload's shape at reduced batch: groups of 8
samples sharing a 2000-token prefix ("23.1 vLLM：高吞吐推理框架原理与部署",
section 二.3), through the split plan and through the one pass.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from tests.parity_util import NTHREADS, TOL, custom, max_abs_err, u16
from tests.test_gpu_cascade import _cascade_case, _oracle

pytestmark = pytest.mark.gpu

PREFILL_RUNS = 120
CASCADE_RUNS = 60


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield
    assert pkv.device_flags() == 0


def test_prefill_short_chunks_over_long_context_repeated():
    B, Hq, Hkv, D, bs = 96, 16, 4, 128, 16
    lens = [520] * B
    chunks = [7] * B
    step = custom("order", B, Hq, Hkv, D, bs, "bf16", lens, seed=520)
    g = torch.Generator().manual_seed(521)
    T = sum(chunks)
    q = torch.randn(T, Hq, D, generator=g).to(torch.bfloat16)
    qs = torch.tensor(np.concatenate([[0], np.cumsum(chunks)]), dtype=torch.int32)
    ref = oracle.paged_attention_prefill(u16(q), qs.numpy(), u16(step["key_cache"]),
                                         u16(step["value_cache"]), step["block_tables"].numpy(),
                                         step["context_lens"].numpy(), step["scale"], "bf16",
                                         nthreads=NTHREADS)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in step.items()}
    qd, qsd = q.cuda(), qs.cuda()
    runs = [torch.empty_like(qd) for _ in range(PREFILL_RUNS)]
    for out in runs:                        # back to back on one stream, no sync in between
        pkv.paged_attention_prefill(qd, qsd, max(chunks), d["key_cache"], d["value_cache"],
                                    d["block_tables"], d["context_lens"], step["scale"], out=out)
    torch.cuda.synchronize()
    err, idx, finite = max_abs_err(runs[0], ref)
    assert finite and err <= TOL["bf16"], (err, idx)
    bad = [i for i, r in enumerate(runs) if not torch.equal(r, runs[0])]
    assert not bad, f"{len(bad)} of {PREFILL_RUNS} runs differ from the first: {bad[:10]}"


@pytest.mark.parametrize("partition_tokens", [512, -1])   # prefix pass + merge; one pass
def test_cascade_repeated(partition_tokens):
    groups = [8] * 12                        # 96 sequences, 12 prompts x 8 samples
    rng = np.random.default_rng(7)
    suffix = [int(x) for x in rng.integers(1, 257, size=sum(groups))]
    case = _cascade_case(groups, [125] * len(groups), suffix, 32, 8, 128, 16, "bf16", seed=2000)
    ref = _oracle(case)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    runs = [pkv.paged_attention_decode_cascade(
        d["query"], d["key_cache"], d["value_cache"], d["prefix_tables"], d["prefix_lens"],
        d["group_start"], d["suffix_tables"], d["suffix_lens"], d["scale"],
        max_group_size=d["max_group_size"], partition_tokens=partition_tokens)
        for _ in range(CASCADE_RUNS)]
    torch.cuda.synchronize()
    err, idx, finite = max_abs_err(runs[0], ref)
    assert finite and err <= TOL["bf16"], (err, idx)
    bad = [i for i, r in enumerate(runs) if not torch.equal(r, runs[0])]
    assert not bad, f"{len(bad)} of {CASCADE_RUNS} runs differ from the first: {bad[:10]}"
