"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_static_workspace takes its split-plan workspace
from a fixed array the library reserves on each GPU, so nothing is allocated
when it runs.  Such callers include a serving runtime whose allocator owns the
whole device pool, or plain C code that has no device allocator at hand.  The
tests call it through the C ABI several times in a row, on different split
workloads (each call reuses the array the previous one left behind), and
check that every output equals, bit for bit, the regular entry point's with a
caller-provided workspace: both run the same kernels on the same plan.  One
plan needs the whole array but 16 bytes; one sequence more is refused.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import pagedkv, workloads
from tests.parity_util import custom

pytestmark = pytest.mark.gpu


def _entry():
    f = pkv.lib().pkv_paged_attention_decode_static_workspace
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.restype = i32
    f.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, ctypes.c_float, i32, P, i32, P]
    return f


def _inputs(cfg, batch):
    step = workloads.make_decode_step(cfg, batch=batch)
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in step.items()}


def _static_call(f, d, partition_tokens):
    B, Hq, D = d["query"].shape
    NB, bs, Hkv, _ = d["key_cache"].shape
    out = torch.empty_like(d["query"])
    st = f(d["query"].data_ptr(), d["key_cache"].data_ptr(), d["value_cache"].data_ptr(),
           d["block_tables"].data_ptr(), d["block_tables"].shape[1], d["context_lens"].data_ptr(),
           B, Hq, Hkv, D, bs, NB, d["scale"], partition_tokens, out.data_ptr(),
           pagedkv.BF16 if d["query"].dtype == torch.bfloat16 else pagedkv.F16,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pagedkv.OK, pkv.lib().pkv_last_error().decode()
    return out


def _regular_call(d, partition_tokens):
    return pkv.paged_attention_decode(d["query"], d["key_cache"], d["value_cache"],
                                      d["block_tables"], d["context_lens"], d["scale"],
                                      partition_tokens=partition_tokens)


def _need(d, partition_tokens):
    B, Hq, D = d["query"].shape
    NB, bs, Hkv, _ = d["key_cache"].shape
    return pkv.decode_workspace_bytes(B, Hq, Hkv, D, d["block_tables"].shape[1], bs,
                                      partition_tokens)


# 205 sequences x 10 query heads x 31 partitions x (64 + 2) floats: 16 bytes
# short of the 16 MiB array (records of (D + 2) * 4 bytes never fill it exactly)
_NEAR_CAP = dict(B=205, Hq=10, Hkv=2, D=64, bs=16, pt=32, span=992)


def _near_cap_inputs(batch):
    c = _NEAR_CAP
    g = torch.Generator().manual_seed(31)
    lens = torch.randint(1, c["span"] + 1, (batch,), generator=g).tolist()
    lens[0] = c["span"]                              # 62 blocks: 31 partitions of 32 tokens
    step = custom("near_cap", batch, c["Hq"], c["Hkv"], c["D"], c["bs"], "bf16", lens, seed=32)
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in step.items()}


def test_static_workspace_matches_regular_entry_twice_in_a_row():
    f = _entry()
    cases = [
        (workloads.CONFIGS["long_split"], 4, 512),      # 64 partitions of 512 tokens, bf16
        (workloads.CONFIGS["llama13b_mha"], 12, 256),   # 8 partitions of 256 tokens, fp16
    ]
    pkv.device_flags(clear=True)
    for cfg, batch, pt in cases:
        d = _inputs(cfg, batch)
        assert _need(d, pt) > 0
        ref = _regular_call(d, pt)
        got = _static_call(f, d, pt)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (cfg.name, (got.float() - ref.float()).abs().max().item())
    assert pkv.device_flags() == 0


def test_static_workspace_plan_that_fills_the_array():
    f = _entry()
    c = _NEAR_CAP
    pkv.device_flags(clear=True)
    # a first call leaves other records in the array
    d0 = _inputs(workloads.CONFIGS["long_split"], 2)
    first = _static_call(f, d0, 512)
    assert torch.equal(first, _regular_call(d0, 512))
    d = _near_cap_inputs(c["B"])
    need = _need(d, c["pt"])
    assert pkv.decode_plan(c["B"], c["Hq"], c["Hkv"], c["D"], d["block_tables"].shape[1], c["bs"],
                           c["pt"]) == (c["pt"], 31)
    assert need == c["B"] * c["Hq"] * 31 * (c["D"] + 2) * 4 == (16 << 20) - 16
    ref = _regular_call(d, c["pt"])
    for _ in range(2):                                # twice: the second reuses the first's records
        got = _static_call(f, d, c["pt"])
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (got.float() - ref.float()).abs().max().item()
    assert pkv.device_flags() == 0


def test_static_workspace_rejects_plans_beyond_its_size():
    f = _entry()
    # 4096 sequences x 64 heads x 64 partitions needs far more than 16 MiB
    st = f(None, None, None, None, 2048, None, 4096, 64, 8, 128, 32, 1 << 20, 0.1, 32, None,
           pagedkv.BF16, None)
    assert st == pagedkv.ERR_WORKSPACE
    assert "static workspace" in pkv.lib().pkv_last_error().decode()
    # one sequence more than the plan that fills the array is refused, before any launch
    c = _NEAR_CAP
    st = f(None, None, None, None, c["span"] // c["bs"], None, c["B"] + 1, c["Hq"], c["Hkv"], c["D"],
           c["bs"], 1 << 16, 0.125, c["pt"], None, pagedkv.BF16, None)
    assert st == pagedkv.ERR_WORKSPACE
