"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_static_workspace takes its split-plan workspace
from a fixed array the library reserves on each GPU, so nothing is allocated
when it runs.  This test calls it through the C ABI twice in a row, on two
different split workloads (the second call reuses the array the first one
left behind), and checks each output against the regular entry point with a
caller-provided workspace, within the parity tolerance of the other tests.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import pagedkv, workloads
from tests.parity_util import TOL

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


def test_static_workspace_matches_regular_entry_twice_in_a_row():
    f = _entry()
    cases = [
        (workloads.CONFIGS["long_split"], 4, 512),      # 64 partitions of 512 tokens, bf16
        (workloads.CONFIGS["llama13b_mha"], 12, 256),   # 8 partitions of 256 tokens, fp16
    ]
    pkv.device_flags(clear=True)
    for cfg, batch, pt in cases:
        d = _inputs(cfg, batch)
        B, Hq, D = d["query"].shape
        NB, bs, Hkv, _ = d["key_cache"].shape
        assert pkv.decode_workspace_bytes(B, Hq, Hkv, D, d["block_tables"].shape[1], bs, pt) > 0
        ref = pkv.paged_attention_decode(d["query"], d["key_cache"], d["value_cache"],
                                         d["block_tables"], d["context_lens"], d["scale"],
                                         partition_tokens=pt)
        got = _static_call(f, d, pt)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs().max().item()
        assert err <= TOL[cfg.dtype], (cfg.name, err)
    assert pkv.device_flags() == 0


def test_static_workspace_rejects_plans_beyond_its_size():
    f = _entry()
    # 4096 sequences x 64 heads x 64 partitions needs far more than 16 MiB
    st = f(None, None, None, None, 2048, None, 4096, 64, 8, 128, 32, 1 << 20, 0.1, 32, None,
           pagedkv.BF16, None)
    assert st == pagedkv.ERR_WORKSPACE
    assert "static workspace" in pkv.lib().pkv_last_error().decode()
