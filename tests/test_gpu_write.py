"""kv_cache_write on the GPU vs the oracle: bit-exact ("大模型推理框架VLLM-0.7.3源码",
sections 2.1 / 3.3: slot_mapping names each current token's cell)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import pagedkv, workloads
from tests.parity_util import custom, to_device, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_flags():
    pkv.device_flags(clear=True)
    yield


def _check_write(step):
    d = to_device(step)
    pkv.kv_cache_write(d["new_key"], d["new_value"], d["slot_mapping"], d["key_cache"],
                       d["value_cache"])
    kc = u16(step["key_cache"]).copy()
    vc = u16(step["value_cache"]).copy()
    oracle.kv_cache_write(u16(step["new_key"]), u16(step["new_value"]),
                          step["slot_mapping"].numpy(), kc, vc, step["block_size"])
    assert np.array_equal(u16(d["key_cache"]), kc)
    assert np.array_equal(u16(d["value_cache"]), vc)
    assert pkv.device_flags() == 0


@pytest.mark.parametrize("name", sorted(workloads.CONFIGS))
def test_write_bit_exact_full_config(name):
    _check_write(workloads.make_decode_step(workloads.CONFIGS[name]))


def test_write_random_unique_slots_many_tokens():
    """Many tokens at random unique slots anywhere in the pool (ragged vector count)."""
    step = custom("w", 4, 8, 8, 64, 16, "f16", [40, 50, 60, 70], seed=5)
    g = torch.Generator().manual_seed(9)
    NB, bs, Hkv, D = 100, 16, 8, 64
    step["key_cache"] = torch.randn(NB, bs, Hkv, D, generator=g).half()
    step["value_cache"] = torch.randn(NB, bs, Hkv, D, generator=g).half()
    T = 1000
    step["new_key"] = torch.randn(T, Hkv, D, generator=g).half()
    step["new_value"] = torch.randn(T, Hkv, D, generator=g).half()
    step["slot_mapping"] = torch.randperm(NB * bs, generator=g)[:T].to(torch.int64)
    step["slot_mapping"][::7] = -1                      # padding tokens
    _check_write(step)


def test_write_out_of_range_slot_sets_flag_and_skips():
    step = custom("w", 2, 8, 2, 128, 16, "bf16", [5, 9], seed=6)
    d = to_device(step)
    NB, bs = step["key_cache"].shape[:2]
    before = u16(d["key_cache"]).copy()
    slots = torch.tensor([NB * bs, 3], dtype=torch.int64, device="cuda")   # first one is out
    pkv.kv_cache_write(d["new_key"], d["new_value"], slots, d["key_cache"], d["value_cache"])
    assert pkv.device_flags() & pagedkv.DEVFLAG_SLOT_RANGE
    after = u16(d["key_cache"])
    flat_b = before.reshape(NB * bs, -1)
    flat_a = after.reshape(NB * bs, -1)
    assert np.array_equal(flat_a[3], u16(step["new_key"][1]).reshape(-1))
    mask = np.ones(NB * bs, bool)
    mask[3] = False
    assert np.array_equal(flat_a[mask], flat_b[mask])


def test_write_zero_tokens_is_noop():
    step = custom("w", 1, 8, 8, 64, 16, "f16", [3], seed=7)
    d = to_device(step)
    before = u16(d["key_cache"]).copy()
    e = torch.empty(0, 8, 64, dtype=torch.float16, device="cuda")
    pkv.kv_cache_write(e, e, torch.empty(0, dtype=torch.int64, device="cuda"), d["key_cache"],
                       d["value_cache"])
    assert np.array_equal(u16(d["key_cache"]), before)
