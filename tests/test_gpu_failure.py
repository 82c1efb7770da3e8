"""Failure detection without a GPU fault: a pipeline wait that never completes
gives up after its limit, sets a flag the host reads, and the context stays
usable (checked by a normal write + decode afterwards)."""
import time

import pytest
import torch

import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import pagedkv, workloads
from tests.parity_util import TOL, gpu_step, max_abs_err, oracle_step, to_device

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    pkv.device_flags(clear=True)
    t0 = time.time()
    pkv.selftest_bounded_wait(50_000_000)          # 50 ms limit; nothing ever arrives
    flags = pkv.device_flags(clear=True)           # synchronises
    elapsed = time.time() - t0
    assert flags & pagedkv.DEVFLAG_WAIT_TIMEOUT
    assert elapsed < 5.0
    # the context is still usable
    step = workloads.make_decode_step(workloads.CONFIGS["tiny_mha"])
    ref, _, _ = oracle_step(step)
    out = gpu_step(to_device(step))
    err, _, finite = max_abs_err(out, ref)
    assert finite and err <= TOL["f16"]
    assert pkv.device_flags() == 0


def test_selftest_rejects_bad_limits():
    with pytest.raises(pagedkv.PagedKVError):
        pkv.selftest_bounded_wait(0)
