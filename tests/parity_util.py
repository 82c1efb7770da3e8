"""Shared helpers for GPU parity tests: run a decode step through the C ABI
and through the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
import paged_kv_cache_468_b200 as pkv
from paged_kv_cache_468_b200 import workloads

# max-abs tolerances against the unrounded fp64 oracle, with fp32 accumulation
TOL = {"f16": 2e-3, "bf16": 1e-2}
NTHREADS = max(1, min(64, os.cpu_count() or 1))


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_device(step: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in step.items()}


def oracle_step(step: dict, write: bool = True) -> tuple:
    """fp64 expected output [B, Hq, D] (after the slot_mapping write) and the
    caches as the oracle leaves them (uint16 codes)."""
    kc = u16(step["key_cache"]).copy()
    vc = u16(step["value_cache"]).copy()
    if write:
        oracle.kv_cache_write(u16(step["new_key"]), u16(step["new_value"]),
                              step["slot_mapping"].numpy(), kc, vc, step["block_size"])
    out = oracle.paged_attention_decode(u16(step["query"]), kc, vc, step["block_tables"].numpy(),
                                        step["context_lens"].numpy(), step["scale"], step["dtype"],
                                        nthreads=NTHREADS)
    return out, kc, vc


def gpu_step(d: dict, write: bool = True, partition_tokens=None) -> torch.Tensor:
    """The hot path on the GPU: slot_mapping write, then decode (in place on d's caches)."""
    if write:
        pkv.kv_cache_write(d["new_key"], d["new_value"], d["slot_mapping"], d["key_cache"],
                           d["value_cache"])
    pt = d["partition_tokens"] if partition_tokens is None else partition_tokens
    return pkv.paged_attention_decode(d["query"], d["key_cache"], d["value_cache"],
                                      d["block_tables"], d["context_lens"], d["scale"],
                                      partition_tokens=pt)


def max_abs_err(gpu_out: torch.Tensor, ref: np.ndarray) -> tuple:
    got = gpu_out.float().cpu().double().numpy()
    err = np.abs(got - ref)
    idx = np.unravel_index(int(np.argmax(err)), err.shape)
    _log_error(float(err.max()), idx)
    return float(err.max()), idx, bool(np.isfinite(got).all())


def _log_error(err: float, idx) -> None:
    """Append (test, max-abs error) to the file named by PKV_PARITY_LOG, if set."""
    path = os.environ.get("PKV_PARITY_LOG")
    if not path:
        return
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, "max_abs_err": err, "at": [int(i) for i in idx]}) + "\n")


def custom(name, B, Hq, Hkv, D, bs, dtype, lens, seed=123, pt=0):
    cfg = workloads.DecodeConfig(name, batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                 block_size=bs, dtype=dtype, ctx_lo=1, ctx_hi=max(lens), seed=seed,
                                 partition_tokens=pt)
    return workloads.make_decode_step(cfg, context_lens=list(lens))
