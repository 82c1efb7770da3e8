#!/usr/bin/env python3
"""Benchmark of the paged KV-cache decode step on B200.

One step = the whole hot path over one batch: kv_cache_write of every
sequence's newest token through slot_mapping, then paged_attention_decode of
one query token per sequence over its paged KV cache (plus the log-sum-exp
merge when the plan splits the context).  Inputs are seeded synthetic data of
the workload's shapes and distributions, resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed on host cores

Multi-GPU (launched by torch.distributed.run): every rank runs an independent
replica of the workload on its own GPU (the path shards by sequence with no
exchange step); the job time is the max over ranks and `value` counts the
bytes of all ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_468_b200 import workloads  # noqa: E402

METRIC = "paged decode attention KV GB/s (fraction of B200 HBM peak); decode tokens/s"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------- helpers --

def esize(dtype: str) -> int:
    return 2


def step_bytes(step: dict, cfg: workloads.DecodeConfig) -> dict:
    """Algorithmic bytes of one step (each byte the definition must touch once)."""
    lens = [int(x) for x in step["context_lens"]]
    B, Hq, D = step["query"].shape
    Hkv, bs, es = cfg.num_kv_heads, cfg.block_size, esize(cfg.dtype)
    kv = sum(lens) * Hkv * D * es * 2                         # K and V rows, read once
    qo = 2 * B * Hq * D * es                                  # query read + output written
    tables = 4 * (sum(-(-L // bs) for L in lens) + B)         # used table entries + lengths
    decode = kv + qo + tables
    T = int((step["slot_mapping"] >= 0).sum())
    write = 2 * (2 * T * Hkv * D * es) + 8 * T                # K,V rows read+written, slots
    # shared prefix: unique KV bytes (each shared block counted once)
    uniq_rows = 0
    seen = set()
    for b, L in enumerate(lens):
        nblk = -(-L // bs)
        for i in range(nblk):
            blk = int(step["block_tables"][b, i])
            if blk in seen:
                continue
            seen.add(blk)
            uniq_rows += min(bs, L - i * bs)
    kv_unique = uniq_rows * Hkv * D * es * 2
    return dict(kv=kv, kv_unique=kv_unique, decode=decode,
                decode_unique=decode - kv + kv_unique, write=write,
                tokens=B, kv_tokens=sum(lens))


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


# The DRAM traffic recorded for a workload's decode call (ncu) stays valid
# while the source text of the code that call runs is unchanged: the PTX
# wrappers, and the named functions / structs below.
CSRC = "paged_kv_cache_468_b200/csrc/"
_DECODE_CODE = [
    ("pkv_kernels.cuh", ["DecodeArgs", "DecodeShape", "pack2", "unpack2", "to_storage",
                         "attend_block", "paged_decode_kernel"]),
    ("pagedkv.cu", ["Tuning", "make_cache_map", "check_shapes", "plan", "launch_pdl",
                    "launch_decode", "dispatch_decode", "pkv_paged_attention_decode"]),
]
_SPLIT_CODE = [
    ("pkv_kernels.cuh", ["load_slice", "lse_merge_kernel", "lse_merge_wide_kernel"]),
    ("pagedkv.cu", ["launch_merge_d", "launch_merge"]),
]
_CASCADE_CODE = [
    ("pkv_kernels.cuh", ["CascadeArgs", "load_slice", "lse_merge_cascade_kernel"]),
    ("pkv_prefill.cuh", ["PrefillArgs", "PfShape", "PfBar", "TcMode", "tc_attend", "prefix_tc_kernel",
                         "cascade_tc_kernel"]),
    ("pagedkv.cu", ["make_query_map", "make_cache_map_4d", "CacheMaps", "make_cache_maps", "cascade_plan",
                    "launch_prefix",
                    "dispatch_prefix", "launch_cascade_one_pass", "dispatch_cascade_one_pass",
                    "cascade_one_pass", "pkv_paged_attention_decode_cascade"]),
]


def _definitions(src: str, name: str) -> list:
    """Source text of every definition of function / struct / enum `name`
    (with the template and attribute lines above it)."""
    import re
    out = []
    for m in re.finditer(r"\b(?:struct|enum)\s+" + re.escape(name) + r"\b[^;{]*\{|\b" + re.escape(name) + r"\s*\(", src):
        i = m.end()
        if src[m.end() - 1] == "(":                       # function: its parameter list
            depth = 1
            while i < len(src) and depth:
                depth += {"(": 1, ")": -1}.get(src[i], 0)
                i += 1
            j = i
            while j < len(src) and (src[j].isspace() or src[j:j + 5] in ("const", "noexc")):
                j += 5 if src[j:j + 5] in ("const", "noexc") else 1
            if j >= len(src) or src[j] != "{":
                continue                                  # a call or a declaration
            i = j + 1
        depth = 1
        while i < len(src) and depth:
            depth += {"{": 1, "}": -1}.get(src[i], 0)
            i += 1
        start = src.rfind("\n", 0, m.start()) + 1
        while start > 0:                                  # template / attribute lines above
            prev = src.rfind("\n", 0, start - 1) + 1
            line = src[prev:start - 1].strip()
            if not line or line.endswith((";", "}", "{")) or line.startswith("//"):
                break
            start = prev
        out.append(src[start:i])
    if not out:
        raise KeyError(name)
    return out


def decode_code_sha(split: bool, cascade: bool, root: str = ROOT) -> str:
    """Fingerprint of the code a decode call runs (16 hex digits)."""
    parts = list(_DECODE_CODE) + (list(_SPLIT_CODE) if split else []) + \
        (list(_CASCADE_CODE) if cascade else [])
    h = hashlib.sha256()
    with open(os.path.join(root, CSRC, "pkv_ptx.cuh"), "rb") as f:
        h.update(f.read())
    for fname, names in parts:
        with open(os.path.join(root, CSRC, fname), encoding="utf-8") as f:
            src = f.read()
        for n in names:
            for text in _definitions(src, n):
                h.update(text.encode())
    return h.hexdigest()[:16]


def committed_traffic(config_name: str, split: bool, cascade: bool):
    """DRAM bytes per decode call from the committed ncu summary, if they were
    taken on the code this call runs now (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    entry = d.get(config_name)
    if not entry or entry.get("source_sha") != decode_code_sha(split, cascade):
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while timed regions run.

    The sampler runs for the whole measurement; mark(True) / mark(False)
    bracket each timed region, and only samples inside a region count."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    PERIOD_MS = 50

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.windows = []          # [t_on, t_off] per timed region

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, on: bool):
        if on:
            self.windows.append([time.time(), None])
        elif self.windows and self.windows[-1][1] is None:
            self.windows[-1][1] = time.time()

    def _inside(self, t: float) -> bool:
        return any(a <= t <= (b if b is not None else float("inf")) + 0.06 for a, b in self.windows)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t, line in self.lines:
            if not self._inside(t):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                rows.append(parts)
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i].lower() == "active"})
        timed_s = sum((b or a) - a for a, b in self.windows)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "period_ms": self.PERIOD_MS,
                "timed_regions": len(self.windows), "timed_s": round(timed_s, 3)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Job time = the slowest rank's (all ranks take part)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Work of the whole job = the sum of every rank's (all ranks take part)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def replica_seed(cfg_seed: int, rank: int) -> int:
    """Each rank draws its own replica of the workload (its own sequences)."""
    return cfg_seed + 1000 * rank


def job_throughput(bytes_local: float, ms_local: float, world: int, device: str = "cuda") -> tuple:
    """(GB/s of the whole job, job ms): all ranks' bytes over the slowest rank's time."""
    ms = max_over_ranks(ms_local, world, device)
    total = sum_over_ranks(bytes_local, world, device)
    return total / (ms * 1e-3) / 1e9, ms


# ------------------------------------------------------- CPU oracle timing --

def oracle_sample_rate(step: dict, cfg, seconds: float, nthreads: int, max_seqs=None):
    """Run the fp64 oracle (write + decode) on the first sequences of the step
    until `seconds` pass; returns (GB/s, sample description, threads)."""
    import numpy as np
    import oracle

    def u16(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    B = step["query"].shape[0]
    n = B if max_seqs is None else max(1, min(B, max_seqs))
    q = u16(step["query"][:n])
    kc = u16(step["key_cache"]).copy()
    vc = u16(step["value_cache"]).copy()
    bt = step["block_tables"][:n].numpy()
    cl = step["context_lens"][:n].numpy()
    nk, nv = u16(step["new_key"][:n]), u16(step["new_value"][:n])
    slots = step["slot_mapping"][:n].numpy()
    sub = dict(step, query=step["query"][:n], context_lens=step["context_lens"][:n],
               block_tables=step["block_tables"][:n], slot_mapping=step["slot_mapping"][:n])
    nbytes = step_bytes(sub, cfg)
    per = nbytes["decode"] + nbytes["write"]
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.kv_cache_write(nk, nv, slots, kc, vc, cfg.block_size)
        oracle.paged_attention_decode(q, kc, vc, bt, cl, cfg.scale, cfg.dtype, nthreads=nthreads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return per * reps / el / 1e9, n, reps, el


def choose_oracle_seqs(step, cfg, nthreads, budget_s):
    """Largest prefix of the batch whose oracle step fits in budget_s."""
    _, _, _, el = oracle_sample_rate(step, cfg, 0.0, nthreads, max_seqs=1)
    B = step["query"].shape[0]
    return max(1, min(B, int(budget_s / max(el, 1e-6))))


L2_BYTES_B200 = 126 << 20     # the B200's L2; workloads whose K/V fit get an L2 flush per iteration


def fits_in_l2(nbytes: dict, l2_bytes: int = L2_BYTES_B200) -> bool:
    return nbytes["kv_unique"] <= l2_bytes


def workload_config(cfg, step: dict, nbytes: dict, world: int) -> dict:
    """The `config` object of a JSON line: the workload and how it is timed.
    Both arms (GPU and reference) print the same one for the same workload."""
    B, Hq, D = step["query"].shape
    NB, bs, Hkv, _ = step["key_cache"].shape
    l2_mib = L2_BYTES_B200 >> 20
    if fits_in_l2(nbytes):
        l2 = (f"inputs fit in L2 ({nbytes['kv_unique'] / 1e6:.1f} MB of K/V vs {l2_mib} MiB): each "
              f"timed iteration has its own CUDA events and a {2 * l2_mib} MiB buffer is written "
              f"between iterations, outside the events")
    else:
        l2 = (f"inputs larger than L2: {nbytes['kv_unique'] / 1e6:.0f} MB of K/V per step vs "
              f"{l2_mib} MiB L2, no flush")
    return {"workload": cfg.name, "description": cfg.description, "batch": int(B),
            "num_heads": int(Hq), "num_kv_heads": int(Hkv), "head_dim": int(D),
            "block_size": int(bs), "num_blocks": int(NB),
            "max_blocks": int(step["block_tables"].shape[1]),
            "context_tokens": int(nbytes["kv_tokens"]), "kv_dtype": cfg.dtype,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "l2": l2}


def run_reference(args, cfg, world, rank):
    """The oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return 0
    nthreads = os.cpu_count() or 1
    step = workloads.make_decode_step(dataclass_replace(cfg, seed=replica_seed(cfg.seed, 0)))
    nbytes = step_bytes(step, cfg)
    total_budget = args.reference_seconds
    per_step = total_budget / max(1, args.steps + args.warmup)
    nseq = choose_oracle_seqs(step, cfg, nthreads, per_step)
    for _ in range(args.warmup):
        oracle_sample_rate(step, cfg, 0.0, nthreads, max_seqs=nseq)
    t_total, gbs_bytes = 0.0, 0.0
    for _ in range(args.steps):
        gbs, n, reps, el = oracle_sample_rate(step, cfg, 0.0, nthreads, max_seqs=nseq)
        t_total += el
        gbs_bytes += gbs * el
    value = gbs_bytes / t_total
    sample = (f"first {nseq} of {cfg.batch} sequences per step (write + decode), "
              f"{args.steps} timed steps, fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, step, nbytes, world),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- GPU arm ----

def time_back_to_back(fn, n: int, stream) -> float:
    """ms per call of fn over n calls issued back to back: one CUDA event pair
    on the launching stream around all of them."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def time_each(fn, n: int, stream, flush_buf=None) -> list:
    """ms of each of n calls (an event pair around each); with flush_buf, a
    write of that buffer between calls, outside the events, so no call reads
    data an earlier one left in L2."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        if flush_buf is not None:
            flush_buf.fill_(i & 0xff)
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [x.elapsed_time(y) for x, y in evs]


class DecodeWorkload:
    """One workload resident on the GPU: its step inputs, the decode call
    (plain or cascade) and the step (slot_mapping write + decode)."""

    def __init__(self, pkv, cfg, dev, seed: int, partition_tokens, cascade_mode: str):
        self.pkv, self.cfg, self.dev = pkv, cfg, dev
        self.step = workloads.make_decode_step(dataclass_replace(cfg, seed=seed))
        self.nbytes = step_bytes(self.step, cfg)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.step.items()}
        self.d = d
        B, Hq, D = d["query"].shape
        NB, bs, Hkv, _ = d["key_cache"].shape
        MB = d["block_tables"].shape[1]
        self.B = int(B)
        self.pt_req = cfg.partition_tokens if partition_tokens is None else partition_tokens
        self.plan_pt, self.plan_np = pkv.decode_plan(B, Hq, Hkv, D, MB, bs, self.pt_req)
        self.cascade = cascade_mode == "on" or (cascade_mode == "auto" and cfg.shared_prefix > 0)
        ws_bytes = pkv.decode_workspace_bytes(B, Hq, Hkv, D, MB, bs, self.pt_req)
        self.launches_per_step = 2 + (1 if self.plan_np > 1 else 0)
        self.cas = None
        self.one_pass = False
        if self.cascade:
            self.cas = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in
                        workloads.cascade_inputs(self.step, cfg.shared_prefix, cfg.samples).items()}
            mpb, msb = self.cas["prefix_tables"].shape[1], self.cas["suffix_tables"].shape[1]
            ws_bytes = int(pkv.lib().pkv_decode_cascade_workspace_bytes(
                B, Hq, Hkv, D, mpb, msb, self.cas["max_group_size"], bs, self.pt_req))
            self.one_pass, self.plan_np = pkv.decode_cascade_plan(
                B, Hq, Hkv, D, mpb, msb, self.cas["max_group_size"],
                self.cas["prefix_tables"].shape[0], bs, self.pt_req)
            self.launches_per_step = 2 if self.one_pass else 4
        self.ws = torch.empty(max(16, ws_bytes), dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(d["query"])
        self.flush = fits_in_l2(self.nbytes)

    # the tensors a caller supplies every step (the rest stays resident: the pool)
    def step_input_names(self) -> list:
        names = ["query", "new_key", "new_value", "slot_mapping"]
        if self.cascade:
            return names + ["prefix_tables", "prefix_lens", "group_start", "suffix_tables",
                            "suffix_lens"]
        return names + ["block_tables", "context_lens"]

    def step_inputs(self) -> dict:
        src = dict(self.d)
        if self.cascade:
            src.update({k: v for k, v in self.cas.items() if isinstance(v, torch.Tensor)})
        return {k: src[k] for k in self.step_input_names()}

    def decode(self, x: dict = None, out=None):
        x = self.step_inputs() if x is None else x
        out = self.out if out is None else out
        d, pkv = self.d, self.pkv
        if self.cascade:
            return pkv.paged_attention_decode_cascade(
                x["query"], d["key_cache"], d["value_cache"], x["prefix_tables"], x["prefix_lens"],
                x["group_start"], x["suffix_tables"], x["suffix_lens"], d["scale"],
                max_group_size=self.cas["max_group_size"], partition_tokens=self.pt_req, out=out,
                workspace=self.ws)
        return pkv.paged_attention_decode(x["query"], d["key_cache"], d["value_cache"],
                                          x["block_tables"], x["context_lens"], d["scale"],
                                          partition_tokens=self.pt_req, out=out, workspace=self.ws)

    def write(self, x: dict = None):
        x = self.step_inputs() if x is None else x
        self.pkv.kv_cache_write(x["new_key"], x["new_value"], x["slot_mapping"], self.d["key_cache"],
                                self.d["value_cache"])

    def one_step(self):
        self.write()
        self.decode()

    def kernel_name(self) -> str:
        if self.cascade and self.one_pass:
            return "cascade_tc_kernel (one pass: prefix and own blocks)"
        if self.cascade:
            return "prefix_tc_kernel + paged_decode_kernel (suffixes) + lse_merge_cascade_kernel"
        return "paged_decode_kernel" + (" + lse_merge_kernel" if self.plan_np > 1 else "")

    def traffic(self):
        return committed_traffic(self.cfg.name, self.plan_np > 1 and not self.cascade, self.cascade)

    def method(self) -> dict:
        if self.cascade:
            return {"cascade": "one pass" if self.one_pass else "split",
                    "prefix_partitions": self.plan_np}
        return {"partition_tokens": self.plan_pt, "num_partitions": self.plan_np, "cascade": False}


def measure_decode_launches(w: DecodeWorkload, n: int, stream, flush_buf, sampler=None) -> dict:
    """The decode call alone, n launches: the mean from one event pair around
    back-to-back launches (per-launch events with an L2 flush in between for
    workloads that fit in L2) and the spread from per-launch events."""
    for _ in range(3):
        w.decode()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark(True)
    if w.flush:
        each = time_each(w.decode, n, stream, flush_buf)
        mean = statistics.mean(each)
        timing = (f"{n} launches, an event pair around each, a {flush_buf.numel() >> 20} MiB "
                  f"L2 flush between them")
    else:
        mean = time_back_to_back(w.decode, n, stream)
        each = time_each(w.decode, min(n, 2000), stream)
        timing = f"mean: one event pair around {n} back-to-back launches; spread: per-launch events"
    if sampler:
        sampler.mark(False)
    q = statistics.quantiles(each, n=10) if len(each) >= 10 else [min(each)] * 9
    return {"mean_ms": mean, "median_ms": statistics.median(each), "p10_ms": q[0],
            "p90_ms": q[-1], "n": n, "timing": timing}


def read_ceiling(pkv, dev, stream, nbytes: int = 2 << 30, reps: int = 40, same_bytes: int = 0) -> dict:
    """Read-only HBM streaming rate (16-byte loads over nbytes), best over a
    few grid sizes: the ceiling of a kernel that only reads.  With same_bytes,
    also the rate of reading just that many bytes (the decode call's) as
    scattered 4 KiB chunks, launched back to back like the decode: a short
    kernel pays its ramp-up and drain too."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    buf.fill_(1)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    rates = {}
    for per_sm in (2, 4, 8):
        grid = sms * per_sm
        fn = lambda: pkv.hbm_read_probe(buf, sink, grid)
        for _ in range(3):
            fn()
        ms = time_back_to_back(fn, reps, stream)
        rates[str(grid)] = round(nbytes / (ms * 1e-3) / 1e9, 1)
    # the same bytes as 4 KiB chunks in a random order: a paged cache's blocks
    # are scattered over the pool, and one kv head of one block (16 rows of a
    # 128-wide head) is 4 KiB
    chunk = 4096
    order = torch.randperm(nbytes // chunk, generator=torch.Generator().manual_seed(5)).to(
        torch.int32).to(dev)
    gather = {}
    for per_sm in (2, 4, 8):
        grid = sms * per_sm
        fn = lambda: pkv.hbm_gather_probe(buf, chunk, order, sink, grid)
        for _ in range(3):
            fn()
        ms = time_back_to_back(fn, reps, stream)
        gather[str(grid)] = round(nbytes / (ms * 1e-3) / 1e9, 1)
    same = {}
    n_same = min(-(-same_bytes // chunk), nbytes // chunk)
    if n_same > 0:
        # the first n_same chunks of the buffer (a pool the size of the decode's
        # blocks), each read once, in a random order
        buf_s = buf[:n_same * chunk]
        order_s = torch.randperm(n_same, generator=torch.Generator().manual_seed(6)).to(torch.int32).to(dev)
        launches = max(reps, int(0.3 / (n_same * chunk / 7e12)))    # ~0.3 s at 7 TB/s
        for per_sm in (2, 4, 8):
            grid = sms * per_sm
            fn = lambda: pkv.hbm_gather_probe(buf_s, chunk, order_s, sink, grid)
            for _ in range(3):
                fn()
            ms = time_back_to_back(fn, launches, stream)
            same[str(grid)] = round(n_same * chunk / (ms * 1e-3) / 1e9, 1)
        del order_s, buf_s
    del buf, order
    r = {"gbs": max(rates.values()), "bytes": nbytes, "reps": reps, "by_grid": rates,
         "kernel": "hbm_read_probe_kernel (16-byte ld.global.nc, 8 in flight per thread)",
         "gather_4k_gbs": max(gather.values()), "gather_4k_by_grid": gather,
         "gather_kernel": "hbm_gather_probe_kernel (4 KiB chunks in a random order, a warp per chunk)"}
    if same:
        r.update({"same_size_gather_gbs": max(same.values()), "same_size_bytes": n_same * chunk,
                  "same_size_by_grid": same, "same_size_launches": launches})
    return r


def roofline_entry(w: DecodeWorkload, t: dict, peaks: dict, ceiling) -> dict:
    bytes_ = w.nbytes["decode_unique"]
    achieved = bytes_ / (t["mean_ms"] * 1e-3) / 1e9
    r = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
         "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": w.traffic(),
         "peak_source": (peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, a copy: read + write)"
                         if peaks["source"] == "measured" else "fallback 6650 GB/s (copy)"),
         "kernel": w.kernel_name(), "bytes_per_launch": bytes_,
         "launch_ms": round(t["mean_ms"], 5), "launch_ms_median": round(t["median_ms"], 5),
         "launch_ms_p10": round(t["p10_ms"], 5), "launch_ms_p90": round(t["p90_ms"], 5),
         "launches_timed": t["n"], "timing": t["timing"],
         "frac_median": round(bytes_ / (t["median_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
         "frac_of_8000": round(achieved / 8000.0, 4)}
    if ceiling:
        r["read_ceiling_gbs"] = ceiling["gbs"]
        r["frac_of_read_ceiling"] = round(achieved / ceiling["gbs"], 4)
        r["gather_ceiling_gbs"] = ceiling["gather_4k_gbs"]
        r["frac_of_gather_ceiling"] = round(achieved / ceiling["gather_4k_gbs"], 4)
        if "same_size_gather_gbs" in ceiling and abs(ceiling["same_size_bytes"] - bytes_) <= 0.1 * bytes_:
            r["same_size_gather_gbs"] = ceiling["same_size_gather_gbs"]
            r["frac_of_same_size_gather"] = round(achieved / ceiling["same_size_gather_gbs"], 4)
    return r


def per_config_entry(w: DecodeWorkload, t: dict, peaks: dict, ceiling) -> dict:
    ms = t["mean_ms"]
    nb = w.nbytes
    e = {"decode_ms": round(ms, 5), "seq_per_s": round(w.B / (ms * 1e-3), 1),
         "tokens_per_s": round(w.B / (ms * 1e-3), 1),
         "kv_tokens_per_s": round(nb["kv_tokens"] / (ms * 1e-3), 1),
         "kv_gbs_unique": round(nb["kv_unique"] / (ms * 1e-3) / 1e9, 1),
         "kv_gbs_logical": round(nb["kv"] / (ms * 1e-3) / 1e9, 1),
         "method": w.method(), "roofline": roofline_entry(w, t, peaks, ceiling)}
    if nb["kv_unique"] != nb["kv"]:
        e["bytes_unique"], e["bytes_logical"] = nb["decode_unique"], nb["decode"]
    return e


def _packed(tensors: dict, make) -> tuple:
    """One byte buffer from make(nbytes) holding every tensor of `tensors` at a
    256-byte aligned offset, and views of it with the tensors' shapes."""
    offs, n = {}, 0
    for k, v in tensors.items():
        offs[k] = n
        n += -(-(v.numel() * v.element_size()) // 256) * 256
    buf = make(n)
    views = {k: buf[o:o + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
             for (k, v), o in zip(tensors.items(), offs.values())}
    return buf, views


E2E_SETS = 3


def e2e_pipelined(w: DecodeWorkload, steps: int, warmup: int, dev) -> dict:
    """The step end to end through the public calls, with host buffers: every
    step copies its inputs from pinned host memory and its output back.  The
    inputs sit packed in one pinned buffer, so a step's upload is one copy;
    three sets of device buffers and two copy streams let step i+1's inputs
    travel while step i computes and step i-1's output returns, and the
    caller reads step i-2's output after enqueuing step i."""
    src = {k: v.cpu() for k, v in w.step_inputs().items()}
    hbuf, hview = _packed(src, lambda n: torch.empty(n, dtype=torch.uint8).pin_memory())
    for k, v in src.items():
        hview[k].copy_(v)
    sets = [_packed(src, lambda n: torch.empty(n, dtype=torch.uint8, device=dev)) for _ in range(E2E_SETS)]
    host_out = [torch.empty(w.out.shape, dtype=w.out.dtype).pin_memory() for _ in range(E2E_SETS)]
    outs = [torch.empty_like(w.out) for _ in range(E2E_SETS)]
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d_done = [torch.cuda.Event() for _ in range(E2E_SETS)]
    comp_done = [torch.cuda.Event() for _ in range(E2E_SETS)]
    d2h_done = [torch.cuda.Event() for _ in range(E2E_SETS)]
    h2d = sum(v.numel() * v.element_size() for v in src.values())
    d2h = host_out[0].numel() * host_out[0].element_size()

    def run(n):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(up)
        checksum = 0.0
        for i in range(n):
            s = i % E2E_SETS
            dbuf, dview = sets[s]
            with torch.cuda.stream(up):
                if i >= E2E_SETS:
                    up.wait_event(comp_done[s])          # step i-3 has read buffer set s
                dbuf.copy_(hbuf, non_blocking=True)
                h2d_done[s].record(up)
            comp.wait_event(h2d_done[s])
            if i >= E2E_SETS:
                comp.wait_event(d2h_done[s])             # step i-3's output has left outs[s]
            w.write(dview)
            w.decode(dview, out=outs[s])
            comp_done[s].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[s])
                host_out[s].copy_(outs[s], non_blocking=True)
                d2h_done[s].record(down)
            if i >= 2:                                   # the caller reads step i-2's result
                r = (i - 2) % E2E_SETS
                d2h_done[r].synchronize()
                checksum += float(host_out[r][0, 0, 0])
        down.wait_stream(comp)
        end.record(down)
        end.synchronize()
        for i in range(max(0, n - 2), n):
            checksum += float(host_out[i % E2E_SETS][0, 0, 0])
        return start.elapsed_time(end) / n

    run(max(3, warmup))
    ms = run(steps)
    return {"ms": ms, "h2d": h2d, "d2h": d2h,
            "mode": f"pipelined: inputs packed in one pinned buffer (one upload per step), "
                    f"{E2E_SETS} device buffer sets, uploads and downloads on two copy streams "
                    f"overlapping the neighbouring steps' kernels; the caller reads step i-2's "
                    f"output after enqueuing step i"}


def e2e_serial(w: DecodeWorkload, steps: int, warmup: int, dev, flush_buf) -> dict:
    """As e2e_pipelined, one step at a time (each synchronised), for workloads
    that fit in L2: an L2 flush between steps, outside the events."""
    host_in = {k: v.cpu().pin_memory() for k, v in w.step_inputs().items()}
    host_out = torch.empty(w.out.shape, dtype=w.out.dtype).pin_memory()
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in host_in.items()}
    stream = torch.cuda.current_stream(dev)

    def one():
        for k, v in host_in.items():
            dev_in[k].copy_(v, non_blocking=True)
        w.write(dev_in)
        w.decode(dev_in)
        host_out.copy_(w.out, non_blocking=True)
        stream.synchronize()                            # the caller reads the result

    for _ in range(max(3, warmup)):
        one()
    each = time_each(one, steps, stream, flush_buf)
    return {"ms": statistics.mean(each), "h2d": sum(t.numel() * t.element_size() for t in host_in.values()),
            "d2h": host_out.numel() * host_out.element_size(),
            "mode": "serial: one step at a time, L2 flushed between steps"}


def run_gpu(args, cfg, world, rank, local):
    import paged_kv_cache_468_b200 as pkv

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    w = DecodeWorkload(pkv, cfg, dev, replica_seed(cfg.seed, rank), args.partition_tokens,
                       args.cascade)
    nbytes = w.nbytes
    l2_dev = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or 0)
    flush_buf = torch.empty(2 * max(l2_dev, L2_BYTES_B200), dtype=torch.uint8, device=dev)

    pkv.device_flags(clear=True)
    for _ in range(args.warmup):
        w.one_step()
    torch.cuda.synchronize()

    # optional: the step as a CUDA graph (same kernels, no per-launch host work)
    step_fn = w.one_step
    graph_note = "off"
    if args.graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                w.one_step()
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            step_fn = graph.replay
            graph_note = "on"
        except Exception as exc:   # capture unsupported here: plain launches
            graph_note = f"capture failed ({type(exc).__name__}); plain launches"
            torch.cuda.synchronize()

    # ---- the contract's timed region: K whole steps, inputs resident in HBM ----
    K = args.steps
    sampler = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark(True)
    if w.flush:
        ms_step_local = statistics.mean(time_each(step_fn, K, stream, flush_buf))
    else:
        ms_step_local = time_back_to_back(step_fn, K, stream)
    if sampler:
        sampler.mark(False)
    barrier(world)

    # ---- the decode call alone, for the roofline: at least --roofline-launches
    # launches and --roofline-seconds of device time, whatever --steps is ----
    n_roof = max(args.roofline_launches,
                 int(math.ceil(args.roofline_seconds * 1e3 / max(ms_step_local, 1e-4))))
    n_roof = min(n_roof, 50000)
    t_main = measure_decode_launches(w, n_roof, stream, flush_buf, sampler)
    flags = pkv.device_flags(clear=True)

    # ---- end to end through the public API, host buffers ----
    e2e = None
    if not args.no_e2e:
        Ke = max(1, min(K, args.e2e_steps)) if w.flush else max(K, args.e2e_steps)
        barrier(world)
        r = e2e_serial(w, Ke, args.warmup, dev, flush_buf) if w.flush else \
            e2e_pipelined(w, Ke, args.warmup, dev)
        barrier(world)
        e2e_ms = max_over_ranks(r["ms"], world)
        e2e_gbs = sum_over_ranks(nbytes["decode_unique"] + nbytes["write"], world) / (e2e_ms * 1e-3) / 1e9
        e2e = {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": r["h2d"],
               "d2h_bytes_per_step": r["d2h"], "ms_per_step": round(e2e_ms, 4), "steps": Ke,
               "tokens_per_s": round(sum_over_ranks(w.B, world) / (e2e_ms * 1e-3), 1),
               "mode": r["mode"]}

    # unique bytes: a block shared by several sequences' tables counts once
    value, ms_step = job_throughput(nbytes["decode_unique"] + nbytes["write"], ms_step_local, world)
    # every collective before any rank-0-only code: all ranks take the same steps
    tokens = sum_over_ranks(w.B, world)
    kv_tokens_all = sum_over_ranks(nbytes["kv_tokens"], world)
    kv_all = sum_over_ranks(nbytes["kv"], world)

    peaks = measured_peaks()
    ceiling = None
    per_config = None
    if rank == 0 and world == 1:
        if not args.no_read_ceiling:
            ceiling = read_ceiling(pkv, dev, stream, same_bytes=nbytes["decode_unique"])
        if not args.no_per_config:
            per_config = {}
            for name in workloads.CONFIGS:
                if name == cfg.name:
                    per_config[name] = per_config_entry(w, t_main, peaks, ceiling)
                    continue
                other = DecodeWorkload(pkv, workloads.CONFIGS[name], dev, replica_seed(
                    workloads.CONFIGS[name].seed, rank), None, args.cascade)
                for _ in range(3):
                    other.one_step()
                est = time_back_to_back(other.decode, 5, stream)
                n = min(20000, max(args.per_config_launches,
                                   int(math.ceil(args.per_config_seconds * 1e3 / max(est, 1e-4)))))
                t = measure_decode_launches(other, n, stream, flush_buf, sampler)
                per_config[name] = per_config_entry(other, t, peaks, ceiling)
                del other
                torch.cuda.empty_cache()
            flags |= pkv.device_flags(clear=True)
    clocks = sampler.stop() if sampler else None
    roofline = roofline_entry(w, t_main, peaks, ceiling)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nthreads = os.cpu_count() or 1
        nseq = choose_oracle_seqs(w.step, cfg, nthreads, args.cpu_seconds / 3)
        gbs, n, reps, el = oracle_sample_rate(w.step, cfg, args.cpu_seconds, nthreads, max_seqs=nseq)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
               "sample": f"first {n} of {w.B} sequences (write + decode), {reps} repetitions "
                         f"in {el:.1f} s, fp64"}

    if rank == 0:
        method = dict(w.method(), cuda_graph=graph_note,
                      step_timing=("an event pair around each step, L2 flushed between steps"
                                   if w.flush else "one event pair around the K steps"))
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": workload_config(cfg, w.step, nbytes, world),
            "method": method,
            "tokens_per_s": round(tokens / (ms_step * 1e-3), 1),
            "kv_tokens_per_s": round(kv_tokens_all / (ms_step * 1e-3), 1),
            "frac_of_hbm_peak": round(value / peaks["hbm_gbs"], 4),
            "logical_kv_gbs": round(kv_all / (ms_step * 1e-3) / 1e9, 1),
            "gpu_launches": w.launches_per_step * K,
            "launches_per_step": w.launches_per_step,
            "device_flags": flags,
            "roofline": roofline,
            "read_ceiling": ceiling,
            "per_config": per_config,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    return 0


def _time_loop(fn, steps, warmup, stream):
    """Mean ms per call of fn over `steps` calls (CUDA events on `stream`)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_other_op(args, cfg, world, rank, local):
    """The NEXT-row operations, one GPU: chunked prefill (tensor roofline),
    copy-on-write block copies (HBM roofline) and swap-out to pinned host."""
    import paged_kv_cache_468_b200 as pkv

    dev = torch.device("cuda", local)
    step = workloads.make_decode_step(cfg)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in step.items()}
    B, Hq, D = d["query"].shape
    NB, bs, Hkv, _ = d["key_cache"].shape
    stream = torch.cuda.current_stream(dev)
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    line = {"impl": "pagedkv", "op": args.op, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "description": cfg.description}}
    if args.op == "prefill":
        lens = [int(x) for x in step["context_lens"]]
        chunks = [min(args.chunk, L) for L in lens]
        g = torch.Generator().manual_seed(cfg.seed + 7)
        T = sum(chunks)
        q = torch.randn(T, Hq, D, generator=g).to(step["query"].dtype).to(dev)
        qs = torch.tensor([0] + list(np.cumsum(chunks)), dtype=torch.int32, device=dev)
        out = torch.empty_like(q)
        fn = lambda: pkv.paged_attention_prefill(q, qs, max(chunks), d["key_cache"], d["value_cache"],
                                                 d["block_tables"], d["context_lens"], d["scale"],
                                                 out=out)
        ms = _time_loop(fn, args.steps, args.warmup, stream)
        # causal attention FLOPs: QK and PV, 2 flops per MAC, over keys 0..p
        keys = sum(sum(L - C + i + 1 for i in range(C)) for L, C in zip(lens, chunks))
        flops = 4.0 * D * Hq * keys
        peak = float(peaks.get("bf16_tflops", 1590.0))
        line.update(metric="chunked prefill attention TFLOP/s", unit="TFLOP/s",
                    value=round(flops / (ms * 1e-3) / 1e12, 2), ms_per_step=round(ms, 4),
                    higher_is_better=True, tokens_per_s=round(T / (ms * 1e-3), 1),
                    roofline={"bound": "tensor", "achieved": round(flops / (ms * 1e-3) / 1e12, 2),
                              "peak": peak, "unit": "TFLOP/s",
                              "frac": round(flops / (ms * 1e-3) / 1e12 / peak, 4),
                              "peak_source": "MEASURED_PEAKS.json bf16_tflops (cuBLAS bf16)",
                              "note": "tcgen05.mma (TMEM accumulators), 128 query rows x 64-key tiles"})
        line["config"].update(chunk=args.chunk, query_tokens=T)
    else:
        n = min(args.pairs, NB // 2)
        g = torch.Generator().manual_seed(cfg.seed + 11)
        perm = torch.randperm(NB, generator=g)
        mapping = torch.stack([perm[:n], perm[n:2 * n]], 1).to(torch.int32).to(dev)
        block_bytes = bs * Hkv * D * 2
        if args.op == "copy":
            fn = lambda: pkv.copy_blocks(d["key_cache"], d["value_cache"], d["key_cache"],
                                         d["value_cache"], mapping)
            moved = 2 * 2 * n * block_bytes                    # K and V, read + write
            peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
            bound = "hbm"
        else:
            hk = torch.empty((n,) + tuple(d["key_cache"].shape[1:]), dtype=d["key_cache"].dtype).pin_memory()
            hv = torch.empty_like(hk).pin_memory()
            out_map = torch.stack([perm[:n], torch.arange(n)], 1).to(torch.int32).to(dev)
            fn = lambda: pkv.copy_blocks(d["key_cache"], d["value_cache"], hk, hv, out_map)
            moved = 2 * n * block_bytes                        # bytes that cross to the host
            peak = None
            bound = "host link"
        ms = _time_loop(fn, args.steps, args.warmup, stream)
        gbs = moved / (ms * 1e-3) / 1e9
        line.update(metric=f"block {args.op} GB/s", unit="GB/s", value=round(gbs, 2),
                    ms_per_step=round(ms, 4), higher_is_better=True,
                    roofline={"bound": bound, "achieved": round(gbs, 2), "peak": peak,
                              "unit": "GB/s", "frac": round(gbs / peak, 4) if peak else None})
        line["config"].update(pairs=n, block_bytes=block_bytes)
    line["device_flags"] = pkv.device_flags(clear=True)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def dataclass_replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default=workloads.HEADLINE, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--impl", default="pagedkv", choices=["pagedkv", "reference"])
    ap.add_argument("--op", default="decode", choices=["decode", "prefill", "copy", "swap"],
                    help="decode step (the contract line) or a NEXT-row operation")
    ap.add_argument("--chunk", type=int, default=512, help="prefill chunk tokens per sequence")
    ap.add_argument("--pairs", type=int, default=2048, help="block pairs for --op copy/swap")
    ap.add_argument("--partition-tokens", type=int, default=None,
                    help="override the workload's partition request (0 auto, <0 never)")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--roofline-launches", type=int, default=2000,
                    help="decode launches timed for the roofline (at least)")
    ap.add_argument("--roofline-seconds", type=float, default=0.6,
                    help="device time the roofline leg covers (at least)")
    ap.add_argument("--per-config-launches", type=int, default=1000)
    ap.add_argument("--per-config-seconds", type=float, default=0.3)
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the roofline of the other workloads")
    ap.add_argument("--no-read-ceiling", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    ap.add_argument("--cascade", default="auto", choices=["auto", "on", "off"],
                    help="shared-prefix decode (auto: for workloads with a shared prefix)")
    ap.add_argument("--graph", action="store_true",
                    help="replay the step as a CUDA graph in the timed loop")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = workloads.CONFIGS[args.config]

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, cfg, world, rank)

    world, rank, local = dist_setup()
    if world != args.gpus and rank == 0:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE {world}; using {world}", file=sys.stderr)
    try:
        if args.op != "decode":
            return run_other_op(args, cfg, world, rank, local)
        return run_gpu(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
