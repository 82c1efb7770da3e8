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
    ("pkv_prefill.cuh", ["PrefillArgs", "PfShape", "PfBar", "tc_attend", "prefix_tc_kernel"]),
    ("pagedkv.cu", ["make_query_map", "cascade_plan", "launch_prefix", "dispatch_prefix",
                    "pkv_paged_attention_decode_cascade"]),
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
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t_on = None
        self.t_off = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
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
            self.t_on = time.time()
        else:
            self.t_off = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t, line in self.lines:
            if self.t_on is not None and self.t_off is not None and not (self.t_on <= t <= self.t_off + 0.06):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            rows.append(parts)
        if not rows:   # timed region shorter than the sampling period: take the nearest
            rows = [[p.strip() for p in l.split(",")] for _, l in self.lines[-3:]]
            rows = [r for r in rows if len(r) == len(self.FIELDS)]
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


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


def run_reference(args, cfg, world, rank):
    """The oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return 0
    nthreads = os.cpu_count() or 1
    step = workloads.make_decode_step(cfg)
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
        "config": {"workload": cfg.name, "description": cfg.description},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- GPU arm ----

def run_gpu(args, cfg, world, rank, local):
    import paged_kv_cache_468_b200 as pkv

    dev = torch.device("cuda", local)
    step = workloads.make_decode_step(dataclass_replace(cfg, seed=replica_seed(cfg.seed, rank)))
    nbytes = step_bytes(step, cfg)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in step.items()}
    B, Hq, D = d["query"].shape
    NB, bs, Hkv, _ = d["key_cache"].shape
    MB = d["block_tables"].shape[1]
    pt_req = cfg.partition_tokens if args.partition_tokens is None else args.partition_tokens
    plan_pt, plan_np = pkv.decode_plan(B, Hq, Hkv, D, MB, bs, pt_req)
    ws_bytes = pkv.decode_workspace_bytes(B, Hq, Hkv, D, MB, bs, pt_req)
    out = torch.empty_like(d["query"])
    launches_per_step = 2 + (1 if plan_np > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    cascade = args.cascade == "on" or (args.cascade == "auto" and cfg.shared_prefix > 0)
    if cascade:
        cas = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in
               workloads.cascade_inputs(step, cfg.shared_prefix, cfg.samples).items()}
        ws_bytes = int(pkv.lib().pkv_decode_cascade_workspace_bytes(
            B, Hq, Hkv, D, cas["prefix_tables"].shape[1], cas["suffix_tables"].shape[1],
            cas["max_group_size"], bs, pt_req))
        launches_per_step = 4
    ws = torch.empty(max(16, ws_bytes), dtype=torch.uint8, device=dev)

    def decode_call(query, tables, lens):
        if cascade:
            return pkv.paged_attention_decode_cascade(
                query, d["key_cache"], d["value_cache"], cas["prefix_tables"], cas["prefix_lens"],
                cas["group_start"], cas["suffix_tables"], cas["suffix_lens"], d["scale"],
                max_group_size=cas["max_group_size"], partition_tokens=pt_req, out=out,
                workspace=ws)
        return pkv.paged_attention_decode(query, d["key_cache"], d["value_cache"], tables, lens,
                                          d["scale"], partition_tokens=pt_req, out=out,
                                          workspace=ws)

    def one_step():
        pkv.kv_cache_write(d["new_key"], d["new_value"], d["slot_mapping"], d["key_cache"],
                           d["value_cache"])
        decode_call(d["query"], d["block_tables"], d["context_lens"])

    pkv.device_flags(clear=True)
    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()

    # optional: the step as a CUDA graph (same kernels, no per-launch host work)
    step_fn = one_step
    graph_note = "off"
    if args.graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                one_step()
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            step_fn = graph.replay
            graph_note = "on"
        except Exception as exc:   # capture unsupported here: plain launches
            graph_note = f"capture failed ({type(exc).__name__}); plain launches"
            torch.cuda.synchronize()

    # ---- L2: inputs that fit in L2 would be read warm from the second
    # iteration on; for those, every timed iteration gets its own events and a
    # write of twice the L2 size in between (outside the events) ----
    l2_bytes = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20))
    flush_l2 = nbytes["kv_unique"] <= l2_bytes
    flush_buf = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev) if flush_l2 else None

    def timed_iterations(fn, n):
        """ms per iteration of fn over n iterations: one event pair around all
        of them, or (inputs fitting in L2) per iteration with an L2 flush
        between iterations; also the per-iteration times when taken."""
        if not flush_l2:
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                fn()
            b_.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b_) / n, None
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for i in range(n):
            flush_buf.fill_(i & 0xff)
            evs[i][0].record(stream)
            fn()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        per = [x.elapsed_time(y) for x, y in evs]
        return sum(per) / n, per

    # ---- device-timed region (inputs resident in HBM): K whole steps ----
    K = args.steps
    sampler = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark(True)
    ms_step_mean, _ = timed_iterations(step_fn, K)
    if sampler:
        sampler.mark(False)
    barrier(world)
    ms_total = ms_step_mean * K
    clocks = sampler.stop() if sampler else None

    # ---- the decode call alone (its kernels), for the roofline: CUDA events
    # around each launch on the launching stream ----
    Kd = max(1, min(K, args.roofline_launches))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(Kd)]
    torch.cuda.synchronize()
    for i in range(Kd):
        if flush_l2:
            flush_buf.fill_(i & 0xff)
        ev[i][0].record(stream)
        decode_call(d["query"], d["block_tables"], d["context_lens"])
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    decode_times = [a.elapsed_time(b) for a, b in ev]
    decode_ms = statistics.mean(decode_times)      # decode (+ merge) per call
    decode_ms_median = statistics.median(decode_times)
    flags = pkv.device_flags(clear=True)

    # ---- end to end through the public API, host buffers ----
    e2e = None
    if not args.no_e2e:
        host_in = {k: d[k].cpu().pin_memory() for k in
                   ("query", "new_key", "new_value", "slot_mapping", "block_tables", "context_lens")}
        host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = host_out.numel() * host_out.element_size()
        dev_in = {k: torch.empty_like(v, device=dev) for k, v in host_in.items()}

        def e2e_step():
            for k, v in host_in.items():
                dev_in[k].copy_(v, non_blocking=True)
            pkv.kv_cache_write(dev_in["new_key"], dev_in["new_value"], dev_in["slot_mapping"],
                               d["key_cache"], d["value_cache"])
            decode_call(dev_in["query"], dev_in["block_tables"], dev_in["context_lens"])
            host_out.copy_(out, non_blocking=True)
            stream.synchronize()                       # the caller reads the result

        for _ in range(max(3, args.warmup)):
            e2e_step()
        Ke = max(1, min(K, args.e2e_steps))
        barrier(world)
        torch.cuda.synchronize()
        e2e_local, _ = timed_iterations(e2e_step, Ke)
        barrier(world)
        e2e_ms = max_over_ranks(e2e_local, world)
        e2e_gbs = sum_over_ranks(nbytes["decode_unique"] + nbytes["write"], world) / (e2e_ms * 1e-3) / 1e9
        e2e = {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4), "steps": Ke,
               "tokens_per_s": round(sum_over_ranks(B, world) / (e2e_ms * 1e-3), 1)}

    # unique bytes: a block shared by several sequences' tables counts once
    value, ms_step = job_throughput(nbytes["decode_unique"] + nbytes["write"], ms_total / K, world)
    # every collective before any rank-0-only code: all ranks take the same steps
    tokens = sum_over_ranks(B, world)
    kv_tokens_all = sum_over_ranks(nbytes["kv_tokens"], world)
    kv_all = sum_over_ranks(nbytes["kv"], world)

    peaks = measured_peaks()
    achieved = nbytes["decode_unique"] / (decode_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": committed_traffic(cfg.name, plan_np > 1 and not cascade, cascade),
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)"
                if peaks["source"] == "measured" else "fallback 6650 GB/s",
                "kernel": ("prefix_tc_kernel + paged_decode_kernel (suffixes) + "
                           "lse_merge_cascade_kernel" if cascade else
                           "paged_decode_kernel" + (" + lse_merge_kernel" if plan_np > 1 else "")),
                "bytes_per_launch": nbytes["decode_unique"], "launch_ms": round(decode_ms, 5),
                "launch_ms_median": round(decode_ms_median, 5),
                "frac_of_8000": round(achieved / 8000.0, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nthreads = os.cpu_count() or 1
        nseq = choose_oracle_seqs(step, cfg, nthreads, args.cpu_seconds / 3)
        gbs, n, reps, el = oracle_sample_rate(step, cfg, args.cpu_seconds, nthreads, max_seqs=nseq)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
               "sample": f"first {n} of {B} sequences (write + decode), {reps} repetitions "
                         f"in {el:.1f} s, fp64"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "description": cfg.description, "batch": B,
                       "num_heads": Hq, "num_kv_heads": Hkv, "head_dim": D, "block_size": bs,
                       "num_blocks": NB, "max_blocks": MB,
                       "context_tokens": nbytes["kv_tokens"],
                       "partition_tokens": plan_pt, "num_partitions": plan_np,
                       "cascade": cascade, "cuda_graph": graph_note,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": (f"inputs fit in L2 ({nbytes['kv_unique'] / 1e6:.1f} MB of K/V vs "
                              f"{l2_bytes / 1e6:.0f} MB): each timed iteration has its own CUDA "
                              f"events and a {2 * l2_bytes / 1e6:.0f} MB buffer is written between "
                              f"iterations, outside the events")
                       if flush_l2 else
                       (f"inputs larger than L2: {nbytes['kv_unique'] / 1e6:.0f} MB of K/V "
                        f"per step vs {l2_bytes / 1e6:.0f} MB L2, no flush")},
            "tokens_per_s": round(tokens / (ms_step * 1e-3), 1),
            "kv_tokens_per_s": round(kv_tokens_all / (ms_step * 1e-3), 1),
            "frac_of_hbm_peak": round(value / peaks["hbm_gbs"], 4),
            "logical_kv_gbs": round(kv_all / (ms_step * 1e-3) / 1e9, 1),
            "gpu_launches": launches_per_step * K,
            "launches_per_step": launches_per_step,
            "device_flags": flags,
            "roofline": roofline,
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
    ap.add_argument("--roofline-launches", type=int, default=500)
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
