"""The multi-GPU path on CPU: world_size-2 gloo ranks run bench.py's replica
and aggregation logic (each rank its own replica; job time = max over ranks;
work = sum over ranks).  No data-path collective exists to test: the path
shards by sequence."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from paged_kv_cache_468_b200 import workloads
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # rank r: 100 * (r + 1) bytes in (r + 1) ms -> job: 300 bytes in 2 ms
        gbs, ms = bench.job_throughput(100.0 * (rank + 1), float(rank + 1), world, device="cpu")
        cfg = workloads.CONFIGS["tiny_mha"]
        step = workloads.make_decode_step(
            bench.dataclass_replace(cfg, seed=bench.replica_seed(cfg.seed, rank)))
        digest = float(step["query"].float().sum())
        dist.barrier()
        q.put((rank, gbs, ms, digest, bench.max_over_ranks(float(rank), world, "cpu"),
               bench.sum_over_ranks(1.0, world, "cpu")))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_aggregation():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, gbs, ms, _, mx, sm in res:
        assert ms == 2.0                       # slowest rank
        assert gbs == pytest.approx(300.0 / 2e-3 / 1e9)
        assert mx == 1.0 and sm == 2.0
    assert res[0][3] != res[1][3]              # each rank drew its own replica


def test_single_rank_is_identity():
    import bench
    gbs, ms = bench.job_throughput(1e9, 1.0, 1)
    assert ms == 1.0 and gbs == pytest.approx(1000.0)
