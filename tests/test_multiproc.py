"""The multi-rank host logic on CPU: two gloo ranks (no GPU).

bench.py runs N independent replicas of the step (weak scaling, no data-path collective):
each rank times its own step, the job's time is the slowest rank's (an all-reduce MAX) and
its rate is all ranks' work over that time. The row / layer sharding helpers used to split a
quantize pass across ranks must hand every unit to exactly one rank.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # replica timing: rank r measured 1.5 + r ms; every rank must see the slowest
        ms = bench.max_over_ranks(1.5 + rank, world, "cpu")
        value = bench.whole_job_tflops(world, 90.6e9, ms)
        # sharding: every row / layer exactly once over the ranks
        rows = workloads.shard_rows(11520, rank, world)
        layers = workloads.shard_layers(210, rank, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, (rows, layers))
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr((ms, value, gathered)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replicas_max_over_ranks_and_sharding(tmp_path, world):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    results = [eval(open(tmp_path / f"rank{r}.txt").read()) for r in range(world)]
    for ms, value, gathered in results:
        assert ms == 1.5 + (world - 1)                              # the slowest rank's time
        assert abs(value - world * 90.6e9 / (ms * 1e-3) / 1e12) < 1e-9
        # rows: contiguous, disjoint, covering [0, 11520)
        spans = sorted(g[0] for g in gathered)
        assert spans[0][0] == 0 and spans[-1][1] == 11520
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        # layers: each of the 210 exactly once
        layers = sorted(l for g in gathered for l in g[1])
        assert layers == list(range(210))
    assert results[0] == results[1]


def test_single_rank_is_local():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert abs(bench.whole_job_tflops(1, 2e12, 1.0) - 2000.0) < 1e-9
