"""The multi-rank host logic on CPU: two gloo ranks (no GPU).

bench.py runs N independent replicas of the step (weak scaling, no data-path collective):
each rank times its own step, the job's time is the slowest rank's (an all-reduce MAX) and
its rate is all ranks' work over that time. The row / layer sharding helpers used to split a
quantize pass across ranks must hand every unit to exactly one rank. The column-parallel
linear (each rank its rows of W, one all-gather of y along N) runs here with the oracle as
the local quantize and product, so the exchange and reassembly are checked without a GPU.
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
    from bit_diffusion_transformer_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # replica timing: rank r measured 1.5 + r ms; every rank must see the slowest
        ms = bench.max_over_ranks(1.5 + rank, world, "cpu")
        value = bench.whole_job_tflops(world, 90.6e9, ms)
        # sharding: every row / layer exactly once over the ranks
        rows = sharded.shard_range(11520, rank, world)
        layers = sharded.shard_layers(210, rank, world)
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


# ------------------------------------------------------------ column-parallel linear --
def _oracle_quantize(w, alpha):
    import numpy as np
    import oracle
    ref = oracle.quantize(w, alpha)
    return (torch.from_numpy(ref["codes"].view(np.int32).copy()), torch.from_numpy(ref["signs"].view(np.int32).copy()),
            torch.from_numpy(ref["scales"].copy()))


def _oracle_linear(x, codes, signs, scales, alpha):
    import numpy as np
    import oracle
    y, _ = oracle.linear(x, codes.numpy().view(np.uint32), signs.numpy().view(np.uint32), scales.numpy(), alpha)
    return torch.from_numpy(y).to(torch.bfloat16)


def _column_main(rank, world, port, out_dir, shapes):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import workloads
    from bit_diffusion_transformer_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = []
        for M, N, K in shapes:
            lin = workloads.Linear("column-parallel", M, N, K, w_seed=N + K, x_seed=M + K)
            x, w = lin.make("cpu")
            shard = sharded.quantize_shard(w, rank, world, lin.alpha, quantize_fn=_oracle_quantize)
            y = sharded.column_parallel_linear(x, shard, linear_fn=_oracle_linear)
            full = _oracle_linear(x, *_oracle_quantize(w, lin.alpha), lin.alpha)
            res.append((shard.lo, shard.hi, bool(torch.equal(y.view(torch.int16), full.view(torch.int16)))))
        # rows [1, 3) of 4 are no rank's shard: every rank refuses it before any collective
        wrong = sharded.ColumnShard(*_oracle_quantize(torch.zeros((2, 32), dtype=torch.bfloat16), 0.73),
                                    lo=1, hi=3, n_rows=4, alpha=0.73)
        try:
            sharded.column_parallel_linear(torch.zeros((1, 32), dtype=torch.bfloat16), wrong,
                                           linear_fn=_oracle_linear)
            refused = False
        except ValueError:
            refused = True
        res.append(refused)
        dist.barrier()
        with open(os.path.join(out_dir, f"col{rank}.txt"), "w") as f:
            f.write(repr(res))
    finally:
        dist.destroy_process_group()


def test_column_parallel_linear_two_ranks(tmp_path):
    # N = 37: shards of 19 and 18 rows (padded block on rank 1); N = 2: one row each
    shapes = [(5, 37, 64), (3, 2, 96), (17, 256, 512)]
    world = 2
    port = _free_port()
    mp.start_processes(_column_main, args=(world, port, str(tmp_path), shapes), nprocs=world, start_method="spawn")
    res = [eval(open(tmp_path / f"col{r}.txt").read()) for r in range(world)]
    assert [r[:2] for r in res[0][:3]] == [(0, 19), (0, 1), (0, 128)]
    assert [r[:2] for r in res[1][:3]] == [(19, 37), (1, 2), (128, 256)]
    for r in res:
        assert all(ok for _, _, ok in r[:3]), "gathered y differs from the unsharded product"
        assert r[3]


def test_shard_range_covers_rows():
    import sys
    sys.path.insert(0, ROOT)
    from bit_diffusion_transformer_b200 import sharded
    for n in (1, 2, 7, 37, 11520):
        for world in (1, 2, 3, 8):
            spans = [sharded.shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1 and max(sizes) == sharded.shard_width(n, world)
    with pytest.raises(ValueError):
        sharded.shard_range(8, 2, 2)
    # more ranks than rows: the rank without a row is refused before it quantizes anything
    calls = []
    with pytest.raises(ValueError):
        sharded.quantize_shard(torch.zeros((1, 32), dtype=torch.bfloat16), 1, 2, 0.73,
                               quantize_fn=lambda w, a: calls.append(w.shape))
    assert calls == []
