"""Column-parallel OPQ linear on one GPU: in a one-rank NCCL group the shard is the whole
weight and the all-gather a copy, so the result must equal the library's linear bit for bit.
The exchange across ranks (uneven shards, reassembly along N) is covered by the two-rank gloo
test in test_multiproc.py; this run has one GPU."""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import bit_diffusion_transformer_b200 as opq
import workloads
from bit_diffusion_transformer_b200 import sharded
from test_gpu_parity import DEV, no_device_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("M,N,K", [(300, 1000, 1024), (5, 37, 64)])
def test_column_parallel_one_rank_equals_linear(one_rank_group, M, N, K):
    lin = workloads.Linear("column-1", M, N, K, w_seed=N, x_seed=M)
    x, w = lin.make(DEV)
    shard = sharded.quantize_shard(w, 0, 1, lin.alpha)
    planes = opq.quantize(w, lin.alpha)
    for a, b in zip((shard.codes, shard.signs, shard.scales), planes):
        assert torch.equal(a, b)
    assert (shard.lo, shard.hi, shard.n_rows) == (0, N, N)
    y = sharded.column_parallel_linear(x, shard)
    ref = opq.linear(x, *planes, lin.alpha)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    no_device_error()
