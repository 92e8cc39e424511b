"""A bounded device wait that runs out, made on the host, and the recovery after it.

The wide linear runs the tiles past its last whole wave as two half-K runs on two CTAs.
Per TMEM lane quarter the first of the pair to finish bumps an arrival counter in the
caller's workspace, publishes its fp32 partial sums and raises a flag; the second waits
(bounded) for the flag. Planting an arrival count of 1 before the call makes both CTAs of
one quarter believe that they are second, so both wait for a flag that nobody raises. No
kernel is changed and nothing faults: the waits end at the (shortened) limit, the kernel
records OPQ_DEVERR_WAIT_TIMEOUT, leaves that quarter of y unwritten, puts the counters back
to zero and returns. A clean call afterwards, and the allocation-free linear, are
bit-identical to a fresh run.
"""
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
COUNTER_BYTES = 64 * 1024   # the workspace's leading arrival-counter region


def _tail_geometry(M, N, grid):
    """First tail tile of the whole-tile schedule and its y block (rows of x, rows of W)."""
    m_tiles, n_tiles = -(-M // 256), -(-N // 128)
    tiles = m_tiles * n_tiles
    full_end = (tiles // grid) * grid
    tile = full_end                     # tail tile 0
    n_blk, m_blk = tile // m_tiles, tile % m_tiles
    return tiles - full_end, (m_blk * 256, min(M, m_blk * 256 + 256)), (n_blk * 128, n_blk * 128 + 32)


def test_tail_flag_wait_times_out_and_recovers():
    lin = workloads.dit_attn_proj()
    x, w = lin.make(DEV)
    M, N, K, alpha = lin.M, lin.N, lin.K, lin.alpha
    planes = opq.quantize(w, alpha)
    path, grid, _ = opq.plan(M, N, K)
    assert path == 0
    n_tail, (m0, m1), (n0, n1) = _tail_geometry(M, N, grid)
    assert 0 < 2 * n_tail <= grid      # the half-K tail split is in use for this shape
    ws = torch.zeros((opq.workspace_size(M, N, K),), dtype=torch.uint8, device=DEV)
    counters = ws[:COUNTER_BYTES].view(torch.int32)
    y_ref = opq.linear(x, *planes, alpha, workspace=ws)
    assert opq.device_error() == 0

    # plant: tail tile 0, lane quarter 0 already counts one arrival, nothing published
    ws.zero_()
    counters[0] = 1
    y = torch.zeros_like(y_ref)
    opq.set_wait_limit_ns(50_000_000)   # 50 ms: far above any wait of a healthy call (~80 us)
    try:
        opq.linear(x, *planes, alpha, out=y, workspace=ws)
        err = opq.device_error()
    finally:
        opq.set_wait_limit_ns(0)
    assert err == opq.DEVERR_WAIT_TIMEOUT
    # the two waiting CTAs put the counters back to zero before returning
    assert int(counters.abs().sum()) == 0
    # that quarter of the tail tile was not written; everything else is the fresh result
    blk = (slice(m0, m1), slice(n0, n1))
    assert int(y[blk].abs().float().sum()) == 0
    mask = torch.ones_like(y_ref, dtype=torch.bool)
    mask[blk] = False
    assert torch.equal(y[mask], y_ref[mask])

    # recovery: a clean call on a zeroed workspace, and the allocation-free linear (whose static
    # counters device_error clears after a time-out), both equal the fresh run bit for bit
    ws.zero_()
    y2 = opq.linear(x, *planes, alpha, workspace=ws)
    assert opq.device_error() == 0
    assert torch.equal(y2, y_ref)
    y3 = opq.linear_noalloc(x, *planes, alpha)
    assert opq.device_error() == 0
    assert torch.equal(y3, y_ref)


def test_wait_limit_default_restored():
    """After the limit is restored, an ordinary call reports no error."""
    lin = workloads.small_m(16)
    x, w = lin.make(DEV)
    planes = opq.quantize(w, lin.alpha)
    ws = torch.zeros((max(opq.workspace_size(lin.M, lin.N, lin.K), 16),), dtype=torch.uint8, device=DEV)
    opq.set_wait_limit_ns(0)
    opq.linear(x, *planes, lin.alpha, workspace=ws)
    assert opq.device_error() == 0
