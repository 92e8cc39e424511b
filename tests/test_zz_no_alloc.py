"""opq_linear_noalloc: the allocation-free linear for callers that cannot call
cudaMalloc (a host runtime that owns the device memory pool, or a fixed operator
signature with no scratch argument). Its split-K partial sums live in a static
16 MiB device array inside libopq.so. Checked through the C ABI against
opq_linear, which takes a caller-allocated workspace, on two calls in a row.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test; it passes alone in a fresh process
as well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call_noalloc(lib, x, planes, alpha, y):
    codes, signs, scales = planes
    M, K = x.shape
    N = codes.shape[0]
    return lib.opq_linear_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, ctypes.c_void_p(codes.data_ptr()),
                                  ctypes.c_void_p(signs.data_ptr()), ctypes.c_void_p(scales.data_ptr()), N,
                                  float(alpha), ctypes.c_void_p(y.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K", [(16, 11520, 3840), (1, 3840, 3840), (64, 2048, 1024), (300, 640, 512)])
def test_noalloc_matches_workspace_entry_point(M, N, K):
    lib = opq.load()
    lin = workloads.Linear("noalloc", M, N, K, w_seed=17 + M, x_seed=19 + N)
    x_cpu, w_cpu = lin.make("cpu")
    ref = oracle.quantize(w_cpu, lin.alpha)
    x = x_cpu.to(DEV)
    planes = (torch.from_numpy(ref["codes"].view(np.int32)).to(DEV),
              torch.from_numpy(ref["signs"].view(np.int32)).to(DEV),
              torch.from_numpy(ref["scales"]).to(DEV))
    want = opq.linear(x, *planes, lin.alpha)           # caller-provided workspace
    # the tolerance of the parity tests, with the oracle's bound |x| |W'|^T on sampled outputs
    rng = np.random.default_rng(M + N)
    ms = rng.integers(0, M, 400)
    ns = rng.integers(0, N, 400)
    _, bound = oracle.linear_pairs(x_cpu, ref["codes"], ref["signs"], ref["scales"], lin.alpha, ms, ns)
    tol = 1e-2 * bound + 1e-3
    w_f = want.float().cpu().numpy().astype(np.float64)
    for call in range(2):                               # two calls in a row share the static scratch
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(lib, x, planes, lin.alpha, y) == 0
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), f"call {call}: unwritten outputs"
        assert (np.abs(got[ms, ns] - w_f[ms, ns]) <= tol).all(), f"call {call}"
        assert torch.equal(y, want), f"call {call}: not identical to opq_linear"
    assert opq.device_error() == 0


def test_noalloc_rejects_shapes_beyond_the_scratch():
    lib = opq.load()
    M, N, K = 128, 11520, 3840          # stream-K partials of 128-row tiles: about 19 MiB
    assert opq.workspace_size(M, N, K) > opq.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=DEV)
    planes = (torch.zeros((N, K // 8), dtype=torch.int32, device=DEV),
              torch.zeros((N, K // 32), dtype=torch.int32, device=DEV),
              torch.zeros((N,), dtype=torch.float32, device=DEV))
    y = torch.zeros((M, N), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(lib, x, planes, 0.73, y) == 4      # OPQ_ERR_WORKSPACE, nothing launched
    assert bool((y == 0).all())
