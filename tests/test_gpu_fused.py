"""GPU parity of the fused epilogue (bias, SiLU, GELU tanh form) against the oracle.

The oracle's linear (fp64) goes through the oracle's epilogue act(y + bias[n]); the GPU
output may differ by the linear's tolerance carried through the activation (Lipschitz
constant below 1.15 for both) plus the bias' share of the bf16 rounding:
|y - y_ref| <= 1.15 (1e-2 (|x| |W'|^T + |bias|) + 1e-3).
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from test_gpu_parity import DEV, check_guards, guarded, no_device_error, to_dev_u32, u16

pytestmark = pytest.mark.gpu

ACTS = {"none": 0, "silu": 1, "gelu_tanh": 2}


def bias_for(N, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(N, generator=g) * 2.0).to(torch.bfloat16)


def check(yg, yref, bound, b):
    got = (u16(yg).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    babs = np.abs((u16(b).astype(np.uint32) << 16).view(np.float32).astype(np.float64))[None, :] if b is not None else 0.0
    tol = 1.15 * (1e-2 * (bound + babs) + 1e-3)
    err = np.abs(got - yref)
    assert not (err > tol).any(), f"{int((err > tol).sum())} outputs out of tolerance"
    assert np.isfinite(got).all()


@pytest.mark.parametrize("act", list(ACTS))
@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("M,N,K", [(1, 300, 512), (40, 1000, 640), (300, 130, 1280), (512, 10240, 1024),
                                   (512, 10240, 256)])
def test_linear_fused(act, with_bias, M, N, K):
    lin = workloads.Linear("fused", M, N, K, w_seed=M + N, x_seed=K)
    x, w = lin.make("cpu")
    ref = oracle.quantize(w, lin.alpha)
    b = bias_for(N, N) if with_bias else None
    yb, y, pad = guarded((M, N), torch.bfloat16, 0x6B)
    opq.linear_fused(x.to(DEV), to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]),
                     torch.from_numpy(ref["scales"]).to(DEV), lin.alpha,
                     bias=b.to(DEV) if b is not None else None, act=act, out=y)
    torch.cuda.synchronize()
    check_guards(yb, pad, 0x6B)
    no_device_error()
    y0, bound = oracle.linear(x, ref["codes"], ref["signs"], ref["scales"], lin.alpha)
    check(y, oracle.apply_epilogue(y0, b, ACTS[act]), bound, b)


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
@pytest.mark.parametrize("M,N,K,gs", [(16, 600, 768, 128), (300, 512, 1024, 64)])
def test_linear_grouped_fused(act, M, N, K, gs):
    lin = workloads.Linear("fused-g", M, N, K, w_seed=N, x_seed=M)
    x, w = lin.make("cpu")
    ref = oracle.quantize_grouped(w, gs, lin.alpha)
    b = bias_for(N, M)
    y = opq.linear_grouped_fused(x.to(DEV), to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]),
                                 torch.from_numpy(ref["gmax"].view(np.float16)).to(DEV), lin.alpha,
                                 bias=b.to(DEV), act=act)
    torch.cuda.synchronize()
    no_device_error()
    y0, bound = oracle.linear_grouped(x, ref["codes"], ref["signs"], ref["gmax"], lin.alpha)
    check(y, oracle.apply_epilogue(y0, b, ACTS[act]), bound, b)


def test_fused_none_equals_unfused():
    # no bias, no activation: the fused entry point writes the same bits as opq_linear
    for M in (16, 700):
        lin = workloads.Linear("fused-eq", M, 1024, 1024, w_seed=1, x_seed=2)
        x, w = lin.make(DEV)
        planes = opq.quantize(w)
        assert torch.equal(opq.linear(x, *planes), opq.linear_fused(x, *planes))
    no_device_error()


def test_fused_bad_activation():
    x = torch.zeros((2, 32), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((4, 32), dtype=torch.bfloat16, device=DEV)
    c, s, sc = opq.quantize(w)
    y = torch.empty((2, 4), dtype=torch.bfloat16, device=DEV)
    lib = opq.load()
    P = opq._ptr
    st = lib.opq_linear_fused(P(x), 2, 32, P(c), P(s), P(sc), 4, 0.73, None, 7, P(y), None, 0, opq._stream(x.device))
    assert st == 1
