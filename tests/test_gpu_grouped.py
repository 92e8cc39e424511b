"""GPU parity of the group-wise format (one float16 max per GS weights) against the oracle.

Same rules as the per-row format: codes and signs bit-exact away from the 1e-6 tie
band (mismatches inside it under 1e-6 of all entries), group maxima bit-exact,
dequantized bf16 bit-exact, linear within 1e-2 |x| |W'|^T + 1e-3. Inputs come from
``workloads`` and explicit edge rows; the packed weights fed to the GPU dequantize
and linear are the oracle's own.
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from oracle_pins import unpack_codes
from test_gpu_parity import (DEV, TIE_FRACTION_LIMIT, alpha32, check_guards, guarded, no_device_error, to_dev_u32, u16,
                             u32)

pytestmark = pytest.mark.gpu

GROUP_SIZES = (32, 64, 128, 256)


def grouped_quant_parity(w: torch.Tensor, gs: int, alpha: float):
    N, K = w.shape
    cb, codes, cpad = guarded((N, K // 8), torch.int32, 0xA5)
    sb, signs, spad = guarded((N, K // 32), torch.int32, 0x5A)
    gb, gmax, gpad = guarded((N, K // gs), torch.float16, 0x3C)
    opq.quantize_grouped(w, gs, alpha, out=(codes, signs, gmax))
    torch.cuda.synchronize()
    check_guards(cb, cpad, 0xA5)
    check_guards(sb, spad, 0x5A)
    check_guards(gb, gpad, 0x3C)
    no_device_error()
    ref = oracle.quantize_grouped(w, gs, alpha32(alpha), want_ties=True)
    assert np.array_equal(u16(gmax), ref["gmax"]), "group maxima differ"
    assert np.array_equal(u32(signs), ref["signs"]), "signs differ"
    qg, qo = unpack_codes(u32(codes)), unpack_codes(ref["codes"])
    mism = qg != qo
    near = ref["near_tie"].astype(bool)
    assert int((mism & ~near).sum()) == 0, f"{int((mism & ~near).sum())} code mismatches away from ties"
    assert int((mism & near).sum()) <= TIE_FRACTION_LIMIT * qo.size
    return ref


@pytest.mark.parametrize("gs", GROUP_SIZES)
@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_quantize_grouped_tiny(gs, alpha):
    grouped_quant_parity(workloads.tiny().make_weights(DEV), gs, alpha)


@pytest.mark.parametrize("gs", GROUP_SIZES)
@pytest.mark.parametrize("N,K", [(37, 512), (129, 4096), (300, 3840), (2, 32768), (3, 1280)])
def test_quantize_grouped_shapes(gs, N, K):
    if K % gs:
        pytest.skip("group size does not divide K")
    lin = workloads.Linear("grouped", 1, N, K, w_seed=N * 7 + K + gs)
    grouped_quant_parity(lin.make_weights(DEV), gs, 0.73)


def test_quantize_grouped_odd_rounds():
    # K = 96 and 160: the row ends inside a 256-weight round (groups of 32)
    for K in (96, 160):
        lin = workloads.Linear("grouped-odd", 1, 9, K, w_seed=K)
        grouped_quant_parity(lin.make_weights(DEV), 32, 0.73)


def test_quantize_grouped_edge_groups():
    # zero groups, negative zeros, a max beyond float16 (saturates to 65504: the big weights
    # code to 15), a max in float16's subnormal range (rounds down: the max codes to 15),
    # exact .5 ties at alpha = 1
    K = 256
    rows = torch.zeros((4, K), dtype=torch.float64)
    rows[0, 40:50] = -0.0
    rows[1, 3] = 1e5
    rows[1, 4] = -7e4
    rows[1, 5] = 300.0
    rows[2, 70] = 2.0 ** -20 + 2.0 ** -27
    rows[2, 71] = -(2.0 ** -22)
    rows[3, :16] = torch.tensor([1.875] + [(2 * i - 1) / 16 for i in range(1, 16)], dtype=torch.float64)
    w = rows.to(torch.bfloat16).to(DEV)
    for gs in GROUP_SIZES:
        for alpha in (0.73, 1.0):
            ref = grouped_quant_parity(w, gs, alpha)
            assert ref["gmax"][1, 0] == 0x7BFF


@pytest.mark.parametrize("gs", GROUP_SIZES)
@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_dequantize_grouped_bit_exact(gs, alpha):
    lin = workloads.Linear("grouped-dq", 1, 257, 1024, w_seed=gs)
    w = lin.make_weights("cpu")
    ref = oracle.quantize_grouped(w, gs, alpha)
    want = oracle.dequantize_grouped_bf16(ref["codes"], ref["signs"], ref["gmax"], alpha32(alpha))
    N, K = w.shape
    ob, out, pad = guarded((N, K), torch.bfloat16, 0x77)
    gmax = torch.from_numpy(ref["gmax"].view(np.float16)).to(DEV)
    opq.dequantize_grouped(to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]), gmax, alpha, out=out)
    torch.cuda.synchronize()
    check_guards(ob, pad, 0x77)
    assert np.array_equal(u16(out), want)
    no_device_error()


def test_grouped_full_size_roundtrip():
    # the attention projection's weight at the card's group size: GPU quantize matches the
    # oracle, GPU dequantize of the GPU planes matches the oracle's dequantize bit for bit
    lin = workloads.dit_attn_proj()
    w = lin.make_weights(DEV)
    ref = grouped_quant_parity(w, 128, lin.alpha)
    codes, signs, gmax = opq.quantize_grouped(w, 128, lin.alpha)
    got = opq.dequantize_grouped(codes, signs, gmax, lin.alpha)
    want = oracle.dequantize_grouped_bf16(u32(codes), u32(signs), u16(gmax), alpha32(lin.alpha))
    assert np.array_equal(u16(got), want)
    assert ref["gmax"].shape == (3840, 30)
    no_device_error()


def test_grouped_argument_errors():
    w = torch.zeros((4, 96), dtype=torch.bfloat16, device=DEV)
    c = torch.empty((4, 12), dtype=torch.int32, device=DEV)
    s = torch.empty((4, 3), dtype=torch.int32, device=DEV)
    g = torch.empty((4, 3), dtype=torch.float16, device=DEV)
    lib = opq.load()
    P = opq._ptr
    st = opq._stream(w.device)
    assert lib.opq_quantize_grouped(P(w), 4, 96, 96, 48, 0.73, P(c), P(s), P(g), st) == 1    # not a listed size
    assert lib.opq_quantize_grouped(P(w), 4, 96, 96, 64, 0.73, P(c), P(s), P(g), st) == 2    # 64 does not divide 96
    assert lib.opq_quantize_grouped(P(w), 4, 96, 96, 32, 0.73, P(c), P(s), P(g), st) == 0
    assert lib.opq_dequantize_grouped(P(c), P(s), P(g), 4, 96, 128, 0.73, P(w), st) == 2
    torch.cuda.synchronize()
    no_device_error()


# -------------------------------------------------------------------- linear --
def grouped_linear_parity(x_cpu, w_cpu, gs, alpha, pairs=None, seed=0):
    ref = oracle.quantize_grouped(w_cpu, gs, alpha)
    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    codes, signs = to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"])
    gmax = torch.from_numpy(ref["gmax"].view(np.float16)).to(DEV)
    yb, y, pad = guarded((M, N), torch.bfloat16, 0x6B)
    opq.linear_grouped(x_cpu.to(DEV), codes, signs, gmax, alpha, out=y)
    torch.cuda.synchronize()
    check_guards(yb, pad, 0x6B)
    no_device_error()
    yg = (u16(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if pairs is None:
        yref, bound = oracle.linear_grouped(x_cpu, ref["codes"], ref["signs"], ref["gmax"], alpha)
        got = yg
    else:
        rng = np.random.default_rng(seed)
        ms = np.concatenate([rng.integers(0, M, pairs), [0, M - 1, 0, M - 1]])
        ns = np.concatenate([rng.integers(0, N, pairs), [0, N - 1, N - 1, 0]])
        yref, bound = oracle.linear_grouped_pairs(x_cpu, ref["codes"], ref["signs"], ref["gmax"], alpha, ms, ns)
        got = yg[ms, ns]
    err = np.abs(got - yref)
    tol = 1e-2 * bound + 1e-3
    assert not (err > tol).any(), f"{int((err > tol).sum())} outputs out of tolerance"
    assert np.isfinite(got).all()
    return y


@pytest.mark.parametrize("gs", GROUP_SIZES)
@pytest.mark.parametrize("M,N,K", [(1, 300, 512), (17, 257, 1024), (129, 600, 768), (300, 130, 1280)])
def test_linear_grouped_shapes(gs, M, N, K):
    if K % gs:
        pytest.skip("group size does not divide K")
    lin = workloads.Linear("grouped-lin", M, N, K, w_seed=M + N + gs, x_seed=K + gs)
    x, w = lin.make("cpu")
    grouped_linear_parity(x, w, gs, 0.73)


@pytest.mark.parametrize("alpha", [0.45, 1.0])
def test_linear_grouped_alpha(alpha):
    lin = workloads.Linear("grouped-alpha", 64, 384, 640, alpha=alpha, w_seed=5, x_seed=6)
    x, w = lin.make("cpu")
    grouped_linear_parity(x, w, 128, alpha)


@pytest.mark.parametrize("M,N,K,gs", [(512, 10240, 1024, 128), (300, 9728, 256, 64), (512, 10240, 1152, 32)])
def test_linear_grouped_tails(M, N, K, gs):
    # past the last whole wave: half-K runs whose partial sums meet in the workspace (K >= 1024),
    # or half-row runs (K = 256)
    lin = workloads.Linear("grouped-tail", M, N, K, w_seed=N, x_seed=M)
    x, w = lin.make("cpu")
    grouped_linear_parity(x, w, gs, 0.73)


@pytest.mark.parametrize("M,K,gs", [(16, 1024, 128), (40, 512, 64)])
def test_linear_grouped_narrow_whole_tiles(M, K, gs):
    # more weight tiles than the stream-K counters cover (4194 > 4096): small M runs whole narrow
    # tiles with the group-wise decode; random packed planes and maxima, sampled outputs
    N = 4194 * 128 - 37
    assert opq.plan(M, N, K)[0] == 0
    codes, signs, _ = workloads.random_planes(N, K, 11)
    gmax = workloads.random_gmax(N, K // gs, 12)
    x = workloads.Linear("grouped-whole", M, N, K, x_seed=13).make_x("cpu")
    y = opq.linear_grouped(x.to(DEV), to_dev_u32(codes), to_dev_u32(signs),
                           torch.from_numpy(gmax.view(np.int16)).to(DEV), 0.73)
    torch.cuda.synchronize()
    no_device_error()
    rng = np.random.default_rng(14)
    ms = np.concatenate([rng.integers(0, M, 3000), np.arange(M), np.arange(M)])
    ns = np.concatenate([rng.integers(0, N, 3000), np.full(M, N - 1), np.zeros(M, np.int64)])
    yref, bound = oracle.linear_grouped_pairs(x, codes, signs, gmax, 0.73, ms, ns)
    got = (u16(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)[ms, ns]
    err = np.abs(got - yref)
    tol = 1e-2 * bound + 1e-3
    assert not (err > tol).any(), f"{int((err > tol).sum())} outputs out of tolerance"


def test_linear_grouped_full_size_sampled():
    lin = workloads.dit_attn_proj()
    x, w = lin.make("cpu")
    grouped_linear_parity(x, w, 128, lin.alpha, pairs=3000, seed=1)


def test_linear_grouped_deterministic_and_planes_from_gpu():
    lin = workloads.Linear("grouped-det", 700, 3840, 1024, w_seed=1, x_seed=2)
    x, w = lin.make(DEV)
    planes = opq.quantize_grouped(w, 128, lin.alpha)
    ws = torch.zeros(max(opq.grouped_workspace_size(700, 3840, 1024, 128), 16), dtype=torch.uint8, device=DEV)
    y1 = opq.linear_grouped(x, *planes, lin.alpha, workspace=ws)
    y2 = opq.linear_grouped(x, *planes, lin.alpha, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert int(ws[:65536].count_nonzero()) == 0
    no_device_error()
