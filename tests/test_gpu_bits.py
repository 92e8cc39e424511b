"""GPU parity of the 3-6 bit magnitudes against the oracle (codes bit-exact away from the
1e-6 tie band, signs and scales bit-exact, dequantized bf16 bit-exact)."""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from oracle_pins import _stream_codes, bits_to_f64
from test_gpu_parity import DEV, TIE_FRACTION_LIMIT, alpha32, check_guards, guarded, no_device_error, to_dev_u32, u16, u32

pytestmark = pytest.mark.gpu


def bits_parity(w, bits, alpha):
    N, K = w.shape
    cb, codes, cpad = guarded((N, K * bits // 32), torch.int32, 0xA5)
    sb, signs, spad = guarded((N, K // 32), torch.int32, 0x5A)
    fb, scales, fpad = guarded((N,), torch.float32, 0x3C)
    opq.quantize_bits(w, bits, alpha, out=(codes, signs, scales))
    torch.cuda.synchronize()
    for b, p, f in ((cb, cpad, 0xA5), (sb, spad, 0x5A), (fb, fpad, 0x3C)):
        check_guards(b, p, f)
    no_device_error()
    ref = oracle.quantize_bits(w, bits, alpha32(alpha), want_ties=True)
    assert np.array_equal(u32(scales.view(torch.int32)), ref["scales"].view(np.uint32))
    assert np.array_equal(u32(signs), ref["signs"])
    if np.array_equal(u32(codes), ref["codes"]):
        return ref
    qg, qo = _stream_codes(u32(codes), K, bits), _stream_codes(ref["codes"], K, bits)
    mism = qg != qo
    near = ref["near_tie"].astype(bool)
    assert int((mism & ~near).sum()) == 0
    assert int((mism & near).sum()) <= TIE_FRACTION_LIMIT * qo.size
    return ref


@pytest.mark.parametrize("bits", [3, 4, 5, 6])
@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_quantize_bits_tiny(bits, alpha):
    bits_parity(workloads.tiny().make_weights(DEV), bits, alpha)


@pytest.mark.parametrize("bits", [3, 5, 6])
@pytest.mark.parametrize("N,K", [(37, 96), (129, 4096), (300, 3840), (3, 32768)])
def test_quantize_bits_shapes(bits, N, K):
    lin = workloads.Linear("bits", 1, N, K, w_seed=N + K + bits)
    bits_parity(lin.make_weights(DEV), bits, 0.73)


@pytest.mark.parametrize("bits", [3, 5, 6])
@pytest.mark.parametrize("alpha", [0.2, 0.35])
@pytest.mark.parametrize("N,K", [(37, 96), (300, 3840), (3, 10240)])
def test_quantize_bits_small_alpha(bits, alpha, N, K):
    # small alpha stretches the levels over many binades: rows whose code table would not fit
    # (alpha below ~0.24 at 3 bits, ~0.44 at 6 bits for K <= 4096) take the threshold search
    lin = workloads.Linear("bits_alpha", 1, N, K, w_seed=7 * N + K + bits)
    bits_parity(lin.make_weights(DEV), bits, alpha)


@pytest.mark.parametrize("bits", [3, 5, 6])
def test_quantize_bits_special_rows(bits):
    N, K = 6, 96
    g = torch.Generator(device=DEV).manual_seed(11)
    w = (torch.randn((N, K), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w[0] = 0                                  # all-zero row
    w[1] = -0.0                               # negative zeros only
    w[2, 5] = -w[2].abs().max() * 2           # negative maximum ...
    w[2, 9] = w[2].abs().max()                # ... duplicated with the other sign
    w[3] = torch.tensor([2.0 ** -130] * 48 + [-(2.0 ** -133)] * 48, dtype=torch.bfloat16, device=DEV)  # subnormal max
    w[4, :] = w[4, 0]                         # a constant row
    for alpha in (0.45, 1.0):
        bits_parity(w, bits, alpha)


def test_quantize_bits_four_equals_nibble_format():
    w = workloads.dit_attn_proj().make_weights(DEV)
    a = opq.quantize_bits(w, 4)
    b = opq.quantize(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    no_device_error()


@pytest.mark.parametrize("bits", [3, 4, 5, 6])
@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_dequantize_bits_bit_exact(bits, alpha):
    lin = workloads.Linear("bits-dq", 1, 257, 1024, w_seed=bits)
    w = lin.make_weights("cpu")
    ref = oracle.quantize_bits(w, bits, alpha)
    want = oracle.dequantize_bits_bf16(ref["codes"], ref["signs"], ref["scales"], bits, alpha32(alpha))
    N, K = w.shape
    ob, out, pad = guarded((N, K), torch.bfloat16, 0x77)
    opq.dequantize_bits(to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]), torch.from_numpy(ref["scales"]).to(DEV),
                        bits, alpha, out=out)
    torch.cuda.synchronize()
    check_guards(ob, pad, 0x77)
    assert np.array_equal(u16(out), want)
    no_device_error()


@pytest.mark.parametrize("bits", [3, 6])
def test_bits_full_size_roundtrip(bits):
    # GPU quantize of the attention projection's weight, GPU dequantize of those planes equal
    # to the oracle's dequantize of the same planes
    lin = workloads.dit_attn_proj()
    w = lin.make_weights(DEV)
    codes, signs, scales = opq.quantize_bits(w, bits, lin.alpha)
    got = opq.dequantize_bits(codes, signs, scales, bits, lin.alpha)
    want = oracle.dequantize_bits_bf16(u32(codes), u32(signs), u32(scales.view(torch.int32)).view(np.float32), bits,
                                       alpha32(lin.alpha))
    assert np.array_equal(u16(got), want)
    no_device_error()


def test_bits_argument_errors():
    w = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(opq.OPQError):
        opq.quantize_bits(w, 7)
    with pytest.raises(opq.OPQError):
        opq.quantize_bits(w, 2)


# ---------------------------------------------------------------- linear --
def linear_bits_parity(x_cpu, w_cpu, bits, alpha, rows=None):
    """GPU linear on the oracle's `bits`-bit planes against x W'^T with the oracle's fp64 W':
    |y - y_ref| <= 1e-2 (|x| |W'|^T) + 1e-3 on every output (or the activation rows `rows`)."""
    ref = oracle.quantize_bits(w_cpu, bits, alpha)
    wq = oracle.dequantize_bits_f64(ref["codes"], ref["signs"], ref["scales"], bits, alpha32(alpha))
    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    yb, y, pad = guarded((M, N), torch.bfloat16, 0x6B)
    opq.linear_bits(x_cpu.to(DEV), to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]),
                    torch.from_numpy(ref["scales"]).to(DEV), bits, alpha, out=y)
    torch.cuda.synchronize()
    check_guards(yb, pad, 0x6B)
    no_device_error()
    sel = np.arange(M) if rows is None else np.asarray(rows)
    xs = bits_to_f64(x_cpu.view(torch.int16).numpy().view(np.uint16))[sel]
    yref = xs @ wq.T
    bound = np.abs(xs) @ np.abs(wq).T
    got = bits_to_f64(u16(y))[sel]
    err = np.abs(got - yref)
    tol = 1e-2 * bound + 1e-3
    assert not (err > tol).any(), f"{int((err > tol).sum())} outputs out of tolerance (worst {float((err / tol).max()):.3f})"


@pytest.mark.parametrize("bits", [3, 5, 6])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 384, 1024), (300, 131, 640), (700, 256, 384),
                                   (512, 10240, 256)])
def test_linear_bits(bits, M, N, K):
    # ragged activation and weight rows, several 128-K blocks; every M runs the 256-row tiles
    # (512 x 10240 x 256: 160 tiles, the 12 past the first wave as two half-width runs each)
    lin = workloads.Linear("bits-lin", M, N, K, w_seed=M + N + K + bits, x_seed=7 * bits + M)
    x, w = lin.make("cpu")
    linear_bits_parity(x, w, bits, 0.73)


@pytest.mark.parametrize("bits", [3, 6])
@pytest.mark.parametrize("alpha", [0.45, 1.0])
def test_linear_bits_alpha(bits, alpha):
    lin = workloads.Linear("bits-lin-a", 64, 256, 1024, w_seed=bits, x_seed=3)
    x, w = lin.make("cpu")
    linear_bits_parity(x, w, bits, alpha)


@pytest.mark.parametrize("bits", [3, 5, 6])
def test_linear_bits_full_size_sampled(bits):
    """The attention projection (x 3072 x 3840, W 3840 x 3840): whole waves of tiles and the
    split tail; every output of 40 activation rows spread over the tiles."""
    lin = workloads.dit_attn_proj()
    x, w = lin.make("cpu")
    rows = sorted(set(list(range(0, lin.M, 79)) + [lin.M - 1, 2047, 2048, 2303]))
    linear_bits_parity(x, w, bits, lin.alpha, rows=rows)


def test_linear_bits_four_is_the_nibble_linear():
    lin = workloads.Linear("bits4", 64, 256, 512, w_seed=5, x_seed=6)
    x, w = lin.make(DEV)
    planes = opq.quantize(w)
    assert torch.equal(opq.linear_bits(x, *planes, 4), opq.linear(x, *planes))


def test_linear_bits_argument_errors():
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((8, 96), dtype=torch.bfloat16, device=DEV)
    c, s, f = opq.quantize_bits(w, 3)
    y = torch.empty((4, 8), dtype=torch.bfloat16, device=DEV)
    lib, st = opq.load(), opq._stream(x.device)
    # K % 128 != 0 at 3 bits
    assert lib.opq_linear_bits(opq._ptr(x), 4, 96, opq._ptr(c), opq._ptr(s), opq._ptr(f), 8, 3, 0.73, opq._ptr(y),
                               None, 0, st) == 2
    for b in (2, 7):
        assert lib.opq_linear_bits(opq._ptr(x), 4, 96, opq._ptr(c), opq._ptr(s), opq._ptr(f), 8, b, 0.73,
                                   opq._ptr(y), None, 0, st) == 1
    no_device_error()
