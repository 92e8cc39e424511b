"""GPU parity of the 3-6 bit magnitudes against the oracle (codes bit-exact away from the
1e-6 tie band, signs and scales bit-exact, dequantized bf16 bit-exact)."""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from oracle_pins import _stream_codes
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
