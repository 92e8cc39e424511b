"""GPU parity of the batched dequantize: a list of packed matrices decoded in one pass must give,
for every matrix, exactly the bf16 W' that the oracle defines (and that opq_dequantize gives on
its own), whatever the mix of shapes in the call, with no write outside an output."""
import ctypes

import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from test_gpu_parity import DEV, alpha32, check_guards, guarded, no_device_error, to_dev_u32, u16

pytestmark = pytest.mark.gpu


def oracle_planes(shapes, alpha, seed=0):
    """(CPU weights, oracle planes on the device) for each shape."""
    out = []
    for i, (n, k) in enumerate(shapes):
        w = workloads.Linear("dqb", 1, n, k, w_seed=seed + 31 * i + n + k).make_weights("cpu")
        ref = oracle.quantize(w, alpha32(alpha))
        out.append((ref, (to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]), torch.from_numpy(ref["scales"]).to(DEV))))
    return out


@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_batched_mixed_shapes_bit_exact(alpha):
    shapes = [(1, 32), (7, 96), (300, 3840), (5, 32768), (129, 10240), (37, 512), (3, 4128)]
    items = oracle_planes(shapes, alpha)
    guards, outs = [], []
    arr = (opq.DequantJob * len(items))()
    for i, ((ref, (c, s, f)), (n, k)) in enumerate(zip(items, shapes)):
        ob, out, pad = guarded((n, k), torch.bfloat16, 0x77)
        guards.append((ob, pad))
        outs.append(out)
        arr[i] = opq.DequantJob(c.data_ptr(), s.data_ptr(), f.data_ptr(), n, k, out.data_ptr())
    st = opq.load().opq_dequantize_batched(ctypes.cast(arr, ctypes.c_void_p), len(items), float(alpha),
                                           opq._stream(torch.device(DEV)))
    assert st == 0, st
    torch.cuda.synchronize()
    for ob, pad in guards:
        check_guards(ob, pad, 0x77)
    no_device_error()
    for (ref, planes), out in zip(items, outs):
        want = oracle.dequantize_bf16(ref["codes"], ref["signs"], ref["scales"], alpha32(alpha))
        assert np.array_equal(u16(out), want)
        assert torch.equal(out, opq.dequantize(*planes, alpha))


def test_batched_many_jobs_and_binding():
    """More matrices than one launch takes (128), through the binding; the descriptors built once
    serve repeated calls."""
    ws = [workloads.Linear("m", 1, 2 + (i % 5), 32 * (1 + i % 4), w_seed=i).make_weights(DEV) for i in range(300)]
    planes = opq.quantize_batched(ws, 0.73)
    outs = opq.dequantize_batched(planes, 0.73)
    jobs = opq.dequantize_jobs(planes, outs)
    for o in outs:
        o.zero_()
    opq.dequantize_batched(planes, 0.73, outs=outs, jobs=jobs)
    no_device_error()
    for p, o in zip(planes, outs):
        assert torch.equal(o, opq.dequantize(*p, 0.73))


def test_batched_whole_model_block():
    """Block 0 of the whole-model pass (7 matrices, 3 shape classes) in one call, every output equal
    to the one-matrix dequantize; sampled rows of each against the oracle."""
    model = workloads.WholeModel(blocks=1)
    ws = [l.make_weights(DEV) for l in model.layers]
    planes = opq.quantize_batched(ws, model.alpha)
    outs = opq.dequantize_batched(planes, model.alpha)
    no_device_error()
    for w, p, o in zip(ws, planes, outs):
        assert torch.equal(o, opq.dequantize(*p, model.alpha))
        rows = list(range(0, w.shape[0], 211)) + [w.shape[0] - 1]
        ref = oracle.quantize(w[rows].cpu(), alpha32(model.alpha))
        want = oracle.dequantize_bf16(ref["codes"], ref["signs"], ref["scales"], alpha32(model.alpha))
        assert np.array_equal(u16(o[rows]), want)


def test_batched_argument_errors():
    w = workloads.tiny().make_weights(DEV)
    c, s, f = opq.quantize(w)
    out = torch.empty_like(w)
    N, K = w.shape
    arr = (opq.DequantJob * 1)()
    lib, st = opq.load(), opq._stream(torch.device(DEV))
    ptr = ctypes.cast(arr, ctypes.c_void_p)
    arr[0] = opq.DequantJob(c.data_ptr(), s.data_ptr(), f.data_ptr(), N, K, out.data_ptr())
    assert lib.opq_dequantize_batched(ptr, 0, 0.73, st) == 1                  # empty list
    assert lib.opq_dequantize_batched(ptr, 1, 0.0, st) == 1                   # bad alpha
    arr[0] = opq.DequantJob(c.data_ptr(), s.data_ptr(), f.data_ptr(), N, K + 8, out.data_ptr())
    assert lib.opq_dequantize_batched(ptr, 1, 0.73, st) == 2                  # K % 32 != 0
    arr[0] = opq.DequantJob(c.data_ptr(), s.data_ptr(), f.data_ptr(), N, K, out.data_ptr() + 2)
    assert lib.opq_dequantize_batched(ptr, 1, 0.73, st) == 3                  # misaligned
    host = torch.empty((N, K), dtype=torch.bfloat16)
    arr[0] = opq.DequantJob(c.data_ptr(), s.data_ptr(), f.data_ptr(), N, K, host.data_ptr())
    assert lib.opq_dequantize_batched(ptr, 1, 0.73, st) == 6                  # host memory
    no_device_error()
