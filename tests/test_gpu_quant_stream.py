"""GPU parity of the batched (row-streaming) quantize against the fp64 oracle.

opq_quantize_batched runs a list of matrices through one persistent kernel: rows are copied
into a shared-memory ring and coded from there. Every matrix of a call must come out exactly
as the oracle quantizes it on its own (codes and signs bit-exact outside the 1e-6 tie band,
scales bit-exact), whatever the mix of shapes in the call, and no write may land outside an
output.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from oracle_pins import unpack_codes
from test_gpu_parity import TIE_FRACTION_LIMIT, alpha32, check_guards, guarded, no_device_error, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def batched_parity(ws, alpha, rows=None, ldws=None):
    """Quantize the bf16 matrices ``ws`` in one batched call (``ldws``: row strides, padding
    columns filled with garbage) and check each against the oracle on ``rows`` (all by default)."""
    jobs, outs, guards, bigs = [], [], [], []
    arr = (opq.QuantJob * len(ws))()
    for i, w in enumerate(ws):
        N, K = w.shape
        ldw = K if ldws is None else ldws[i]
        big = torch.full((N, ldw), float("nan"), dtype=torch.bfloat16, device=DEV)
        big[:, :K] = w
        bigs.append(big)
        cb, codes, cpad = guarded((N, K // 8), torch.int32, 0xA5)
        sb, signs, spad = guarded((N, K // 32), torch.int32, 0x5A)
        fb, scales, fpad = guarded((N,), torch.float32, 0x3C)
        guards += [(cb, cpad, 0xA5), (sb, spad, 0x5A), (fb, fpad, 0x3C)]
        outs.append((codes, signs, scales))
        arr[i] = opq.QuantJob(big.data_ptr(), N, K, ldw, codes.data_ptr(), signs.data_ptr(), scales.data_ptr())
    st = opq.load().opq_quantize_batched(ctypes.cast(arr, ctypes.c_void_p), len(ws), float(alpha),
                                         opq._stream(torch.device(DEV)))
    assert st == 0, st
    torch.cuda.synchronize()
    for g in guards:
        check_guards(*g)
    no_device_error()
    for i, (w, (codes, signs, scales)) in enumerate(zip(ws, outs)):
        sel = slice(None) if rows is None or rows[i] is None else np.asarray(rows[i])
        wc = w if rows is None or rows[i] is None else w[torch.as_tensor(rows[i], device=w.device)]
        ref = oracle.quantize(wc, alpha32(alpha), want_ties=True)
        assert np.array_equal(u32(scales.view(torch.int32))[sel], ref["scales"].view(np.uint32)), f"job {i}: scales"
        assert np.array_equal(u32(signs)[sel], ref["signs"]), f"job {i}: signs"
        qg, qo = unpack_codes(u32(codes)[sel]), unpack_codes(ref["codes"])
        mism = qg != qo
        near = ref["near_tie"].astype(bool)
        assert int((mism & ~near).sum()) == 0, f"job {i}: {int((mism & ~near).sum())} code mismatches"
        assert int((mism & near).sum()) <= TIE_FRACTION_LIMIT * qo.size
    return outs


@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_batched_tiny_and_projection(alpha):
    ws = [workloads.tiny().make_weights(DEV), workloads.dit_attn_proj().make_weights(DEV)]
    batched_parity(ws, alpha)


def test_batched_ragged_mix():
    """Row counts that leave partial units, K from 32 to 32768 in one call (one ring geometry for
    all: the widest row sets the slot, narrower rows share slots), padded row strides."""
    shapes = [(7, 32), (1, 64), (300, 3840), (5, 32768), (129, 10240), (37, 512), (3, 96), (1, 4128)]
    ws = [workloads.Linear("mix", 1, n, k, w_seed=17 * n + k).make_weights(DEV) for n, k in shapes]
    ldws = [k + 8 * (i % 3) for i, (_, k) in enumerate(shapes)]
    batched_parity(ws, 0.73, ldws=ldws)


@pytest.mark.parametrize("alpha", [0.1, 0.2, 3.0])
def test_batched_alpha_range(alpha):
    # alpha 0.1: most rows' code tables do not fit and those rows take the threshold search
    ws = [workloads.Linear("ar", 1, n, k, w_seed=n + k).make_weights(DEV) for n, k in ((40, 3840), (3, 10240))]
    batched_parity(ws, alpha)


def test_batched_special_rows():
    N, K = 8, 96
    g = torch.Generator(device=DEV).manual_seed(3)
    w = (torch.randn((N, K), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w[0] = 0                                  # all-zero row
    w[1] = -0.0                               # negative zeros only
    w[2, 5] = -w[2].abs().max() * 2           # negative maximum ...
    w[2, 9] = w[2].abs().max()                # ... duplicated with the other sign
    w[3] = torch.tensor([1.875] + [(2 * i - 1) / 16 for i in range(1, 16)] * 5 + [0.0] * 20,
                        dtype=torch.bfloat16, device=DEV)   # exact .5 ties at alpha = 1
    w[4] = torch.tensor([2.0 ** -130] * 48 + [-(2.0 ** -133)] * 48, dtype=torch.bfloat16, device=DEV)  # subnormal max
    for alpha in (0.73, 1.0):
        batched_parity([w], alpha)


def test_batched_whole_model_sampled():
    """Block 0 of the whole-model pass (7 matrices, 3 shape classes) in one call; sampled rows of
    each against the oracle, and every output equal to the one-matrix quantize."""
    model = workloads.WholeModel(blocks=1)
    ws = [l.make_weights(DEV) for l in model.layers]
    rows = [list(range(0, w.shape[0], 97)) + [w.shape[0] - 1] for w in ws]
    outs = batched_parity(ws, model.alpha, rows=rows)
    for w, got in zip(ws, outs):
        one = opq.quantize(w, model.alpha)
        for a, b in zip(got, one):
            assert torch.equal(a, b)


def test_batched_many_jobs_and_binding():
    """More matrices than one launch takes (128), through the Python binding; the descriptors
    built once serve repeated calls."""
    ws = [workloads.Linear("m", 1, 2 + (i % 5), 32 * (1 + i % 4), w_seed=i).make_weights(DEV) for i in range(300)]
    outs = opq.quantize_batched(ws, 0.73)
    jobs = opq.quantize_jobs(ws, outs, 0.73)
    outs2 = [tuple(torch.empty_like(t) for t in o) for o in outs]
    jobs2 = opq.quantize_jobs(ws, outs2, 0.73)
    opq.quantize_batched(ws, 0.73, outs=outs2, jobs=jobs2)
    opq.quantize_batched(ws, 0.73, outs=outs, jobs=jobs)
    no_device_error()
    for w, o, o2 in zip(ws, outs, outs2):
        ref = oracle.quantize(w, alpha32(0.73))
        assert np.array_equal(u32(o[0]), ref["codes"]) and np.array_equal(u32(o[1]), ref["signs"])
        assert np.array_equal(u32(o[2].view(torch.int32)), ref["scales"].view(np.uint32))
        for a, b in zip(o, o2):
            assert torch.equal(a, b)


def test_batched_argument_errors():
    w = workloads.tiny().make_weights(DEV)
    c, s, f = opq.quantize(w)
    arr = (opq.QuantJob * 1)()
    lib, st = opq.load(), opq._stream(torch.device(DEV))
    ptr = ctypes.cast(arr, ctypes.c_void_p)
    arr[0] = opq.QuantJob(w.data_ptr(), 256, 512, 512, c.data_ptr(), s.data_ptr(), f.data_ptr())
    assert lib.opq_quantize_batched(ptr, 0, 0.73, st) == 1                   # empty list
    assert lib.opq_quantize_batched(None, 1, 0.73, st) == 1                  # no list
    assert lib.opq_quantize_batched(ptr, 1, float("nan"), st) == 1           # bad alpha
    arr[0] = opq.QuantJob(w.data_ptr(), 256, 500, 512, c.data_ptr(), s.data_ptr(), f.data_ptr())
    assert lib.opq_quantize_batched(ptr, 1, 0.73, st) == 2                   # K % 32 != 0
    arr[0] = opq.QuantJob(w.data_ptr(), 256, 512, 508, c.data_ptr(), s.data_ptr(), f.data_ptr())
    assert lib.opq_quantize_batched(ptr, 1, 0.73, st) == 1                   # ldw < K
    arr[0] = opq.QuantJob(w.data_ptr() + 2, 256, 512, 512, c.data_ptr(), s.data_ptr(), f.data_ptr())
    assert lib.opq_quantize_batched(ptr, 1, 0.73, st) == 3                   # misaligned
    host = torch.empty((256, 512), dtype=torch.bfloat16)
    arr[0] = opq.QuantJob(host.data_ptr(), 256, 512, 512, c.data_ptr(), s.data_ptr(), f.data_ptr())
    assert lib.opq_quantize_batched(ptr, 1, 0.73, st) == 6                   # host memory
    no_device_error()


# a launch gives each CTA hundreds of one-warp rows from about 512 x 148 rows on: then the rows read
# the shared mantissa tables (built once per CTA) instead of building their own
STAB_ROWS = 80000


@pytest.mark.parametrize("alpha", [0.73, 1.0])
def test_power_of_two_scaled_rows(alpha):
    """A row scaled by powers of two from 2^-126 to 2^126, repeated over a matrix large enough for
    the shared mantissa tables (the rows share their max's mantissa: the tables serve them while
    their thresholds stay normal, the smallest scales fall back to the per-row path), with random
    rows between. Every row must match the oracle, and the scaled rows' codes must equal the
    unscaled row's while they stay normal."""
    K = 256
    g = torch.Generator(device=DEV).manual_seed(5)
    base = (torch.randn((1, K), generator=g, device=DEV) * 0.02).to(torch.bfloat16).float()
    exps = list(range(-126, 127, 2))
    scaled = torch.cat([base * (2.0 ** e) for e in exps]).to(torch.bfloat16)
    rand = (torch.randn((STAB_ROWS - len(exps), K), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w = torch.cat([scaled, rand])
    assert torch.isfinite(w.float()).all()
    codes, signs, scales = opq.quantize(w, alpha)
    no_device_error()
    ref = oracle.quantize(w, alpha32(alpha), want_ties=True)
    assert np.array_equal(u32(scales.view(torch.int32)), ref["scales"].view(np.uint32))
    assert np.array_equal(u32(signs), ref["signs"])
    qg, qo = unpack_codes(u32(codes)), unpack_codes(ref["codes"])
    mism = qg != qo
    near = ref["near_tie"].astype(bool)
    assert int((mism & ~near).sum()) == 0
    assert int((mism & near).sum()) <= TIE_FRACTION_LIMIT * qo.size
    i0 = exps.index(0)
    for i, e in enumerate(exps):
        if -96 <= e <= 126:
            assert torch.equal(codes[i], codes[i0]), f"exponent {e}"


def test_batched_large_launch_sampled():
    """21 projection-sized matrices in one call (80640 one-warp rows: the shared mantissa tables),
    sampled rows of each against the oracle and one whole matrix against the one-matrix call,
    which (3840 rows) builds per-row tables."""
    ws = [workloads.Linear("big", 1, 3840, 3840, w_seed=100 + i).make_weights(DEV) for i in range(21)]
    outs = opq.quantize_batched(ws, 0.73)
    no_device_error()
    rows = list(range(0, 3840, 173)) + [3839]
    for w, (c, s_, f) in zip(ws, outs):
        ref = oracle.quantize(w[rows].cpu(), alpha32(0.73), want_ties=True)
        assert np.array_equal(u32(f[rows].view(torch.int32)), ref["scales"].view(np.uint32))
        assert np.array_equal(u32(s_[rows]), ref["signs"])
        qg, qo = unpack_codes(u32(c[rows])), unpack_codes(ref["codes"])
        assert int(((qg != qo) & ~ref["near_tie"].astype(bool)).sum()) == 0
    one = opq.quantize(ws[7], 0.73)
    for a, b in zip(outs[7], one):
        assert torch.equal(a, b)
