"""C-ABI checks that need no GPU: the library loads, exports every entry point
that include/opq.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_diffusion_transformer_b200 as opq
from bit_diffusion_transformer_b200 import build as opq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "opq.h")


@pytest.fixture(scope="module")
def lib():
    opq_build.build()
    return opq.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(opq_[a-z_0-9]+)\s*\(", src)))


def test_header_declarations_are_exported(lib):
    names = declared_functions()
    assert "opq_quantize" in names and "opq_linear" in names and "opq_dequantize" in names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in opq.h but not exported"
    assert set(names) == set(opq.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.opq_abi_version() == 1
    for code, name in [(0, b"OPQ_OK"), (1, b"OPQ_ERR_INVALID_ARG"), (2, b"OPQ_ERR_UNSUPPORTED_SHAPE"),
                       (3, b"OPQ_ERR_MISALIGNED"), (4, b"OPQ_ERR_WORKSPACE"), (5, b"OPQ_ERR_CUDA"),
                       (6, b"OPQ_ERR_NOT_DEVICE_MEMORY"), (99, b"OPQ_ERR_UNKNOWN")]:
        assert lib.opq_status_string(code) == name


def _buf(nbytes, offset=0):
    a = np.zeros(nbytes + 64, np.uint8)
    base = (-a.ctypes.data) % 16
    return a, ctypes.c_void_p(a.ctypes.data + base + offset)


def test_quantize_argument_errors(lib):
    keep = []
    def b(n, off=0):
        a, p = _buf(n, off)
        keep.append(a)
        return p
    w, c, s, sc = b(256 * 2), b(64), b(16), b(16)
    q = lib.opq_quantize
    assert q(None, 4, 32, 32, 0.73, c, s, sc, None) == 1          # null pointer
    assert q(w, 0, 32, 32, 0.73, c, s, sc, None) == 1             # N = 0
    assert q(w, 4, 48, 48, 0.73, c, s, sc, None) == 2             # K % 32 != 0
    assert q(w, 4, 32 * 1025 * 1, 32 * 1025, 0.73, c, s, sc, None) == 2  # K beyond 32768
    assert q(w, 4, 32, 16, 0.73, c, s, sc, None) == 1             # ldw < K
    assert q(w, 4, 32, 36, 0.73, c, s, sc, None) == 1             # ldw % 8 != 0
    for bad in (0.0, -0.5, float("nan"), float("inf")):
        assert q(w, 4, 32, 32, bad, c, s, sc, None) == 1          # alpha
    assert q(b(512, 2), 4, 32, 32, 0.73, c, s, sc, None) == 3     # misaligned
    assert q(w, 4, 32, 32, 0.73, c, s, sc, None) == 6             # host memory, not device memory


def test_dequantize_and_linear_argument_errors(lib):
    keep = []
    def b(n, off=0):
        a, p = _buf(n, off)
        keep.append(a)
        return p
    c, s, sc, out = b(64), b(16), b(16), b(512)
    assert lib.opq_dequantize(c, s, sc, 4, 40, 0.73, out, None) == 2
    assert lib.opq_dequantize(c, s, sc, 4, 32, 0.0, out, None) == 1
    assert lib.opq_dequantize(c, None, sc, 4, 32, 0.73, out, None) == 1
    assert lib.opq_dequantize(c, s, sc, 4, 32, 0.73, out, None) == 6
    # the batched form: the list, then every descriptor, is checked before anything runs
    J = (opq.DequantJob * 2)()
    J[0] = opq.DequantJob(c, s, sc, 4, 32, out)
    J[1] = opq.DequantJob(c, s, sc, 4, 32, out)
    jp = ctypes.cast(J, ctypes.c_void_p)
    assert lib.opq_dequantize_batched(None, 1, 0.73, None) == 1          # no list
    assert lib.opq_dequantize_batched(jp, 0, 0.73, None) == 1            # empty list
    assert lib.opq_dequantize_batched(jp, 2, float("nan"), None) == 1    # bad alpha
    J[1] = opq.DequantJob(c, s, sc, 4, 40, out)
    assert lib.opq_dequantize_batched(jp, 2, 0.73, None) == 2            # K % 32 != 0 in the second job
    J[1] = opq.DequantJob(c, s, sc, 4, 32, out)
    J[0] = opq.DequantJob(c, None, sc, 4, 32, out)
    assert lib.opq_dequantize_batched(jp, 2, 0.73, None) == 1            # null pointer
    J[0] = opq.DequantJob(c, s, sc, 4, 32, out)
    assert lib.opq_dequantize_batched(jp, 2, 0.73, None) == 6            # host memory
    x, y = b(4096), b(4096)
    L = lib.opq_linear
    assert L(x, 0, 32, c, s, sc, 4, 0.73, y, None, 0, None) == 1
    assert L(x, 2, 33, c, s, sc, 4, 0.73, y, None, 0, None) == 2
    assert L(x, 2, 32, c, s, sc, 0, 0.73, y, None, 0, None) == 1
    assert L(x, 2, 32, c, s, sc, 4, float("nan"), y, None, 0, None) == 1
    assert L(x, 2, 32, c, s, sc, 4, 0.73, b(64, 8), None, 0, None) == 3
    assert L(x, 2, 32, c, s, sc, 4, 0.73, y, None, 0, None) == 6


def test_grouped_fused_bits_alpha_argument_errors(lib):
    keep = []
    def b(n, off=0):
        a, p = _buf(n, off)
        keep.append(a)
        return p
    w, c, s, g, sc, out = b(256 * 2), b(64), b(16), b(64), b(16), b(512)
    # group-wise: listed sizes only, dividing K
    assert lib.opq_quantize_grouped(w, 4, 96, 96, 48, 0.73, c, s, g, None) == 1
    assert lib.opq_quantize_grouped(w, 4, 96, 96, 64, 0.73, c, s, g, None) == 2
    assert lib.opq_quantize_grouped(w, 4, 96, 96, 32, 0.73, c, s, g, None) == 6     # host memory
    assert lib.opq_dequantize_grouped(c, s, g, 4, 96, 128, 0.73, out, None) == 2
    sz = ctypes.c_size_t(0)
    assert lib.opq_linear_grouped_workspace_size(4, 4, 96, 48, ctypes.byref(sz)) == 1
    # fused epilogue: activation codes 0..2 only, checked before the pointers
    x, y = b(4096), b(4096)
    assert lib.opq_linear_fused(x, 2, 32, c, s, sc, 4, 0.73, None, 3, y, None, 0, None) == 1
    assert lib.opq_linear_fused(x, 2, 32, c, s, sc, 4, 0.73, None, -1, y, None, 0, None) == 1
    assert lib.opq_linear_fused(x, 2, 32, c, s, sc, 4, 0.73, None, 1, y, None, 0, None) == 6
    assert lib.opq_linear_grouped_fused(x, 2, 32, c, s, g, 4, 48, 0.73, None, 1, y, None, 0, None) == 1
    # bit widths 3..6
    for bits in (0, 2, 7, 8):
        assert lib.opq_quantize_bits(w, 4, 32, 32, bits, 0.73, c, s, sc, None) == 1
        assert lib.opq_dequantize_bits(c, s, sc, 4, 32, bits, 0.73, out, None) == 1
    assert lib.opq_quantize_bits(w, 4, 48, 48, 3, 0.73, c, s, sc, None) == 2
    assert lib.opq_quantize_bits(w, 4, 32, 36, 3, 0.73, c, s, sc, None) == 1       # ldw % 8 != 0
    assert lib.opq_quantize_bits(w, 4, 32, 32, 5, 0.73, c, s, sc, None) == 6
    assert lib.opq_dequantize_bits(c, s, sc, 4, 32, 6, float("nan"), out, None) == 1
    assert lib.opq_dequantize_bits(c, s, sc, 4, 32, 6, 0.73, out, None) == 6
    # alpha search: at least one candidate, every candidate finite and > 0
    alphas = (ctypes.c_float * 2)(0.5, 0.73)
    snr = (ctypes.c_double * 2)()
    best = ctypes.c_float()
    ab = lib.opq_alpha_search
    assert ab(w, 4, 32, 32, 0, alphas, 0, snr, ctypes.byref(best), None, 0, None) == 1
    assert ab(w, 4, 32, 32, 0, (ctypes.c_float * 1)(-1.0), 1, snr, ctypes.byref(best), None, 0, None) == 1
    assert ab(w, 4, 32, 32, 48, alphas, 2, snr, ctypes.byref(best), None, 0, None) == 1
    assert ab(w, 4, 32, 32, 0, alphas, 2, None, ctypes.byref(best), None, 0, None) == 1
    assert ab(w, 4, 32, 32, 0, alphas, 2, snr, ctypes.byref(best), None, 0, None) == 6


def test_plan_and_workspace_host_logic(lib):
    # small M: stream-K over (128-row weight tile, load group) units on at most 148 CTAs; a load
    # group is 4 (16-row tiles), 2 (32- and 64-row tiles) or 1 consecutive 128-K blocks, the
    # tile's blocks split into ceil(blocks / group) groups; narrow tiles need K % 128 == 0
    for M, N, K in [(1, 11520, 3840), (16, 11520, 3840), (64, 11520, 3840), (128, 11520, 3840),
                    (1, 3840, 3840), (17, 257, 96), (1, 64, 32), (5, 300, 640), (40, 1000, 160)]:
        path, ctas, launches = opq.plan(M, N, K)
        assert path == 1 and launches == 1
        bx = 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128
        if K % 128:
            bx = 128
        grp = 4 if bx <= 16 else 2 if bx <= 64 else 1
        groups = -(-(-(-K // 128)) // grp)
        units = -(-N // 128) * groups
        assert ctas == min(148, units)
        per = -(-units // ctas)
        runs_max = -(-per // groups) + 1
        counters = 4096 * 4 * 4        # fixed region: 4 arrival counters for each of up to 4096 weight tiles
        assert opq.workspace_size(M, N, K) == counters + ctas * runs_max * bx * 128 * 4
    # stream-K deals its units in 32-bit arithmetic: it is planned only while units x 148 CTAs
    # stays below 2^31 (4096 weight tiles x 3542 load groups of 4 blocks is the last such shape)
    for groups in (3541, 3542, 3543, 4000):
        K = 128 * 4 * groups
        units = 4096 * groups
        path, ctas, _ = opq.plan(1, 4096 * 128, K)
        assert path == (1 if units * 148 < 2 ** 31 else 0) and ctas == 148
        assert (opq.workspace_size(1, 4096 * 128, K) > 0) == (path == 1)
    # small M past stream-K's range runs whole narrow tiles only for whole 128-K blocks; with
    # K % 128 != 0 (sign words copied by cp.async) that schedule is refused, not run
    sz = ctypes.c_size_t(0)
    pth, cts, lau = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    for M, N, K in [(8, 4194 * 128 - 37, 160), (100, 4097 * 128, 96), (1, 4096 * 128, 128 * 4 * 3543 + 32)]:
        assert lib.opq_linear_workspace_size(M, N, K, ctypes.byref(sz)) == 2
        assert lib.opq_linear_plan(M, N, K, ctypes.byref(pth), ctypes.byref(cts), ctypes.byref(lau)) == 2
        with pytest.raises(opq.OPQError):
            opq.plan(M, N, K)
    assert opq.plan(129, 4097 * 128, 96)[0] == 0          # M > 128: the 256-row tiles serve it
    assert opq.plan(8, 4096 * 128, 160)[0] == 1           # within stream-K's range: served
    # large M: whole 128 x 256 tiles, one persistent CTA per SM. Tiles past the last whole wave,
    # when at most half as many as CTAs, run on two CTAs each; 256-row tiles of at least 8
    # 128-K blocks split K, and their fp32 partial sums (128 x 256 per tail tile) meet in the
    # workspace after the counter region; everything else needs no workspace
    for M, N, K in [(129, 100, 32), (3072, 3840, 3840), (4096, 10240, 3840), (8, 4097 * 128, 128),
                    (512, 10240, 256), (512, 10240, 1024), (300, 9728, 160)]:
        path, ctas, launches = opq.plan(M, N, K)
        assert path == 0 and launches == 1
        bx = 256 if M > 128 else 128
        tiles = -(-M // bx) * -(-N // 128)
        assert ctas == min(148, tiles)
        tail = tiles - (tiles // ctas) * ctas
        ksplit = bx == 256 and 0 < tail and 2 * tail <= ctas and -(-K // 128) >= 8
        want = 4096 * 4 * 4 + tail * 256 * 128 * 4 if ksplit else 0
        assert opq.workspace_size(M, N, K) == want
    assert opq.workspace_size(3072, 3840, 3840) == 65536 + 64 * 131072     # 360 tiles: 64 past 2 waves
    assert opq.workspace_size(512, 10240, 1024) == 65536 + 12 * 131072     # 160 tiles: 12 past 1 wave
    sz = ctypes.c_size_t(0)
    assert lib.opq_linear_workspace_size(0, 4, 32, ctypes.byref(sz)) == 1
    assert lib.opq_linear_workspace_size(4, 4, 40, ctypes.byref(sz)) == 2
    assert lib.opq_linear_workspace_size(4, 4, 32, None) == 1


def test_python_binding_refuses_cpu_tensors():
    import torch
    w = torch.zeros(4, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        opq.quantize(w)


def test_missing_library_fails_loudly(tmp_path):
    import importlib
    mod = importlib.import_module("bit_diffusion_transformer_b200")
    saved = mod._lib
    mod._lib = None
    try:
        with pytest.raises(ImportError):
            mod.load(str(tmp_path / "nope.so"))
    finally:
        mod._lib = saved
