"""ctypes front end of the fp64 OPQ oracle (``opq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The CUDA library never
imports this package and shares no code with it.

All array arguments are numpy arrays; bf16 tensors travel as their uint16 bit
patterns. The shared object is built on first use with gcc (``build()``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "opq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle (plain C99, -O2, OpenMP over rows, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int64
    D = ctypes.c_double
    lib.oracle_quantize.argtypes = [P, I, I, I, D, P, P, P, P, P]
    lib.oracle_quantize.restype = None
    lib.oracle_dequantize_f64.argtypes = [P, P, P, I, I, D, P]
    lib.oracle_dequantize_bf16.argtypes = [P, P, P, I, I, D, P]
    lib.oracle_linear.argtypes = [P, I, I, P, P, P, I, D, P, P]
    lib.oracle_linear_pairs.argtypes = [P, I, I, P, P, P, I, D, I, P, P, P, P]
    lib.oracle_snr_db.argtypes = [P, P, I]
    lib.oracle_snr_db.restype = D
    lib.oracle_uniform_int4.argtypes = [P, I, I, P]
    lib.oracle_double_to_bf16.argtypes = [D]
    lib.oracle_double_to_bf16.restype = ctypes.c_uint16
    lib.oracle_quantize_grouped.argtypes = [P, I, I, I, I, D, P, P, P, P, P]
    lib.oracle_quantize_grouped.restype = None
    lib.oracle_dequantize_grouped_f64.argtypes = [P, P, P, I, I, I, D, P]
    lib.oracle_dequantize_grouped_bf16.argtypes = [P, P, P, I, I, I, D, P]
    lib.oracle_linear_grouped.argtypes = [P, I, I, P, P, P, I, I, D, P, P]
    lib.oracle_linear_grouped_pairs.argtypes = [P, I, I, P, P, P, I, I, D, I, P, P, P, P]
    lib.oracle_fp16_value.argtypes = [ctypes.c_uint16]
    lib.oracle_fp16_value.restype = D
    lib.oracle_fp16_from_nonneg.argtypes = [D]
    lib.oracle_fp16_from_nonneg.restype = ctypes.c_uint16
    lib.oracle_quantize_bits.argtypes = [P, I, I, I, ctypes.c_int, D, P, P, P, P, P]
    lib.oracle_quantize_bits.restype = None
    lib.oracle_dequantize_bits_f64.argtypes = [P, P, P, I, I, ctypes.c_int, D, P]
    lib.oracle_dequantize_bits_bf16.argtypes = [P, P, P, I, I, ctypes.c_int, D, P]
    lib.oracle_apply_epilogue.argtypes = [P, I, I, P, ctypes.c_int]
    lib.oracle_apply_epilogue.restype = None
    lib.oracle_rounding_mode_ok.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 bit patterns."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16
            return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16
    return a


class Oracle:
    """The oracle's entry points bound to one compiled shared object."""

    def __init__(self, so_path: str):
        self._lib = _bind(so_path)
        self.path = so_path

    def quantize(self, w, alpha: float, want_ties: bool = False, want_v15: bool = False):
        """OPQ-quantize bf16 W[N, K] row by row.

        Returns dict(codes uint32[N, K/8], signs uint32[N, K/32], scales float32[N],
        near_tie uint8[N, K] | None, v15 float64[N, K] | None).
        """
        w = _u16(w)
        N, K = w.shape
        assert K % 32 == 0
        lib = self._lib
        assert lib.oracle_rounding_mode_ok() == 1
        codes = np.zeros((N, K // 8), np.uint32)
        signs = np.zeros((N, K // 32), np.uint32)
        scales = np.zeros((N,), np.float32)
        ties = np.zeros((N, K), np.uint8) if want_ties else None
        v15 = np.zeros((N, K), np.float64) if want_v15 else None
        lib.oracle_quantize(_p(w), N, K, K, float(alpha), _p(codes), _p(signs), _p(scales),
                            _p(ties) if ties is not None else None,
                            _p(v15) if v15 is not None else None)
        return dict(codes=codes, signs=signs, scales=scales, near_tie=ties, v15=v15)

    def dequantize_f64(self, codes, signs, scales, alpha: float) -> np.ndarray:
        codes = np.ascontiguousarray(codes, np.uint32)
        signs = np.ascontiguousarray(signs, np.uint32)
        scales = np.ascontiguousarray(scales, np.float32)
        N, cw = codes.shape
        K = cw * 8
        out = np.zeros((N, K), np.float64)
        self._lib.oracle_dequantize_f64(_p(codes), _p(signs), _p(scales), N, K, float(alpha), _p(out))
        return out

    def dequantize_bf16(self, codes, signs, scales, alpha: float) -> np.ndarray:
        """Returns uint16 bf16 bit patterns [N, K]."""
        codes = np.ascontiguousarray(codes, np.uint32)
        signs = np.ascontiguousarray(signs, np.uint32)
        scales = np.ascontiguousarray(scales, np.float32)
        N, cw = codes.shape
        K = cw * 8
        out = np.zeros((N, K), np.uint16)
        self._lib.oracle_dequantize_bf16(_p(codes), _p(signs), _p(scales), N, K, float(alpha), _p(out))
        return out

    def linear(self, x, codes, signs, scales, alpha: float):
        """y = x @ W'^T in fp64 with its error bound B = |x| @ |W'|^T. Returns (y, B)."""
        x = _u16(x)
        M, K = x.shape
        codes = np.ascontiguousarray(codes, np.uint32)
        signs = np.ascontiguousarray(signs, np.uint32)
        scales = np.ascontiguousarray(scales, np.float32)
        N = codes.shape[0]
        assert codes.shape[1] * 8 == K
        y = np.zeros((M, N), np.float64)
        b = np.zeros((M, N), np.float64)
        self._lib.oracle_linear(_p(x), M, K, _p(codes), _p(signs), _p(scales), N, float(alpha), _p(y), _p(b))
        return y, b

    def linear_pairs(self, x, codes, signs, scales, alpha: float, ms, ns):
        """y[m_i, n_i] and B[m_i, n_i] for the listed output positions."""
        x = _u16(x)
        M, K = x.shape
        codes = np.ascontiguousarray(codes, np.uint32)
        signs = np.ascontiguousarray(signs, np.uint32)
        scales = np.ascontiguousarray(scales, np.float32)
        N = codes.shape[0]
        ms = np.ascontiguousarray(ms, np.int64)
        ns = np.ascontiguousarray(ns, np.int64)
        assert ms.shape == ns.shape
        assert (ms >= 0).all() and (ms < M).all() and (ns >= 0).all() and (ns < N).all()
        y = np.zeros(ms.shape, np.float64)
        b = np.zeros(ms.shape, np.float64)
        self._lib.oracle_linear_pairs(_p(x), M, K, _p(codes), _p(signs), _p(scales), N, float(alpha),
                                    ms.size, _p(ms), _p(ns), _p(y), _p(b))
        return y, b

    # ---- group-wise variant: one float16 max per GS consecutive weights of a row ----
    def quantize_grouped(self, w, gs: int, alpha: float, want_ties: bool = False, want_v15: bool = False):
        """OPQ-quantize bf16 W[N, K] group by group (GS weights per group along K).

        Returns dict(codes uint32[N, K/8], signs uint32[N, K/32], gmax uint16[N, K/GS] (float16
        bits), near_tie uint8[N, K] | None, v15 float64[N, K] | None).
        """
        w = _u16(w)
        N, K = w.shape
        assert K % 32 == 0 and K % gs == 0
        lib = self._lib
        assert lib.oracle_rounding_mode_ok() == 1
        codes = np.zeros((N, K // 8), np.uint32)
        signs = np.zeros((N, K // 32), np.uint32)
        gmax = np.zeros((N, K // gs), np.uint16)
        ties = np.zeros((N, K), np.uint8) if want_ties else None
        v15 = np.zeros((N, K), np.float64) if want_v15 else None
        lib.oracle_quantize_grouped(_p(w), N, K, K, int(gs), float(alpha), _p(codes), _p(signs), _p(gmax),
                                    _p(ties) if ties is not None else None,
                                    _p(v15) if v15 is not None else None)
        return dict(codes=codes, signs=signs, gmax=gmax, near_tie=ties, v15=v15)

    def _grouped_planes(self, codes, signs, gmax):
        codes = np.ascontiguousarray(codes, np.uint32)
        signs = np.ascontiguousarray(signs, np.uint32)
        gmax = np.ascontiguousarray(gmax, np.uint16)
        N, cw = codes.shape
        K = cw * 8
        assert gmax.shape[0] == N and K % gmax.shape[1] == 0
        return codes, signs, gmax, N, K, K // gmax.shape[1]

    def dequantize_grouped_f64(self, codes, signs, gmax, alpha: float) -> np.ndarray:
        codes, signs, gmax, N, K, gs = self._grouped_planes(codes, signs, gmax)
        out = np.zeros((N, K), np.float64)
        self._lib.oracle_dequantize_grouped_f64(_p(codes), _p(signs), _p(gmax), N, K, gs, float(alpha), _p(out))
        return out

    def dequantize_grouped_bf16(self, codes, signs, gmax, alpha: float) -> np.ndarray:
        """Returns uint16 bf16 bit patterns [N, K]."""
        codes, signs, gmax, N, K, gs = self._grouped_planes(codes, signs, gmax)
        out = np.zeros((N, K), np.uint16)
        self._lib.oracle_dequantize_grouped_bf16(_p(codes), _p(signs), _p(gmax), N, K, gs, float(alpha), _p(out))
        return out

    def linear_grouped(self, x, codes, signs, gmax, alpha: float):
        """y = x @ W'^T in fp64 with its error bound B = |x| @ |W'|^T. Returns (y, B)."""
        x = _u16(x)
        M, K = x.shape
        codes, signs, gmax, N, Kc, gs = self._grouped_planes(codes, signs, gmax)
        assert Kc == K
        y = np.zeros((M, N), np.float64)
        b = np.zeros((M, N), np.float64)
        self._lib.oracle_linear_grouped(_p(x), M, K, _p(codes), _p(signs), _p(gmax), N, gs, float(alpha),
                                        _p(y), _p(b))
        return y, b

    def linear_grouped_pairs(self, x, codes, signs, gmax, alpha: float, ms, ns):
        x = _u16(x)
        M, K = x.shape
        codes, signs, gmax, N, Kc, gs = self._grouped_planes(codes, signs, gmax)
        assert Kc == K
        ms = np.ascontiguousarray(ms, np.int64)
        ns = np.ascontiguousarray(ns, np.int64)
        assert ms.shape == ns.shape
        assert (ms >= 0).all() and (ms < M).all() and (ns >= 0).all() and (ns < N).all()
        y = np.zeros(ms.shape, np.float64)
        b = np.zeros(ms.shape, np.float64)
        self._lib.oracle_linear_grouped_pairs(_p(x), M, K, _p(codes), _p(signs), _p(gmax), N, gs, float(alpha),
                                              ms.size, _p(ms), _p(ns), _p(y), _p(b))
        return y, b

    # ---- other bit widths: 2^bits - 1 levels, codes as one little-endian bit stream per row ----
    def quantize_bits(self, w, bits: int, alpha: float, want_ties: bool = False, want_v: bool = False):
        """Per-row OPQ with `bits`-bit magnitudes. Returns dict(codes uint32[N, K bits/32], signs,
        scales, near_tie, v) as quantize does (v = L u^alpha)."""
        w = _u16(w)
        N, K = w.shape
        assert K % 32 == 0 and bits in (3, 4, 5, 6)
        lib = self._lib
        assert lib.oracle_rounding_mode_ok() == 1
        codes = np.zeros((N, K * bits // 32), np.uint32)
        signs = np.zeros((N, K // 32), np.uint32)
        scales = np.zeros((N,), np.float32)
        ties = np.zeros((N, K), np.uint8) if want_ties else None
        v = np.zeros((N, K), np.float64) if want_v else None
        lib.oracle_quantize_bits(_p(w), N, K, K, int(bits), float(alpha), _p(codes), _p(signs), _p(scales),
                                 _p(ties) if ties is not None else None, _p(v) if v is not None else None)
        return dict(codes=codes, signs=signs, scales=scales, near_tie=ties, v=v)

    def _bits_planes(self, codes, signs, scales, bits):
        codes = np.ascontiguousarray(codes, np.uint32)
        signs = np.ascontiguousarray(signs, np.uint32)
        scales = np.ascontiguousarray(scales, np.float32)
        N = codes.shape[0]
        K = codes.shape[1] * 32 // bits
        return codes, signs, scales, N, K

    def dequantize_bits_f64(self, codes, signs, scales, bits: int, alpha: float) -> np.ndarray:
        codes, signs, scales, N, K = self._bits_planes(codes, signs, scales, bits)
        out = np.zeros((N, K), np.float64)
        self._lib.oracle_dequantize_bits_f64(_p(codes), _p(signs), _p(scales), N, K, int(bits), float(alpha), _p(out))
        return out

    def dequantize_bits_bf16(self, codes, signs, scales, bits: int, alpha: float) -> np.ndarray:
        codes, signs, scales, N, K = self._bits_planes(codes, signs, scales, bits)
        out = np.zeros((N, K), np.uint16)
        self._lib.oracle_dequantize_bits_bf16(_p(codes), _p(signs), _p(scales), N, K, int(bits), float(alpha), _p(out))
        return out

    def apply_epilogue(self, y: np.ndarray, bias=None, act: int = 0) -> np.ndarray:
        """act(y + bias[n]) on a copy of y[M, N] (fp64); bias as bf16 bits [N] or None;
        act 0 none, 1 SiLU, 2 GELU (tanh form)."""
        y = np.array(y, dtype=np.float64, order="C", copy=True)
        M, N = y.shape
        b = None if bias is None else _u16(bias)
        assert b is None or b.shape == (N,)
        self._lib.oracle_apply_epilogue(_p(y), M, N, _p(b) if b is not None else None, int(act))
        return y

    def fp16_value(self, bits: int) -> float:
        return float(self._lib.oracle_fp16_value(int(bits)))

    def fp16_from_nonneg(self, v: float) -> int:
        return int(self._lib.oracle_fp16_from_nonneg(float(v)))

    def snr_db(self, w, w_rec: np.ndarray) -> float:
        w = _u16(w)
        w_rec = np.ascontiguousarray(w_rec, np.float64)
        assert w.size == w_rec.size
        return float(self._lib.oracle_snr_db(_p(w), _p(w_rec), w.size))

    def uniform_int4(self, w) -> np.ndarray:
        w = _u16(w)
        N, K = w.shape
        out = np.zeros((N, K), np.float64)
        self._lib.oracle_uniform_int4(_p(w), N, K, _p(out))
        return out

    def num_threads(self) -> int:
        """OpenMP threads the oracle's loops run on."""
        return int(self._lib.oracle_num_threads())

    def double_to_bf16(self, v: float) -> int:
        return int(self._lib.oracle_double_to_bf16(float(v)))


_default = None


def default() -> Oracle:
    """The oracle built from ``opq_oracle.c`` (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def quantize(*a, **k):
    return default().quantize(*a, **k)


def dequantize_f64(*a, **k):
    return default().dequantize_f64(*a, **k)


def dequantize_bf16(*a, **k):
    return default().dequantize_bf16(*a, **k)


def linear(*a, **k):
    return default().linear(*a, **k)


def linear_pairs(*a, **k):
    return default().linear_pairs(*a, **k)


def snr_db(*a, **k):
    return default().snr_db(*a, **k)


def quantize_grouped(*a, **k):
    return default().quantize_grouped(*a, **k)


def dequantize_grouped_f64(*a, **k):
    return default().dequantize_grouped_f64(*a, **k)


def dequantize_grouped_bf16(*a, **k):
    return default().dequantize_grouped_bf16(*a, **k)


def linear_grouped(*a, **k):
    return default().linear_grouped(*a, **k)


def linear_grouped_pairs(*a, **k):
    return default().linear_grouped_pairs(*a, **k)


def fp16_value(*a, **k):
    return default().fp16_value(*a, **k)


def alpha_search(w, alphas, group_size: int = 0):
    """SNR (dB) of the oracle's OPQ at each alpha: quantize, decode (unrounded fp64), SNR against
    the bf16 weights -> (first alpha with the largest SNR, [snr per alpha])."""
    o = default()
    snr = []
    for a in alphas:
        if group_size:
            r = o.quantize_grouped(w, group_size, float(a))
            rec = o.dequantize_grouped_f64(r["codes"], r["signs"], r["gmax"], float(a))
        else:
            r = o.quantize(w, float(a))
            rec = o.dequantize_f64(r["codes"], r["signs"], r["scales"], float(a))
        snr.append(o.snr_db(w, rec))
    best = max(range(len(snr)), key=lambda i: (snr[i], -i))
    return float(alphas[best]), snr


def apply_epilogue(*a, **k):
    return default().apply_epilogue(*a, **k)


def quantize_bits(*a, **k):
    return default().quantize_bits(*a, **k)


def dequantize_bits_f64(*a, **k):
    return default().dequantize_bits_f64(*a, **k)


def dequantize_bits_bf16(*a, **k):
    return default().dequantize_bits_bf16(*a, **k)


def fp16_from_nonneg(*a, **k):
    return default().fp16_from_nonneg(*a, **k)


def uniform_int4(*a, **k):
    return default().uniform_int4(*a, **k)


def num_threads() -> int:
    return default().num_threads()


def double_to_bf16(*a, **k):
    return default().double_to_bf16(*a, **k)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (a plain reinterpretation, no arithmetic)."""
    bits = np.ascontiguousarray(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
