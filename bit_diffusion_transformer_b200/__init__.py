"""Python binding of libopq.so: OPQ (Optimal Power Quantization) weights and the
linear layer that consumes them, on B200 (sm_100a).

The binding only marshals arguments: torch tensors provide device memory and the
current CUDA stream; every step runs in the library's kernels. There is no CPU
or PyTorch fallback: if ``libopq.so`` is missing or a tensor is not on a CUDA
device, the call raises.

Packed weight of W[N, K] (K % 32 == 0):
  codes  int32 [N, K/8]   element (n, 8j+i) is bits 4i..4i+3 of word j (4-bit magnitude)
  signs  int32 [N, K/32]  element (n, 32j+i) is bit i of word j (1 = negative)
  scales float32 [N]      max |w| of row n
(int32 tensors carry the uint32 words bit for bit.)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libopq.so")
ALPHA = 0.73

_STATUS = {0: "OPQ_OK", 1: "OPQ_ERR_INVALID_ARG", 2: "OPQ_ERR_UNSUPPORTED_SHAPE", 3: "OPQ_ERR_MISALIGNED",
           4: "OPQ_ERR_WORKSPACE", 5: "OPQ_ERR_CUDA", 6: "OPQ_ERR_NOT_DEVICE_MEMORY"}

EXPORTS = ["opq_quantize", "opq_dequantize", "opq_linear_workspace_size", "opq_linear", "opq_linear_plan",
           "opq_linear_noalloc", "opq_device_error", "opq_status_string", "opq_last_cuda_error",
           "opq_abi_version", "opq_quantize_grouped", "opq_dequantize_grouped",
           "opq_linear_grouped", "opq_linear_grouped_workspace_size", "opq_linear_fused",
           "opq_linear_grouped_fused", "opq_alpha_search", "opq_alpha_search_workspace_size",
           "opq_quantize_bits", "opq_dequantize_bits", "opq_set_wait_limit_ns",
           "opq_quantize_batched", "opq_linear_bits", "opq_linear_bits_workspace_size", "opq_dequantize_batched"]
ACTIVATIONS = {"none": 0, "silu": 1, "gelu_tanh": 2}
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class OPQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


_lib = None


def load(path: str = LIB_PATH):
    """Load libopq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libopq.so not found at {path}; build it with "
                          f"`python -m bit_diffusion_transformer_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.opq_quantize.argtypes = [P, I, I, I, F, P, P, P, P]
    lib.opq_dequantize.argtypes = [P, P, P, I, I, F, P, P]
    lib.opq_linear_workspace_size.argtypes = [I, I, I, ctypes.POINTER(S)]
    lib.opq_linear.argtypes = [P, I, I, P, P, P, I, F, P, P, S, P]
    lib.opq_linear_plan.argtypes = [I, I, I, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                    ctypes.POINTER(ctypes.c_int)]
    lib.opq_linear_noalloc.argtypes = [P, I, I, P, P, P, I, F, P, P]
    lib.opq_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.opq_quantize_grouped.argtypes = [P, I, I, I, I, F, P, P, P, P]
    lib.opq_dequantize_grouped.argtypes = [P, P, P, I, I, I, F, P, P]
    lib.opq_linear_grouped.argtypes = [P, I, I, P, P, P, I, I, F, P, P, S, P]
    lib.opq_linear_grouped_workspace_size.argtypes = [I, I, I, I, ctypes.POINTER(S)]
    lib.opq_alpha_search_workspace_size.argtypes = [I, ctypes.POINTER(S)]
    lib.opq_quantize_bits.argtypes = [P, I, I, I, ctypes.c_int32, F, P, P, P, P]
    lib.opq_dequantize_bits.argtypes = [P, P, P, I, I, ctypes.c_int32, F, P, P]
    lib.opq_alpha_search.argtypes = [P, I, I, I, I, P, ctypes.c_int32, P, P, P, S, P]
    lib.opq_linear_fused.argtypes = [P, I, I, P, P, P, I, F, P, ctypes.c_int, P, P, S, P]
    lib.opq_linear_grouped_fused.argtypes = [P, I, I, P, P, P, I, I, F, P, ctypes.c_int, P, P, S, P]
    lib.opq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.opq_quantize_batched.argtypes = [P, I, F, P]
    lib.opq_dequantize_batched.argtypes = [P, I, F, P]
    lib.opq_linear_bits.argtypes = [P, I, I, P, P, P, I, ctypes.c_int32, F, P, P, S, P]
    lib.opq_linear_bits_workspace_size.argtypes = [I, I, I, ctypes.c_int32, ctypes.POINTER(S)]
    lib.opq_status_string.argtypes = [ctypes.c_int]
    lib.opq_status_string.restype = ctypes.c_char_p
    for f in ("opq_quantize", "opq_dequantize", "opq_linear_workspace_size", "opq_linear", "opq_linear_plan",
              "opq_linear_noalloc", "opq_device_error", "opq_quantize_grouped", "opq_dequantize_grouped", "opq_linear_grouped",
              "opq_linear_grouped_workspace_size", "opq_linear_fused", "opq_linear_grouped_fused",
              "opq_alpha_search", "opq_alpha_search_workspace_size", "opq_quantize_bits", "opq_dequantize_bits",
              "opq_set_wait_limit_ns", "opq_quantize_batched", "opq_linear_bits", "opq_linear_bits_workspace_size",
              "opq_dequantize_batched"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise OPQError(status, where)


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("opq: tensors must be on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("opq: tensors must be contiguous")


def quantize(w: torch.Tensor, alpha: float = ALPHA, out=None):
    """OPQ-quantize bf16 W[N, K] -> (codes, signs, scales)."""
    assert w.dtype == torch.bfloat16 and w.dim() == 2
    _need_cuda(w)
    N, K = w.shape
    if out is None:
        codes = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
        signs = torch.empty((N, K // 32), dtype=torch.int32, device=w.device)
        scales = torch.empty((N,), dtype=torch.float32, device=w.device)
    else:
        codes, signs, scales = out
    _check(load().opq_quantize(_ptr(w), N, K, K, float(alpha), _ptr(codes), _ptr(signs), _ptr(scales),
                               _stream(w.device)), "opq_quantize")
    return codes, signs, scales


class QuantJob(ctypes.Structure):
    """One matrix of opq_quantize_batched (the C struct opq_quant_job)."""
    _fields_ = [("w", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("ldw", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


def quantize_jobs(ws, outs, alpha: float = ALPHA):
    """The descriptor array of opq_quantize_batched for bf16 weights ``ws`` and their
    output planes ``outs`` [(codes, signs, scales), ...] (built once, reusable)."""
    assert len(ws) == len(outs) and len(ws) > 0
    arr = (QuantJob * len(ws))()
    for i, (w, (c, s, f)) in enumerate(zip(ws, outs)):
        assert w.dtype == torch.bfloat16 and w.dim() == 2
        _need_cuda(w, c, s, f)
        N, K = w.shape
        arr[i] = QuantJob(w.data_ptr(), N, K, K, c.data_ptr(), s.data_ptr(), f.data_ptr())
    return arr


def quantize_batched(ws, alpha: float = ALPHA, outs=None, jobs=None):
    """OPQ-quantize a list of bf16 matrices in one pass -> [(codes, signs, scales), ...].
    ``jobs`` (from quantize_jobs) skips rebuilding the descriptors for the same buffers."""
    if outs is None:
        outs = [(torch.empty((w.shape[0], w.shape[1] // 8), dtype=torch.int32, device=w.device),
                 torch.empty((w.shape[0], w.shape[1] // 32), dtype=torch.int32, device=w.device),
                 torch.empty((w.shape[0],), dtype=torch.float32, device=w.device)) for w in ws]
    if jobs is None:
        jobs = quantize_jobs(ws, outs, alpha)
    _check(load().opq_quantize_batched(ctypes.cast(jobs, ctypes.c_void_p), len(jobs), float(alpha),
                                       _stream(ws[0].device)), "opq_quantize_batched")
    return outs


def dequantize(codes: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor, alpha: float = ALPHA, out=None):
    """Packed planes -> bf16 W'[N, K]."""
    _need_cuda(codes, signs, scales)
    N, cw = codes.shape
    K = cw * 8
    w = out if out is not None else torch.empty((N, K), dtype=torch.bfloat16, device=codes.device)
    _check(load().opq_dequantize(_ptr(codes), _ptr(signs), _ptr(scales), N, K, float(alpha), _ptr(w),
                                 _stream(codes.device)), "opq_dequantize")
    return w


class DequantJob(ctypes.Structure):
    """One matrix of opq_dequantize_batched (the C struct opq_dequant_job)."""
    _fields_ = [("codes", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("w_out", ctypes.c_void_p)]


def dequantize_jobs(planes, outs):
    """The descriptor array of opq_dequantize_batched for packed weights ``planes``
    [(codes, signs, scales), ...] and their bf16 outputs ``outs`` (built once, reusable)."""
    assert len(planes) == len(outs) and len(planes) > 0
    arr = (DequantJob * len(planes))()
    for i, ((c, s, f), w) in enumerate(zip(planes, outs)):
        _need_cuda(c, s, f, w)
        N, cw = c.shape
        assert w.dtype == torch.bfloat16 and tuple(w.shape) == (N, cw * 8)
        arr[i] = DequantJob(c.data_ptr(), s.data_ptr(), f.data_ptr(), N, cw * 8, w.data_ptr())
    return arr


def dequantize_batched(planes, alpha: float = ALPHA, outs=None, jobs=None):
    """Decode a list of packed weights in one pass -> [bf16 W', ...]. ``jobs`` (from
    dequantize_jobs) skips rebuilding the descriptors for the same buffers."""
    if outs is None:
        outs = [torch.empty((c.shape[0], c.shape[1] * 8), dtype=torch.bfloat16, device=c.device) for c, _, _ in planes]
    if jobs is None:
        jobs = dequantize_jobs(planes, outs)
    _check(load().opq_dequantize_batched(ctypes.cast(jobs, ctypes.c_void_p), len(jobs), float(alpha),
                                         _stream(planes[0][0].device)), "opq_dequantize_batched")
    return outs


def quantize_grouped(w: torch.Tensor, group_size: int = 128, alpha: float = ALPHA, out=None):
    """Group-wise OPQ of bf16 W[N, K] -> (codes, signs, gmax float16 [N, K/group_size])."""
    assert w.dtype == torch.bfloat16 and w.dim() == 2
    _need_cuda(w)
    N, K = w.shape
    if out is None:
        codes = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
        signs = torch.empty((N, K // 32), dtype=torch.int32, device=w.device)
        gmax = torch.empty((N, K // group_size), dtype=torch.float16, device=w.device)
    else:
        codes, signs, gmax = out
    _check(load().opq_quantize_grouped(_ptr(w), N, K, K, int(group_size), float(alpha), _ptr(codes), _ptr(signs),
                                       _ptr(gmax), _stream(w.device)), "opq_quantize_grouped")
    return codes, signs, gmax


def dequantize_grouped(codes: torch.Tensor, signs: torch.Tensor, gmax: torch.Tensor, alpha: float = ALPHA,
                       out=None):
    """Group-wise packed planes -> bf16 W'[N, K] (the group size is K / gmax.shape[1])."""
    _need_cuda(codes, signs, gmax)
    N, cw = codes.shape
    K = cw * 8
    gs = K // gmax.shape[1]
    w = out if out is not None else torch.empty((N, K), dtype=torch.bfloat16, device=codes.device)
    _check(load().opq_dequantize_grouped(_ptr(codes), _ptr(signs), _ptr(gmax), N, K, gs, float(alpha), _ptr(w),
                                         _stream(codes.device)), "opq_dequantize_grouped")
    return w


def grouped_workspace_size(M: int, N: int, K: int, group_size: int) -> int:
    b = ctypes.c_size_t(0)
    _check(load().opq_linear_grouped_workspace_size(M, N, K, int(group_size), ctypes.byref(b)),
           "opq_linear_grouped_workspace_size")
    return int(b.value)


def linear_grouped(x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor, gmax: torch.Tensor,
                   alpha: float = ALPHA, out=None, workspace=None):
    """y = x @ W'^T for bf16 x[M, K] and a group-wise packed W[N, K] -> bf16 y[M, N]."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    _need_cuda(x, codes, signs, gmax)
    M, K = x.shape
    N = codes.shape[0]
    gs = K // gmax.shape[1]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = grouped_workspace_size(M, N, K, gs)
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=x.device)   # must start zeroed
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().opq_linear_grouped(_ptr(x), M, K, _ptr(codes), _ptr(signs), _ptr(gmax), N, gs, float(alpha),
                                     _ptr(y), ws_ptr, ws_bytes, _stream(x.device)), "opq_linear_grouped")
    return y


def _workspace(need: int, workspace, device):
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=device)   # must start zeroed
    ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return workspace, ptr, nbytes


def linear_fused(x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor,
                 alpha: float = ALPHA, bias: torch.Tensor | None = None, act: str = "none", out=None,
                 workspace=None):
    """y = act(x @ W'^T + bias) (the nn.Linear a OPQLinear replaces, with the activation that follows)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    _need_cuda(x, codes, signs, scales)
    if bias is not None:
        assert bias.dtype == torch.bfloat16
        _need_cuda(bias)
    M, K = x.shape
    N = codes.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    workspace, ws_ptr, ws_bytes = _workspace(workspace_size(M, N, K), workspace, x.device)
    _check(load().opq_linear_fused(_ptr(x), M, K, _ptr(codes), _ptr(signs), _ptr(scales), N, float(alpha),
                                   _ptr(bias) if bias is not None else ctypes.c_void_p(0), ACTIVATIONS[act],
                                   _ptr(y), ws_ptr, ws_bytes, _stream(x.device)), "opq_linear_fused")
    return y


def linear_grouped_fused(x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor, gmax: torch.Tensor,
                         alpha: float = ALPHA, bias: torch.Tensor | None = None, act: str = "none", out=None,
                         workspace=None):
    """y = act(x @ W'^T + bias) for a group-wise packed W."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    _need_cuda(x, codes, signs, gmax)
    if bias is not None:
        assert bias.dtype == torch.bfloat16
        _need_cuda(bias)
    M, K = x.shape
    N = codes.shape[0]
    gs = K // gmax.shape[1]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    workspace, ws_ptr, ws_bytes = _workspace(grouped_workspace_size(M, N, K, gs), workspace, x.device)
    _check(load().opq_linear_grouped_fused(_ptr(x), M, K, _ptr(codes), _ptr(signs), _ptr(gmax), N, gs,
                                           float(alpha), _ptr(bias) if bias is not None else ctypes.c_void_p(0),
                                           ACTIVATIONS[act], _ptr(y), ws_ptr, ws_bytes, _stream(x.device)),
           "opq_linear_grouped_fused")
    return y


def quantize_bits(w: torch.Tensor, bits: int, alpha: float = ALPHA, out=None):
    """Per-row OPQ with `bits`-bit magnitudes (3..6) -> (codes int32 [N, K*bits/32], signs, scales)."""
    assert w.dtype == torch.bfloat16 and w.dim() == 2
    _need_cuda(w)
    N, K = w.shape
    if out is None:
        codes = torch.empty((N, K * bits // 32), dtype=torch.int32, device=w.device)
        signs = torch.empty((N, K // 32), dtype=torch.int32, device=w.device)
        scales = torch.empty((N,), dtype=torch.float32, device=w.device)
    else:
        codes, signs, scales = out
    _check(load().opq_quantize_bits(_ptr(w), N, K, K, int(bits), float(alpha), _ptr(codes), _ptr(signs), _ptr(scales),
                                    _stream(w.device)), "opq_quantize_bits")
    return codes, signs, scales


def dequantize_bits(codes: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor, bits: int, alpha: float = ALPHA,
                    out=None):
    """`bits`-bit packed planes -> bf16 W'[N, K]."""
    _need_cuda(codes, signs, scales)
    N = codes.shape[0]
    K = codes.shape[1] * 32 // bits
    w = out if out is not None else torch.empty((N, K), dtype=torch.bfloat16, device=codes.device)
    _check(load().opq_dequantize_bits(_ptr(codes), _ptr(signs), _ptr(scales), N, K, int(bits), float(alpha), _ptr(w),
                                      _stream(codes.device)), "opq_dequantize_bits")
    return w


def bits_workspace_size(M: int, N: int, K: int, bits: int) -> int:
    b = ctypes.c_size_t(0)
    _check(load().opq_linear_bits_workspace_size(M, N, K, int(bits), ctypes.byref(b)), "opq_linear_bits_workspace_size")
    return int(b.value)


def linear_bits(x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor, bits: int,
                alpha: float = ALPHA, out=None, workspace=None):
    """y = x @ W'^T for a W[N, K] packed with `bits`-bit magnitudes (3..6, codes int32 [N, K*bits/32])."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    _need_cuda(x, codes, signs, scales)
    M, K = x.shape
    N = codes.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = bits_workspace_size(M, N, K, bits)
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=x.device)   # must start zeroed
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().opq_linear_bits(_ptr(x), M, K, _ptr(codes), _ptr(signs), _ptr(scales), N, int(bits), float(alpha),
                                  _ptr(y), ws_ptr, ws_bytes, _stream(x.device)), "opq_linear_bits")
    return y


ALPHA_GRID = tuple(round(0.30 + 0.05 * i, 2) for i in range(15))   # 0.30 .. 1.00


def alpha_search(w: torch.Tensor, alphas=ALPHA_GRID, group_size: int = 0):
    """SNR (dB) of OPQ at each alpha for bf16 W[N, K] (per-row format, or group-wise when
    group_size > 0) -> (best alpha, [snr_db per alpha])."""
    import numpy as np
    assert w.dtype == torch.bfloat16 and w.dim() == 2
    _need_cuda(w)
    N, K = w.shape
    b = ctypes.c_size_t(0)
    _check(load().opq_alpha_search_workspace_size(N, ctypes.byref(b)), "opq_alpha_search_workspace_size")
    ws = torch.empty((b.value,), dtype=torch.uint8, device=w.device)
    a = np.ascontiguousarray(alphas, dtype=np.float32)
    snr = np.zeros(a.shape, dtype=np.float64)
    best = ctypes.c_float(0.0)
    _check(load().opq_alpha_search(_ptr(w), N, K, K, int(group_size), a.ctypes.data_as(ctypes.c_void_p), a.size,
                                   snr.ctypes.data_as(ctypes.c_void_p), ctypes.byref(best), _ptr(ws), b.value,
                                   _stream(w.device)), "opq_alpha_search")
    i = int(np.argmax(snr))            # the first largest, as the library picks it
    assert float(np.float32(alphas[i])) == best.value
    return alphas[i], snr.tolist()


def workspace_size(M: int, N: int, K: int) -> int:
    b = ctypes.c_size_t(0)
    _check(load().opq_linear_workspace_size(M, N, K, ctypes.byref(b)), "opq_linear_workspace_size")
    return int(b.value)


def plan(M: int, N: int, K: int):
    """(path, splits, launches) that opq_linear uses for this shape."""
    p, s, l = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(load().opq_linear_plan(M, N, K, ctypes.byref(p), ctypes.byref(s), ctypes.byref(l)), "opq_linear_plan")
    return p.value, s.value, l.value


def linear(x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor,
           alpha: float = ALPHA, out=None, workspace=None):
    """y = x @ W'^T for bf16 x[M, K] and a packed W[N, K] -> bf16 y[M, N].

    ``workspace`` (uint8 device tensor of at least workspace_size(M, N, K) bytes)
    must be zero-filled before its first use; every call leaves it reusable."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    _need_cuda(x, codes, signs, scales)
    M, K = x.shape
    N = codes.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = workspace_size(M, N, K)
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=x.device)   # must start zeroed
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().opq_linear(_ptr(x), M, K, _ptr(codes), _ptr(signs), _ptr(scales), N, float(alpha), _ptr(y),
                             ws_ptr, ws_bytes, _stream(x.device)), "opq_linear")
    return y


def linear_noalloc(x: torch.Tensor, codes: torch.Tensor, signs: torch.Tensor, scales: torch.Tensor,
                   alpha: float = ALPHA, out=None):
    """y = x @ W'^T without a caller workspace: split-K partial sums use the library's
    static 16 MiB device array (for callers that cannot allocate device memory).
    Calls that overlap on the GPU race on that array; shapes needing more scratch raise."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    _need_cuda(x, codes, signs, scales)
    M, K = x.shape
    N = codes.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(load().opq_linear_noalloc(_ptr(x), M, K, _ptr(codes), _ptr(signs), _ptr(scales), N, float(alpha),
                                     _ptr(y), _stream(x.device)), "opq_linear_noalloc")
    return y


DEVERR_WAIT_TIMEOUT = 1
DEVERR_SMEM_ALIGN = 2


def device_error(device=None) -> int:
    """Read and clear the library's device-side error word (synchronises the current stream)."""
    v = ctypes.c_uint32(0)
    _check(load().opq_device_error(_stream(device), ctypes.byref(v)), "opq_device_error")
    return int(v.value)


def set_wait_limit_ns(ns: int = 0):
    """Time after which the kernels' bounded waits give up on the current device (0: the 4 s default)."""
    _check(load().opq_set_wait_limit_ns(int(ns)), "opq_set_wait_limit_ns")
