"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Rules, from the acceptance criteria of the method's contract:
  * codes and signs bit-exact, except entries whose oracle 15 u^alpha lies within
    1e-6 of a .5 tie; mismatches there are counted and must stay under 1e-6 of
    all entries (mismatches anywhere else: none);
  * scales bit-exact; dequantized bf16 bit-exact (both sides form the fp64
    product and round once);
  * linear: |y - y_ref| <= 1e-2 * (|x| |W'|^T) + 1e-3 elementwise.
The oracle's inputs never come from the CUDA path: weights and activations are
drawn by ``workloads`` and the packed weights fed to the GPU linear and
dequantize are the oracle's own.
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from oracle_pins import unpack_codes, unpack_signs, bits_to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
TIE_FRACTION_LIMIT = 1e-6


def alpha32(alpha: float) -> float:
    """The alpha a call receives: the C ABI passes it as float32, so bit-exact comparisons
    evaluate the oracle at that value."""
    return float(np.float32(alpha))


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def to_dev_u32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)


def guarded(shape, dtype, fill):
    """A device tensor with 4 KiB canary regions on both sides (checked by check_guards)."""
    n = int(np.prod(shape))
    esz = torch.empty(0, dtype=dtype).element_size()
    pad = 4096 // esz
    buf = torch.empty(n + 2 * pad, dtype=dtype, device=DEV)
    buf.view(torch.uint8).fill_(fill)
    return buf, buf[pad:pad + n].view(shape), pad


def check_guards(buf, pad, fill):
    b = buf.view(torch.uint8)
    esz = buf.element_size()
    head = b[: pad * esz]
    tail = b[b.numel() - pad * esz:]
    assert bool((head == fill).all()) and bool((tail == fill).all()), "write outside the output tensor"


def no_device_error():
    assert opq.device_error() == 0


# ------------------------------------------------------------------ quantize --
def quant_parity(w: torch.Tensor, alpha: float, rows=None):
    """GPU quantize of all of w; oracle on `rows` (default all). Returns (gpu planes, oracle dict)."""
    N, K = w.shape
    cb, codes, cpad = guarded((N, K // 8), torch.int32, 0xA5)
    sb, signs, spad = guarded((N, K // 32), torch.int32, 0x5A)
    fb, scales, fpad = guarded((N,), torch.float32, 0x3C)
    opq.quantize(w, alpha, out=(codes, signs, scales))
    torch.cuda.synchronize()
    check_guards(cb, cpad, 0xA5)
    check_guards(sb, spad, 0x5A)
    check_guards(fb, fpad, 0x3C)
    no_device_error()
    wc = w if rows is None else w[torch.as_tensor(rows, device=w.device)]
    ref = oracle.quantize(wc, alpha32(alpha), want_ties=True)
    sel = slice(None) if rows is None else np.asarray(rows)
    g_scales = u32(scales.view(torch.int32))[sel]
    assert np.array_equal(g_scales, ref["scales"].view(np.uint32)), "scales differ"
    g_signs = u32(signs)[sel]
    assert np.array_equal(g_signs, ref["signs"]), "signs differ"
    qg = unpack_codes(u32(codes)[sel])
    qo = unpack_codes(ref["codes"])
    mism = qg != qo
    near = ref["near_tie"].astype(bool)
    assert int((mism & ~near).sum()) == 0, f"{int((mism & ~near).sum())} code mismatches away from ties"
    in_band = int((mism & near).sum())
    assert in_band <= TIE_FRACTION_LIMIT * qo.size, f"{in_band} mismatches in the tie band"
    return (codes, signs, scales), ref


@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_quantize_tiny(alpha):
    w = workloads.tiny().make_weights(DEV)
    quant_parity(w, alpha)


@pytest.mark.parametrize("N,K", [(1, 32), (3, 96), (37, 512), (129, 4096), (5, 4128), (9, 10240),
                                 (2, 32768), (300, 3840)])
def test_quantize_shapes(N, K):
    lin = workloads.Linear("shape", 1, N, K, w_seed=N * 131 + K)
    quant_parity(lin.make_weights(DEV), 0.73)


@pytest.mark.parametrize("alpha", [0.1, 0.2, 0.3, 3.0])
@pytest.mark.parametrize("N,K", [(40, 3840), (3, 10240)])
def test_quantize_alpha_range(alpha, N, K):
    # a row's code table covers bits(max) - bits(|w|) up to 4095: alpha 0.2 and 0.3 fill
    # most of it, alpha 0.1 needs more (those rows take the threshold search instead),
    # alpha 3 crowds the levels near the max; one warp per row (K = 3840) and eight (10240)
    lin = workloads.Linear("alpha-range", 1, N, K, w_seed=N + K)
    quant_parity(lin.make_weights(DEV), alpha)


def test_quantize_ldw_and_special_rows():
    N, K, ldw = 8, 96, 136
    g = torch.Generator(device=DEV).manual_seed(3)
    big = (torch.randn((N, ldw), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    big[0] = 0                               # all-zero row
    big[1, :K] = -0.0                        # negative zeros only
    big[2, 5] = -big[2].abs().max() * 2      # negative maximum ...
    big[2, 9] = big[2].abs().max()           # ... duplicated with the other sign
    big[3, :K] = torch.tensor([1.875] + [(2 * i - 1) / 16 for i in range(1, 16)] * 5 + [0.0] * 20,
                              dtype=torch.bfloat16, device=DEV)   # exact .5 ties at alpha = 1
    codes = torch.empty((N, K // 8), dtype=torch.int32, device=DEV)
    signs = torch.empty((N, K // 32), dtype=torch.int32, device=DEV)
    scales = torch.empty((N,), dtype=torch.float32, device=DEV)
    for alpha in (0.73, 1.0):
        st = opq.load().opq_quantize(opq._ptr(big), N, K, ldw, alpha, opq._ptr(codes), opq._ptr(signs),
                                     opq._ptr(scales), opq._stream(big.device))
        assert st == 0
        ref = oracle.quantize(big[:, :K].contiguous(), alpha32(alpha), want_ties=True)
        assert np.array_equal(u32(codes), ref["codes"])
        assert np.array_equal(u32(signs), ref["signs"])
        assert np.array_equal(u32(scales.view(torch.int32)), ref["scales"].view(np.uint32))
    no_device_error()


def test_quantize_deterministic():
    w = workloads.dit_attn_proj().make_weights(DEV)
    a = opq.quantize(w)
    b = opq.quantize(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ---------------------------------------------------------------- dequantize --
@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_dequantize_bit_exact(alpha):
    w = workloads.tiny().make_weights("cpu")
    ref = oracle.quantize(w, alpha)
    want = oracle.dequantize_bf16(ref["codes"], ref["signs"], ref["scales"], alpha32(alpha))
    codes, signs = to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"])
    scales = torch.from_numpy(ref["scales"]).to(DEV)
    N, K = w.shape
    ob, out, pad = guarded((N, K), torch.bfloat16, 0x77)
    opq.dequantize(codes, signs, scales, alpha, out=out)
    torch.cuda.synchronize()
    check_guards(ob, pad, 0x77)
    assert np.array_equal(u16(out), want)
    no_device_error()


def test_dequantize_full_size_bit_exact():
    lin = workloads.small_m(1)
    w = lin.make_weights("cpu")
    ref = oracle.quantize(w, lin.alpha)
    want = oracle.dequantize_bf16(ref["codes"], ref["signs"], ref["scales"], alpha32(lin.alpha))
    got = opq.dequantize(to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"]),
                         torch.from_numpy(ref["scales"]).to(DEV), lin.alpha)
    assert np.array_equal(u16(got), want)
    no_device_error()


# -------------------------------------------------------------------- linear --
def linear_parity(x_cpu, w_cpu, alpha, pairs=None, seed=0):
    """GPU linear on the oracle's packed weights vs the fp64 oracle (all outputs or sampled pairs)."""
    ref = oracle.quantize(w_cpu, alpha)
    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    x = x_cpu.to(DEV)
    codes, signs = to_dev_u32(ref["codes"]), to_dev_u32(ref["signs"])
    scales = torch.from_numpy(ref["scales"]).to(DEV)
    yb, y, pad = guarded((M, N), torch.bfloat16, 0x6B)
    opq.linear(x, codes, signs, scales, alpha, out=y)
    torch.cuda.synchronize()
    check_guards(yb, pad, 0x6B)
    no_device_error()
    yg = bits_to_f64(u16(y))
    if pairs is None:
        yref, bound = oracle.linear(x_cpu, ref["codes"], ref["signs"], ref["scales"], alpha)
        got = yg
    else:
        rng = np.random.default_rng(seed)
        ms = rng.integers(0, M, pairs)
        ns = rng.integers(0, N, pairs)
        # always include the corners and the ragged edges
        ms = np.concatenate([ms, [0, M - 1, 0, M - 1]])
        ns = np.concatenate([ns, [0, N - 1, N - 1, 0]])
        yref, bound = oracle.linear_pairs(x_cpu, ref["codes"], ref["signs"], ref["scales"], alpha, ms, ns)
        got = yg[ms, ns]
    err = np.abs(got - yref)
    tol = 1e-2 * bound + 1e-3
    bad = err > tol
    assert not bad.any(), f"{int(bad.sum())} outputs out of tolerance; worst excess {float((err - tol).max())}"
    assert np.isfinite(got).all()
    return y


def test_linear_tiny():
    x, w = workloads.tiny().make("cpu")
    linear_parity(x, w, 0.73)


@pytest.mark.parametrize("M", [1, 2, 17, 129, 256, 257, 300])
@pytest.mark.parametrize("N,K", [(1, 32), (100, 96), (257, 512), (600, 160)])
def test_linear_shapes(M, N, K):
    lin = workloads.Linear("shape", M, N, K, w_seed=7 * M + N, x_seed=11 * M + K)
    x, w = lin.make("cpu")
    linear_parity(x, w, 0.73)


@pytest.mark.parametrize("alpha", [0.45, 1.0])
def test_linear_alpha(alpha):
    lin = workloads.Linear("alpha", 130, 384, 640, alpha=alpha, w_seed=5, x_seed=6)
    x, w = lin.make("cpu")
    linear_parity(x, w, alpha)


@pytest.mark.parametrize("M", [1, 16, 33, 64])
@pytest.mark.parametrize("N,K", [(300, 384), (1000, 640), (130, 128), (2000, 1152)])
def test_linear_load_groups(M, N, K):
    # narrow tiles fetch 2 or 4 consecutive 128-K blocks per copy; K = 128 (one block), 384
    # (a group shorter than the copy), 640 (groups of 3 and 2) and 1152 (three groups of 3)
    lin = workloads.Linear("groups", M, N, K, w_seed=3 * M + N, x_seed=5 * M + K)
    x, w = lin.make("cpu")
    linear_parity(x, w, 0.73)


@pytest.mark.parametrize("M,N,K", [(16, 8192, 1152), (40, 9000, 640)])
def test_linear_load_groups_split_tiles(M, N, K):
    # more (tile, load group) units than CTAs: tiles shared by several CTAs, partial sums added
    # in CTA order
    lin = workloads.Linear("groups-split", M, N, K, w_seed=N, x_seed=M)
    x, w = lin.make("cpu")
    linear_parity(x, w, 0.73)


@pytest.mark.parametrize("M,N,K", [(512, 10240, 256), (300, 9728, 160)])
def test_linear_tail_split(M, N, K):
    # more tiles than one wave of CTAs, with the leftover tiles (at most half a wave) each
    # run as two half-width runs on two CTAs: every output, including the ragged last m-tile
    lin = workloads.Linear("tail", M, N, K, w_seed=M + N, x_seed=K)
    x, w = lin.make("cpu")
    linear_parity(x, w, 0.73)


@pytest.mark.parametrize("M,N,K", [(260, 700, 576), (512, 10240, 192), (257, 300, 64)])
def test_linear_wide_half_block(M, N, K):
    # 256-row tiles whose last 128-K block holds one 64-K half (K % 128 == 64): the second half
    # of that block reads as zeros; the middle case also splits its leftover tiles in two
    lin = workloads.Linear("half-block", M, N, K, w_seed=M * 3 + K, x_seed=N)
    x, w = lin.make("cpu")
    linear_parity(x, w, 0.73)


@pytest.mark.parametrize("M,N,K", [(512, 10240, 1024), (300, 9728, 1152)])
def test_linear_tail_ksplit(M, N, K):
    # the tiles past the last whole wave each run as two half-K runs on two CTAs whose fp32
    # partial sums meet in the workspace (3 + 5 and 3 + 6 blocks; the second has a ragged m-tile)
    lin = workloads.Linear("tail-k", M, N, K, w_seed=M + K, x_seed=N)
    x, w = lin.make("cpu")
    linear_parity(x, w, 0.73)


def test_linear_ksplit_workspace_reuse():
    # one zero-filled workspace serves repeated calls: y is bitwise the same each time and the
    # arrival counters at the workspace start are back at zero after every call
    M, N, K = 512, 10240, 1024
    need = opq.workspace_size(M, N, K)
    assert need > 65536
    lin = workloads.Linear("ws-reuse", M, N, K, w_seed=3, x_seed=4)
    x, w = lin.make(DEV)
    planes = opq.quantize(w)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    ys = []
    for _ in range(3):
        ys.append(opq.linear(x, *planes, workspace=ws))
        torch.cuda.synchronize()
        assert int(ws[:65536].count_nonzero()) == 0
        no_device_error()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])
    assert torch.equal(ys[0], opq.linear_noalloc(x, *planes))


def test_linear_deterministic():
    for M in (16, 700, 512):
        N = 10240 if M == 512 else 1024   # 512 x 10240: a half-K tail
        lin = workloads.Linear("det", M, N, 1024, w_seed=1, x_seed=2)
        x, w = lin.make(DEV)
        planes = opq.quantize(w)
        y1 = opq.linear(x, *planes)
        y2 = opq.linear(x, *planes)
        assert torch.equal(y1, y2)


# ----------------------------------------------- full sizes, sampled outputs --
def test_full_dit_attn_proj():
    lin = workloads.dit_attn_proj()
    x, w = lin.make("cpu")
    quant_parity(w.to(DEV), lin.alpha)
    linear_parity(x, w, lin.alpha, pairs=3000)


@pytest.mark.parametrize("alpha", [0.45, 0.73, 1.0])
def test_full_dit_ffn_pair(alpha):
    up, down = workloads.dit_ffn_pair(alpha)
    for lin in (up, down):
        x, w = lin.make("cpu")
        quant_parity(w.to(DEV), alpha, rows=np.arange(0, lin.N, 7))
        linear_parity(x, w, alpha, pairs=1500)


@pytest.mark.parametrize("M", workloads.SMALL_M_SWEEP)
def test_full_small_m(M):
    lin = workloads.small_m(M)
    x, w = lin.make("cpu")
    if M == 1:
        quant_parity(w.to(DEV), lin.alpha)
    linear_parity(x, w, lin.alpha, pairs=min(4000, M * lin.N))


def test_full_whole_model_sampled_layers():
    model = workloads.WholeModel()
    for idx in (0, 4, 6, 7 * 29 + 5):       # an attention, W1, W2 and a last-block layer
        lin = model.layers[idx]
        x, w = lin.make("cpu")
        quant_parity(w.to(DEV), lin.alpha, rows=np.arange(0, lin.N, 13))
        linear_parity(x, w, lin.alpha, pairs=800)


def linear_parity_planes(M, N, K, seed, pairs, extra_rows):
    """GPU linear vs the fp64 oracle on random packed planes (no quantize: the largest shapes),
    at sampled output positions plus every activation row of `extra_rows` weight rows."""
    codes, signs, scales = workloads.random_planes(N, K, seed)
    x_cpu = workloads.Linear("planes", M, N, K, x_seed=seed + 1).make_x("cpu")
    yb, y, pad = guarded((M, N), torch.bfloat16, 0x6B)
    opq.linear(x_cpu.to(DEV), to_dev_u32(codes), to_dev_u32(signs), torch.from_numpy(scales).to(DEV), 0.73, out=y)
    torch.cuda.synchronize()
    check_guards(yb, pad, 0x6B)
    no_device_error()
    rng = np.random.default_rng(seed)
    ms = np.concatenate([rng.integers(0, M, pairs), np.repeat(np.arange(M), len(extra_rows))])
    ns = np.concatenate([rng.integers(0, N, pairs), np.tile(np.asarray(extra_rows), M)])
    yref, bound = oracle.linear_pairs(x_cpu, codes, signs, scales, 0.73, ms, ns)
    got = bits_to_f64(u16(y))[ms, ns]
    err = np.abs(got - yref)
    tol = 1e-2 * bound + 1e-3
    bad = err > tol
    assert not bad.any(), f"{int(bad.sum())} outputs out of tolerance; worst excess {float((err - tol).max())}"
    assert np.isfinite(got).all()


@pytest.mark.parametrize("M,K", [(1, 1024), (16, 1024), (1, 1056)])
def test_linear_stream_k_most_tiles(M, K):
    # the largest stream-K shape by weight tiles (4096: the arrival counters' whole region),
    # K = 1024 (two load groups per tile, so CTA boundaries split tiles all along N); K = 1056
    # (not a whole number of 128-K blocks: 128-row tiles, one block per copy, signs by cp.async)
    N = 4096 * 128
    path, ctas, _ = opq.plan(M, N, K)
    assert path == 1 and ctas == 148
    rows = [0, 1, 127, 128, N // 2, N - 129, N - 128, N - 2, N - 1]
    linear_parity_planes(M, N, K, seed=1000 + M + K, pairs=1500, extra_rows=rows)


@pytest.mark.parametrize("M,K", [(8, 256), (40, 256), (100, 256)])
def test_linear_narrow_whole_tiles(M, K):
    # more weight tiles than the counter region (4194 > 4096): small M runs whole narrow tiles
    # strided over the CTAs; 4194 = 28 waves of 148 + 50 tiles, which at M = 100 (128-row
    # tiles, one block per copy) run as two half-width runs each (16- to 64-row tiles fetch
    # several blocks per copy and run them whole); a ragged last tile (N = 4194 x 128 - 37).
    # The same shapes with K % 128 != 0 are refused (test_abi)
    N = 4194 * 128 - 37
    path, ctas, _ = opq.plan(M, N, K)
    assert path == 0 and ctas == 148
    tail0 = 4144 * 128
    rows = [0, 5, tail0 - 1, tail0, tail0 + 77, N - 90, N - 2, N - 1]
    linear_parity_planes(M, N, K, seed=2000 + M + K, pairs=1500, extra_rows=rows)


def test_linear_workspace_reuse_across_shapes():
    """One zero-filled workspace serves calls of different shapes in a row: every
    call leaves its arrival counters at zero for the next one."""
    shapes = [(16, 11520, 3840), (64, 2048, 1024), (1, 3840, 3840), (16, 11520, 3840), (128, 640, 4096)]
    need = max(opq.workspace_size(*s) for s in shapes)
    ws = torch.zeros((need,), dtype=torch.uint8, device=DEV)
    for i, (M, N, K) in enumerate(shapes):
        lin = workloads.Linear("reuse", M, N, K, w_seed=31 + i, x_seed=37 + i)
        x, w = lin.make(DEV)
        planes = opq.quantize(w)
        y_shared = opq.linear(x, *planes, workspace=ws)
        y_fresh = opq.linear(x, *planes)
        assert torch.equal(y_shared, y_fresh), (M, N, K)
    torch.cuda.synchronize()
    counters = ws[: 4096 * 4 * 4].view(torch.int32)
    assert int(counters.abs().sum()) == 0
    assert opq.device_error() == 0
