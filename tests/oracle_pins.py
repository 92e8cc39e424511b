"""Pins that tie the fp64 OPQ oracle to facts fixed outside the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with a closed form, an exact-rational evaluation, a
hand-derived fixture (``tests/golden``), a brute-force search in extended
precision, or an invariant of the method ("OPQ INT4 Z-Image" model card,
"OPQ principle": u = |w|/max|w|, v = u^alpha, q = round(15 v),
w' = sign(w) (q/15)^(1/alpha) max|w|). The mutation test plants mistakes in
copies of the oracle source and checks that some pin catches each of them.
"""
from __future__ import annotations

import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers --
def bf16_bits(values) -> np.ndarray:
    """Exact bf16 bit patterns of values that are representable in bf16."""
    t = torch.tensor(list(values), dtype=torch.float64)
    b = t.to(torch.float32).to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), t), "fixture value not exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """uint32 [N, K/8] -> uint8 [N, K] with element 8j+i = nibble i of word j."""
    N, cw = codes.shape
    shifts = (4 * np.arange(8, dtype=np.uint32))[None, None, :]
    return ((codes[:, :, None] >> shifts) & 0xF).reshape(N, cw * 8).astype(np.uint8)


def unpack_signs(signs: np.ndarray) -> np.ndarray:
    N, sw = signs.shape
    shifts = np.arange(32, dtype=np.uint32)[None, None, :]
    return ((signs[:, :, None] >> shifts) & 1).reshape(N, sw * 32).astype(np.uint8)


def read_golden(name: str):
    """Blocks of 'key values...' lines; '#' comments; 'block X' starts a block."""
    blocks, cur = [], {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "block":
                if cur:
                    blocks.append(cur)
                cur = {}
                continue
            cur[key] = vals
    if cur:
        blocks.append(cur)
    return blocks


def tiny_weights() -> np.ndarray:
    w = workloads.tiny().make_weights("cpu")
    return w.view(torch.int16).numpy().view(np.uint16).copy()


# -------------------------------------------------------------------- pins --
def pin_golden_fixtures(orc):
    """Hand-derived rows: exact .5 ties at alpha = 1, bit layout, zero and duplicate-max rows."""
    for fname in ("alpha1_ties_row.txt", "special_rows.txt"):
        for blk in read_golden(fname):
            alpha = float(blk["alpha"][0])
            w = bf16_bits(float(v) for v in blk["w"])[None, :]
            r = orc.quantize(w, alpha)
            want_codes = np.array([int(v, 16) for v in blk["codes"]], np.uint32)
            want_signs = np.array([int(v, 16) for v in blk["signs"]], np.uint32)
            assert r["scales"][0] == np.float32(float(blk["scale"][0])), (fname, r["scales"])
            assert np.array_equal(r["codes"][0], want_codes), (fname, [hex(c) for c in r["codes"][0]])
            assert np.array_equal(r["signs"][0], want_signs), (fname, [hex(c) for c in r["signs"][0]])
            if "dequant" in blk:
                want = bf16_bits(float(v) for v in blk["dequant"])
                got = orc.dequantize_bf16(r["codes"], r["signs"], r["scales"], alpha)[0]
                assert np.array_equal(got, want), (fname, got, want)


def pin_alpha1_exact_rational(orc):
    """alpha = 1 reduces to round-half-even(15 |w| / max) in exact rational arithmetic."""
    w = tiny_weights()[:64]
    r = orc.quantize(w, 1.0)
    q = unpack_codes(r["codes"])
    s = unpack_signs(r["signs"])
    vals = bits_to_f64(w)
    for n in range(w.shape[0]):
        row = [Fraction(float(v)) for v in vals[n]]
        mx = max(abs(v) for v in row)
        assert Fraction(float(r["scales"][n])) == mx
        for k, v in enumerate(row):
            want = round(15 * abs(v) / mx) if mx != 0 else 0   # Fraction round(): half to even
            assert q[n, k] == want, (n, k, q[n, k], want)
            assert s[n, k] == (1 if v < 0 else 0)
    # dequantize at alpha = 1 is q/15 * max: check against exact rationals rounded once
    deq = orc.dequantize_f64(r["codes"], r["signs"], r["scales"], 1.0)
    for n in range(8):
        mx = Fraction(float(r["scales"][n]))
        for k in range(w.shape[1]):
            exact = Fraction(int(q[n, k]), 15) * mx * (-1 if s[n, k] else 1)
            assert abs(Fraction(deq[n, k]) - exact) <= abs(exact) * Fraction(1, 2 ** 51)


def pin_max_zero_monotone(orc):
    """max element -> q = 15 and w' = +-max bit-exactly; zero -> 0; codes monotone in |w|."""
    w = tiny_weights()
    w = w.copy()
    w[3, :] = 0                       # an all-zero row
    w[5, 7] = 0x8000                  # a negative zero
    for alpha in (0.45, 0.73, 1.0):
        r = orc.quantize(w, alpha)
        q = unpack_codes(r["codes"])
        mag = w & 0x7FFF
        mx = mag.max(axis=1)
        at_max = mag == mx[:, None]
        nz = mx > 0
        assert (q[at_max & nz[:, None]] == 15).all()
        assert (q[mag == 0] == 0).all()
        assert (q[~nz] == 0).all() and (r["scales"][~nz] == 0).all()
        deq = orc.dequantize_bf16(r["codes"], r["signs"], r["scales"], alpha)
        sel = at_max & nz[:, None]
        assert np.array_equal(deq[sel], w[sel]), "max element must reconstruct exactly"
        assert ((deq[mag == 0] & 0x7FFF) == 0).all()
        for n in range(w.shape[0]):
            order = np.argsort(mag[n], kind="stable")
            assert (np.diff(q[n, order].astype(np.int32)) >= 0).all(), "codes not monotone in |w|"


def _longdouble_levels(w: np.ndarray, alpha: float):
    """15 (|w|/max)^alpha in extended precision (x87 long double)."""
    a = np.abs(bits_to_f64(w)).astype(np.longdouble)
    mx = a.max(axis=1, keepdims=True)
    u = np.where(mx > 0, a / np.where(mx > 0, mx, 1), 0)
    return np.longdouble(15) * np.power(u, np.longdouble(alpha))


def pin_bruteforce_nearest_level(orc):
    """Every entry of the tiny weights: q = argmin_k |15 u^alpha - k| (extended precision, ties even)."""
    w = tiny_weights()
    for alpha in (0.45, 0.73, 1.0):
        v = _longdouble_levels(w, alpha)
        ks = np.arange(16, dtype=np.longdouble)
        d = np.abs(v[..., None] - ks)
        best = np.argmin(d, axis=-1)
        # a tie between k and k+1 resolves to the even one
        dmin = np.take_along_axis(d, best[..., None], -1)[..., 0]
        nxt = np.minimum(best + 1, 15)
        tie = np.take_along_axis(d, nxt[..., None], -1)[..., 0] == dmin
        best = np.where(tie & (best % 2 == 1), nxt, best)
        frac = v - np.floor(v)
        near = np.abs(frac - np.longdouble(0.5)) <= np.longdouble(1e-6)
        r = orc.quantize(w, alpha, want_ties=True)
        q = unpack_codes(r["codes"])
        bad = (q != best) & ~near
        assert not bad.any(), (alpha, int(bad.sum()))
        # the oracle's own near-tie flag marks the same entries
        assert np.array_equal(r["near_tie"].astype(bool), near), alpha


def pin_threshold_identity(orc):
    """q >= k  <=>  u >= ((k - 1/2)/15)^(1/alpha), checked in 50-digit decimal arithmetic."""
    getcontext().prec = 50
    w = tiny_weights()[:16]
    vals = bits_to_f64(w)
    for alpha in (0.45, 0.73):
        r = orc.quantize(w, alpha)
        q = unpack_codes(r["codes"])
        inv = Decimal(1) / Decimal(repr(alpha))
        t = [Decimal(0)] + [((Decimal(2 * k - 1) / Decimal(30)) ** inv) for k in range(1, 16)]
        for n in range(w.shape[0]):
            mx = Decimal(abs(vals[n]).max())
            for kk in range(w.shape[1]):
                u = Decimal(abs(vals[n, kk])) / mx
                want = sum(1 for k in range(1, 16) if u >= t[k])
                assert q[n, kk] == want, (alpha, n, kk, q[n, kk], want)


def pin_lut_decimal(orc):
    """Dequantized magnitudes (q/15)^(1/alpha) * max against 50-digit decimal values."""
    getcontext().prec = 50
    for alpha in (0.45, 0.73, 1.0):
        codes = np.array([[0x76543210, 0xFEDCBA98]], np.uint32)      # q = 0..15
        signs = np.array([[0x0000AAAA]], np.uint32)                  # odd elements negative
        codes = np.concatenate([codes, codes], axis=1)
        scales = np.array([1.0], np.float32)
        got = orc.dequantize_f64(codes, signs, scales, alpha)[0]
        inv = Decimal(1) / Decimal(repr(alpha))
        for k in range(32):
            q = k % 16
            mag = (Decimal(q) / Decimal(15)) ** inv if q else Decimal(0)
            want = -mag if (k < 16 and k % 2 == 1) else mag
            assert abs(Decimal(got[k]) - want) <= Decimal(2) ** -50, (alpha, k, got[k], want)


def pin_roundtrip_idempotent(orc):
    """quantize(bf16(dequantize(codes))) returns the codes (and signs where q > 0)."""
    w = tiny_weights()
    for alpha in (0.45, 0.73, 1.0):
        r = orc.quantize(w, alpha)
        deq = orc.dequantize_bf16(r["codes"], r["signs"], r["scales"], alpha)
        r2 = orc.quantize(deq, alpha)
        assert np.array_equal(r2["scales"], r["scales"])
        assert np.array_equal(r2["codes"], r["codes"]), alpha
        q = unpack_codes(r["codes"])
        s1, s2 = unpack_signs(r["signs"]), unpack_signs(r2["signs"])
        assert np.array_equal(s1[q > 0], s2[q > 0])


def pin_linear(orc):
    """y = x W'^T: one-hot rows of x return rows of W'; a BLAS matmul of W' agrees."""
    x, w = workloads.tiny().make("cpu")
    M, K = x.shape
    r = orc.quantize(w, 0.73)
    wq = orc.dequantize_f64(r["codes"], r["signs"], r["scales"], 0.73)
    # one-hot activations: 1.0 at column (7 * m) % K
    onehot = np.zeros((M, K), np.uint16)
    cols = (7 * np.arange(M)) % K
    onehot[np.arange(M), cols] = 0x3F80
    y, b = orc.linear(onehot, r["codes"], r["signs"], r["scales"], 0.73)
    assert np.array_equal(y, wq[:, cols].T)
    assert np.array_equal(b, np.abs(wq[:, cols].T))
    xv = bits_to_f64(x.view(torch.int16).numpy().view(np.uint16))
    y, b = orc.linear(x, r["codes"], r["signs"], r["scales"], 0.73)
    ref = xv @ wq.T
    assert np.abs(y - ref).max() <= 1e-12 * b.max()
    assert np.allclose(b, np.abs(xv) @ np.abs(wq).T, rtol=1e-12, atol=0)
    # sampled positions agree with the full product
    ms = np.array([0, 5, 63, 17]); ns = np.array([0, 255, 100, 3])
    yp, bp = orc.linear_pairs(x, r["codes"], r["signs"], r["scales"], 0.73, ms, ns)
    assert np.array_equal(yp, y[ms, ns]) and np.array_equal(bp, b[ms, ns])


def pin_bf16_rounding(orc):
    """double -> bf16 round-to-nearest-even against exact rational rounding."""
    rng = np.random.default_rng(7)
    vals = list(rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000))
    # exact ties between neighbours 1 + 2^-7 k, and just off them
    vals += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -40,
             3.0e38, 3.4e38, 1e-40, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 0.0, -0.0]
    for v in vals:
        got = orc.double_to_bf16(v)
        # reference: nearest bf16 by exhaustive neighbour search on exact rationals
        f32 = np.float32(v) if abs(v) < 3.4e38 else np.float32(np.sign(v) * 3.4e38)
        base = int(np.array([f32], np.float32).view(np.uint32)[0] >> 16)
        cands = [(base + d) & 0xFFFF for d in (-2, -1, 0, 1, 2)]
        best = None
        for c in cands:
            if (c & 0x7FFF) >= 0x7F80:
                continue
            cv = float(bits_to_f64(np.array([c], np.uint16))[0])
            err = abs(Fraction(cv) - Fraction(v))
            key = (err, (c & 1))  # ties: even mantissa wins
            if best is None or key < best[0]:
                best = (key, c)
        want = best[1]
        if abs(v) >= (2.0 - 2.0 ** -8) * 2.0 ** 127:   # at or past max + half an ulp: overflow
            want = 0xFF80 if v < 0 else 0x7F80
        if v == 0.0:
            want = 0x8000 if np.signbit(v) else 0
        assert got == want, (v, hex(got), hex(want))


def pin_snr_ordering(orc):
    """The method's claim, as an inequality: OPQ(alpha<1) beats alpha = 1 and uniform INT4
    on heavy-tailed weights (a Student-t(4) 512 x 3840 block)."""
    lin = workloads.Linear("snr", 1, 512, 3840, w_seed=11)
    w = lin.make_weights("cpu").view(torch.int16).numpy().view(np.uint16).copy()
    snr = {}
    for alpha in (0.45, 0.73, 1.0):
        r = orc.quantize(w, alpha)
        snr[alpha] = orc.snr_db(w, orc.dequantize_f64(r["codes"], r["signs"], r["scales"], alpha))
    snr["int4"] = orc.snr_db(w, orc.uniform_int4(w))
    assert snr[0.73] > snr[1.0] + 2.0, snr
    assert snr[1.0] > snr["int4"] + 2.0, snr


def pin_snr_closed_form(orc):
    """SNR = 10 log10(sum w^2 / sum (w - w')^2) on hand-worked pairs (the model card's
    "+7.2 dB" is a ratio of signal to quantization-error power in decibels):
    w = [1, 1], w' = [1, 0.5]: 10 log10(2 / 0.25) = 10 log10 8;
    w = [2, -1], w' = [1.5, -1]: 10 log10(5 / 0.25) = 10 log10 20 (the values differ from
    their absolute values and squares, so an unsquared term changes the result);
    an exact reconstruction has no error power: +inf."""
    w = bf16_bits([1.0, 1.0])
    got = orc.snr_db(w, np.array([1.0, 0.5]))
    assert abs(got - 10.0 * np.log10(8.0)) < 1e-12, got
    assert abs(got - 9.030899869919435) < 1e-12, got
    w = bf16_bits([2.0, -1.0])
    got = orc.snr_db(w, np.array([1.5, -1.0]))
    assert abs(got - 13.010299956639813) < 1e-12, got
    got = orc.snr_db(bf16_bits([0.25, -3.0, 0.0]), np.array([0.25, -3.0, 0.0]))
    assert got == float("inf"), got


def pin_uniform_int4_worked(orc):
    """The symmetric INT4 baseline clip(RNE(w / (max/7)), -7, 7) * max/7 on hand-worked rows.
    Row 0 has max 0.4375 = 7/16, so the step is exactly 1/16 and w/step is exact:
    0.03125 -> 0.5 -> 0 and 0.15625 -> 2.5 -> 2 (ties to even), 0.09375 -> 1.5 -> 2,
    -0.09375 -> -2, 0.1875 -> 3, the max -> 7 (reconstructs to itself).
    Row 1 has its max on a negative weight: -0.4375 -> -7. Row 2 is all zero."""
    K = 8
    rows = [[0.03125, 0.15625, 0.09375, -0.09375, 0.1875, 0.4375, 0.0, -0.03125],
            [-0.4375, 0.25, 0.3125, -0.21875, 0.0, 0.0625, -0.0625, 0.125],
            [0.0] * K]
    w = np.stack([bf16_bits(r) for r in rows])
    want_q = np.array([[0, 2, 2, -2, 3, 7, 0, 0],
                       [-7, 4, 5, -4, 0, 1, -1, 2],   # 0.21875 -> 3.5 -> 4 (even)
                       [0] * K], np.float64)
    want = want_q * np.array([[0.0625], [0.0625], [0.0]])
    got = orc.uniform_int4(w)
    assert np.array_equal(got, want), (got, want)


PINS = [pin_golden_fixtures, pin_alpha1_exact_rational, pin_max_zero_monotone,
        pin_bruteforce_nearest_level, pin_threshold_identity, pin_lut_decimal,
        pin_roundtrip_idempotent, pin_linear, pin_bf16_rounding, pin_snr_ordering,
        pin_snr_closed_form, pin_uniform_int4_worked]


# ------------------------------------------------- group-wise variant pins --
def pin_fp16_conversion(orc):
    """float16 decode and encode against numpy's binary16 (an independent implementation)."""
    bits = np.arange(0x7C00, dtype=np.uint16)                  # every non-negative finite pattern
    want = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.fp16_value(int(b)) for b in bits[::7]])
    assert np.array_equal(got, want[::7])
    assert orc.fp16_value(0x8001) == -(2.0 ** -24)
    # encode every positive finite bf16 value (RNE; beyond 65504 the reading saturates)
    pos = np.arange(1, 0x7F80, 3, dtype=np.uint16)
    vals = bits_to_f64(pos)
    enc = np.array([orc.fp16_from_nonneg(float(v)) for v in vals], dtype=np.uint16)
    inrange = vals <= 65504.0
    ref = vals[inrange].astype(np.float16).view(np.uint16)
    assert np.array_equal(enc[inrange], ref)
    assert (enc[~inrange] == 0x7BFF).all()
    # hand-derived: 1.0, 65504, 0.10009765625 = bf16 0x3DCD, 2^-24, 2^-20 + 2^-27 (rounds down)
    assert orc.fp16_from_nonneg(1.0) == 0x3C00
    assert orc.fp16_from_nonneg(65504.0) == 0x7BFF
    assert orc.fp16_from_nonneg(0.10009765625) == 0x2E68
    assert orc.fp16_from_nonneg(2.0 ** -24) == 0x0001
    assert orc.fp16_from_nonneg(2.0 ** -20 + 2.0 ** -27) == 0x0010
    assert orc.fp16_from_nonneg(0.0) == 0
    # 11 significant bits survive; ties go to even (1 + 2^-11 -> 1.0, 1 + 3 * 2^-11 -> 1 + 2^-9)
    assert orc.fp16_from_nonneg(1.0 + 2.0 ** -10) == 0x3C01
    assert orc.fp16_from_nonneg(1.0 + 2.0 ** -11) == 0x3C00
    assert orc.fp16_from_nonneg(1.0 + 3 * 2.0 ** -11) == 0x3C02
    # arbitrary doubles across float16's range against numpy's conversion
    rng = np.random.default_rng(3)
    v = np.exp(rng.uniform(np.log(2.0 ** -26), np.log(60000.0), 4000))
    got = np.array([orc.fp16_from_nonneg(float(a)) for a in v], dtype=np.uint16)
    assert np.array_equal(got, v.astype(np.float16).view(np.uint16))


def _grouped_weights(N, K, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(N, K, generator=g, dtype=torch.float64) * 0.02
    w[:, ::17] *= 6.0                                          # a few larger weights per group
    return w.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def pin_grouped_is_rowwise_per_group(orc):
    """Group-wise quantization of W[N, K] with group size GS is the per-row quantization of W
    reshaped to [N K / GS, GS] (each group a row), with the row max stored as float16."""
    N, K = 6, 1024
    w = _grouped_weights(N, K, 11)
    for gs in (32, 64, 128, 256):
        for alpha in (0.45, 0.73, 1.0):
            rg = orc.quantize_grouped(w, gs, alpha, want_ties=True)
            rr = orc.quantize(w.reshape(N * K // gs, gs), alpha, want_ties=True)
            assert np.array_equal(rg["codes"].reshape(-1), rr["codes"].reshape(-1))
            assert np.array_equal(rg["signs"].reshape(-1), rr["signs"].reshape(-1))
            assert np.array_equal(rg["near_tie"].reshape(-1), rr["near_tie"].reshape(-1))
            want_g = rr["scales"].astype(np.float16).view(np.uint16)   # exact: maxima in float16's normal range
            assert np.array_equal(rg["gmax"].reshape(-1), want_g)
            dg = orc.dequantize_grouped_f64(rg["codes"], rg["signs"], rg["gmax"], alpha)
            dr = orc.dequantize_f64(rr["codes"], rr["signs"], rr["scales"], alpha)
            assert np.array_equal(dg.reshape(-1), dr.reshape(-1))
            bg = orc.dequantize_grouped_bf16(rg["codes"], rg["signs"], rg["gmax"], alpha)
            br = orc.dequantize_bf16(rr["codes"], rr["signs"], rr["scales"], alpha)
            assert np.array_equal(bg.reshape(-1), br.reshape(-1))


def pin_grouped_worked_example(orc):
    """One 32-weight group by hand: max 0.5 (float16 0x3800), u = 1, 1/2, 1/4, 1/8, 0 at
    alpha 0.73 -> 15 u^alpha = 15, 9.04, 5.45, 3.29, 0 -> codes 15, 9, 5, 3, 0; a second group
    of the same row holds only zeros (max 0: all codes 0, sign of -0.0 is 0)."""
    row = [0.5, -0.25, 0.125, 0.0625, 0.0] + [0.0] * 27 + [0.0, -0.0] + [0.0] * 30
    w = bf16_bits(row).reshape(1, 64)
    r = orc.quantize_grouped(w, 32, 0.73)
    q = unpack_codes(r["codes"])[0]
    s = unpack_signs(r["signs"])[0]
    assert list(q[:5]) == [15, 9, 5, 3, 0] and not q[5:].any()
    assert list(s[:5]) == [0, 1, 0, 0, 0] and not s[5:].any()
    assert list(r["gmax"][0]) == [0x3800, 0]
    d = orc.dequantize_grouped_f64(r["codes"], r["signs"], r["gmax"], 0.73)[0]
    assert d[0] == 0.5 and d[1] == -((9 / 15) ** (1 / 0.73)) * 0.5 and not d[32:].any()


def pin_grouped_range_edges(orc):
    """A max beyond float16 saturates to 65504 (codes of larger weights clamp at 15); a max in
    float16's subnormal range rounds (2^-20 + 2^-27 -> 2^-20) and the max itself codes to 15."""
    big = [1e5 if i == 3 else 0.0 for i in range(32)]
    tiny_max = 2.0 ** -20 + 2.0 ** -27
    tiny = [tiny_max if i == 5 else (2.0 ** -22 if i == 6 else 0.0) for i in range(32)]
    big_b = bf16_bits([float(torch.tensor(v).to(torch.bfloat16)) for v in big])
    w = np.concatenate([big_b, bf16_bits(tiny)]).reshape(1, 64)
    r = orc.quantize_grouped(w, 32, 0.73)
    q = unpack_codes(r["codes"])[0]
    assert list(r["gmax"][0]) == [0x7BFF, 0x0010]
    assert q[3] == 15 and q[32 + 5] == 15
    # 2^-22 / 2^-20 = 1/4 -> 15 * 0.25^0.73 = 5.45 -> 5
    assert q[32 + 6] == 5


def pin_grouped_linear(orc):
    """The group-wise linear is x @ W'^T with W' the group-wise dequantization (numpy fp64
    matmul as the independent sum), and the pair list agrees with the full product."""
    N, K, M = 40, 512, 7
    w = _grouped_weights(N, K, 5)
    g = torch.Generator().manual_seed(6)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    for gs in (64, 128):
        r = orc.quantize_grouped(w, gs, 0.73)
        wd = orc.dequantize_grouped_f64(r["codes"], r["signs"], r["gmax"], 0.73)
        y, b = orc.linear_grouped(x, r["codes"], r["signs"], r["gmax"], 0.73)
        xf = bits_to_f64(x)
        assert np.allclose(y, xf @ wd.T, rtol=1e-12, atol=1e-12)
        assert np.allclose(b, np.abs(xf) @ np.abs(wd).T, rtol=1e-12, atol=1e-12)
        ms = np.array([0, 6, 3, 2]); ns = np.array([0, 39, 17, 5])
        yp, bp = orc.linear_grouped_pairs(x, r["codes"], r["signs"], r["gmax"], 0.73, ms, ns)
        assert np.array_equal(yp, y[ms, ns]) and np.array_equal(bp, b[ms, ns])


PINS += [pin_fp16_conversion, pin_grouped_is_rowwise_per_group, pin_grouped_worked_example,
         pin_grouped_range_edges, pin_grouped_linear]


# ------------------------------------------------------- fused epilogue pins --
def pin_epilogue(orc):
    """act(y + b): SiLU and GELU's tanh form against torch's fp64 implementations, closed forms
    at 0 and 1 (silu(1) = 1 / (1 + e^-1), gelu_tanh(1) = (1 + tanh(sqrt(2/pi) 1.044715)) / 2),
    and the bias added per output column."""
    rng = np.random.default_rng(9)
    y = rng.normal(0.0, 3.0, (5, 40))
    t = torch.from_numpy(y)
    assert np.allclose(orc.apply_epilogue(y, None, 1), torch.nn.functional.silu(t).numpy(), rtol=1e-14, atol=1e-15)
    assert np.allclose(orc.apply_epilogue(y, None, 2),
                       torch.nn.functional.gelu(t, approximate="tanh").numpy(), rtol=1e-14, atol=1e-15)
    assert np.array_equal(orc.apply_epilogue(y, None, 0), y)
    e = orc.apply_epilogue(np.array([[0.0, 1.0]]), None, 1)[0]
    assert e[0] == 0.0 and abs(e[1] - 0.7310585786300049) < 1e-15
    g = orc.apply_epilogue(np.array([[0.0, 1.0]]), None, 2)[0]
    assert g[0] == 0.0 and abs(g[1] - 0.8411919906082768) < 1e-15
    b = bf16_bits([0.5 * (i % 7) - 1.5 for i in range(40)])
    got = orc.apply_epilogue(y, b, 0)
    assert np.array_equal(got, y + bits_to_f64(b)[None, :])
    assert np.allclose(orc.apply_epilogue(y, b, 1),
                       torch.nn.functional.silu(t + torch.from_numpy(bits_to_f64(b))[None, :]).numpy(),
                       rtol=1e-14, atol=1e-15)


PINS += [pin_epilogue]


# ------------------------------------------------------ other bit widths pins --
def pin_bits_four_is_default(orc):
    """4-bit codes through the bit-width path equal the card's nibble format."""
    w = tiny_weights()
    for alpha in (0.45, 0.73, 1.0):
        a = orc.quantize_bits(w, 4, alpha, want_ties=True)
        b = orc.quantize(w, alpha, want_ties=True)
        for k in ("codes", "signs", "scales", "near_tie"):
            assert np.array_equal(a[k], b[k]), k


def _stream_codes(codes: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Unpack a little-endian bit stream with Python integers (independent of the oracle)."""
    out = np.zeros((codes.shape[0], K), np.int64)
    for n in range(codes.shape[0]):
        big = 0
        for j, word in enumerate(codes[n].tolist()):
            big |= int(word) << (32 * j)
        for k in range(K):
            out[n, k] = (big >> (k * bits)) & ((1 << bits) - 1)
    return out


def pin_bits_bruteforce(orc):
    """3, 5 and 6 bits: every code is the nearest level of L u^alpha (L = 2^bits - 1, ties to
    even) in long double, unpacked from the stream with Python integers."""
    w = tiny_weights()[:24]
    x = bits_to_f64(w).astype(np.longdouble)
    mx = np.abs(x).max(axis=1, keepdims=True)
    for bits in (3, 5, 6):
        L = (1 << bits) - 1
        for alpha in (0.45, 0.73):
            r = orc.quantize_bits(w, bits, alpha, want_ties=True)
            got = _stream_codes(r["codes"], w.shape[1], bits)
            v = L * (np.abs(x) / mx) ** np.longdouble(alpha)
            want = np.clip(np.rint(v), 0, L).astype(np.int64)
            mism = (got != want) & ~r["near_tie"].astype(bool)
            assert not mism.any(), (bits, alpha, int(mism.sum()))
            assert np.array_equal(unpack_signs(r["signs"]), (x < 0).astype(np.uint8))


def pin_bits_worked_stream(orc):
    """3 bits at alpha = 1, by hand: row q/4 for q = 7, 0, 1, ..., 6 (max 1.75, so 7 |w| / max
    = q exactly) -> codes q_k at bits 3k of a 96-bit stream, and the decode gives the row back."""
    qs = [7, 0, 1, 2, 3, 4, 5, 6] * 4
    row = [q / 4 for q in qs]
    w = bf16_bits(row).reshape(1, 32)
    r = orc.quantize_bits(w, 3, 1.0)
    big = sum(q << (3 * k) for k, q in enumerate(qs))
    want = [(big >> (32 * j)) & 0xFFFFFFFF for j in range(3)]
    assert [int(v) for v in r["codes"][0]] == want
    assert r["scales"][0] == 1.75
    d = orc.dequantize_bits_f64(r["codes"], r["signs"], r["scales"], 3, 1.0)
    assert np.array_equal(d[0], np.array(row))
    db = orc.dequantize_bits_bf16(r["codes"], r["signs"], r["scales"], 3, 1.0)
    assert np.array_equal(db[0], w[0])


PINS += [pin_bits_four_is_default, pin_bits_bruteforce, pin_bits_worked_stream]
