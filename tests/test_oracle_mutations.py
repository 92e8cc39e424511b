"""Plant one plausible mistake at a time in a copy of the oracle source and
check that at least one pin rejects the mutant. The mistakes are planted on
the CPU, in temporary copies; the committed oracle is never modified."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "opq_oracle.c")

# (id, text in the oracle source, replacement): each must occur exactly once
MUTANTS = [
    ("round_half_up", "double qd = nearbyint(v15);", "double qd = floor(v15 + 0.5);"),
    ("nibble_order_reversed", "codes[n * cw + bit / 32] |= q << (bit % 32);",
     "codes[n * cw + bit / 32] |= q << (28 - bit % 32);"),
    ("sign_bit_order_reversed", "signs[n * sw + k / 32] |= s << (k % 32);",
     "signs[n * sw + k / 32] |= s << (31 - k % 32);"),
    ("forward_exponent_inverted", "v15 = levels * pow(a / mx, alpha);",
     "v15 = levels * pow(a / mx, 1.0 / alpha);"),
    ("inverse_exponent_not_inverted", "double mag = pow((double)q / levels, 1.0 / alpha) * mx;",
     "double mag = pow((double)q / levels, alpha) * mx;"),
    ("fourteen_levels", "v15 = levels * pow(a / mx, alpha);", "v15 = (levels - 1.0) * pow(a / mx, alpha);"),
    ("scale_dropped_in_dequant", "double mag = pow((double)q / levels, 1.0 / alpha) * mx;",
     "double mag = pow((double)q / levels, 1.0 / alpha);"),
    ("sign_test_flipped", "uint32_t s = (wk < 0.0) ? 1u : 0u;", "uint32_t s = (wk > 0.0) ? 1u : 0u;"),
    ("negative_zero_negative", "uint32_t s = (wk < 0.0) ? 1u : 0u;", "uint32_t s = signbit(wk) ? 1u : 0u;"),
    ("sign_dropped_in_dequant", "return s ? -mag : mag;", "return mag;"),
    ("x_transposed", "double xv = bf16_value(x[m * K + k]);\n                    acc += xv * wrow[k];",
     "double xv = bf16_value(x[k * M + m]);\n                    acc += xv * wrow[k];"),
    ("pairs_n_for_m", "int64_t m = ms[i], n = ns[i];", "int64_t m = ms[i], n = ms[i];"),
    ("bound_signed", "b += fabs(xv) * fabs(wrow[k]);", "b += xv * wrow[k];"),
    ("max_signed", "double a = fabs(bf16_value(row[k]));\n        if (a > mx)",
     "double a = bf16_value(row[k]);\n        if (a > mx)"),
    ("bf16_round_half_up", "double r = nearbyint(ldexp(a, -qexp));", "double r = floor(ldexp(a, -qexp) + 0.5);"),
    ("bf16_truncate", "double r = nearbyint(ldexp(a, -qexp));", "double r = floor(ldexp(a, -qexp));"),
    ("near_tie_band_wide", "<= 1e-6) ? 1 : 0;", "<= 1e-3) ? 1 : 0;"),
    # group-wise variant
    ("group_index_wrapped", "return fp16_value(gmax[n * (K / GS) + k / GS]);",
     "return fp16_value(gmax[n * (K / GS) + k % (K / GS)]);"),
    ("group_max_cumulative", "max_abs(row, g * GS, (g + 1) * GS)", "max_abs(row, 0, (g + 1) * GS)"),
    ("fp16_truncate", "double v = ldexp(nearbyint(ldexp(a, -qexp)), qexp);",
     "double v = ldexp(floor(ldexp(a, -qexp)), qexp);"),
    ("fp16_ten_bits", "int qexp = e - 11;", "int qexp = e - 10;"),
    ("fp16_no_saturation", "if (v > 65504.0)\n        v = 65504.0;", "if (v > 1e30)\n        v = 65504.0;"),
    # bit widths other than 4
    ("stream_carry_dropped", "two |= (uint64_t)codes[n * cw + bit / 32 + 1] << 32;", "two |= 0;"),
    ("stream_carry_write_dropped", "codes[n * cw + bit / 32 + 1] |= q >> (32 - bit % 32);", "(void)0;"),
    # fused epilogue
    ("silu_exp_sign", "v = v / (1.0 + exp(-v));", "v = v / (1.0 + exp(v));"),
    ("gelu_square", "0.044715 * v * v * v", "0.044715 * v * v"),
    ("bias_dropped", "double v = y[m * N + n] + (bias ? bf16_value(bias[n]) : 0.0);", "double v = y[m * N + n];"),
    ("fp16_subnormal_floor", "if (qexp < -24)\n        qexp = -24;", "if (qexp < -25)\n        qexp = -25;"),
    # SNR and the symmetric INT4 baseline (quality context)
    ("snr_amplitude_decibels", "return 10.0 * log10(sig / err);", "return 20.0 * log10(sig / err);"),
    ("snr_ratio_inverted", "return 10.0 * log10(sig / err);", "return 10.0 * log10(err / sig);"),
    ("snr_error_unsquared", "err += d * d;", "err += fabs(d);"),
    ("snr_signal_unsquared", "sig += a * a;", "sig += fabs(a);"),
    ("int4_step_over_eight", "nearbyint(v / (mx / 7.0));", "nearbyint(v / (mx / 8.0));"),
    ("int4_round_half_up", "nearbyint(v / (mx / 7.0));", "floor(v / (mx / 7.0) + 0.5);"),
    ("int4_reconstruction_unscaled", "w_rec[n * K + k] = q * mx / 7.0;", "w_rec[n * K + k] = q / 7.0;"),
]


@pytest.mark.parametrize("mid,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(mid, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {mid} not unique"
    mut = tmp_path / f"{mid}.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / f"{mid}.so"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(so), str(mut), "-lm"])
    orc = oracle.Oracle(str(so))
    caught = []
    for pin in oracle_pins.PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
            break
    assert caught, f"no pin rejects the mutant {mid}"
