"""Planted mistakes in the oracle must fail its pins.

Each case compiles a copy of oracle/wq_oracle.c with one plausible mistake
(a dropped term, a wrong sign, a wrong constant, a transposed index, another
rounding rule), binds the wrappers to it, runs the pin tests and expects at
least one of them to fail.  CPU only; the real oracle is rebound afterwards.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

MUTANTS = {
    "zero_point_sign": ("nearbyintf(-mn / s)", "nearbyintf(mn / s)"),
    "range_over_16": ("(mx - mn) / 15.0f", "(mx - mn) / 16.0f"),
    "encode_minus_z": ("nearbyintf(wg[i] / s + z)", "nearbyintf(wg[i] / s - z)"),
    "truncate_not_round": ("nearbyintf(wg[i] / s + z)", "floorf(wg[i] / s + z)"),
    "ties_away_from_zero": ("nearbyintf(wg[i] / s + z)", "roundf(wg[i] / s + z)"),
    "no_upper_clip": ("if (t > 15.0f) t = 15.0f;", ";"),
    "z_not_rounded": ("float z = store_param(nearbyintf(-mn / s) + 0.0f, mode);",
                      "float z = store_param(-mn / s, mode);"),
    "int8_qmax_128": ("amax / 127.0f", "amax / 128.0f"),
    "int8_no_round": ("float t = nearbyintf(wg[i] / s);", "float t = truncf(wg[i] / s);"),
    "dequant_plus_z": ("((double)codes[n * K + k] - (double)z[n * G + k / g])",
                       "((double)codes[n * K + k] + (double)z[n * G + k / g])"),
    "dequant_group_index": ("s[n * G + k / g] * ((double)codes", "s[n * G + k % G] * ((double)codes"),
    "matmul_transposed": ("x[m * K + k] * w_hat[n * K + k]", "x[m * K + k] * w_hat[k * N + n]"),
    "matmul_drops_abs": ("aacc += fabs(p);", "aacc += p;"),
    "pack_nibbles_swapped": ("(codes[n * K + 2 * j] & 0xf) | ((codes[n * K + 2 * j + 1] & 0xf) << 4)",
                             "(codes[n * K + 2 * j + 1] & 0xf) | ((codes[n * K + 2 * j] & 0xf) << 4)"),
    "bf16_truncates": ("if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;", ";"),
    "sym_levels_8": ("amax / 7.0f", "amax / 8.0f"),
    "sym_offset_7": ("(uint8_t)((int)q + 8)", "(uint8_t)((int)q + 7)"),
    "sym_truncate": ("float q = nearbyintf(wg[i] / s);", "float q = truncf(wg[i] / s);"),
    "sym_ties_away": ("float q = nearbyintf(wg[i] / s);", "float q = roundf(wg[i] / s);"),
    "sym_signed_max": ("const float a = fabsf(wg[i]);", "const float a = wg[i];"),
    "fp8_bias_off_by_one": ("const int bias = (1 << (ebits - 1)) - 1;", "const int bias = (1 << (ebits - 1));"),
    "fp8_ties_to_odd": ("(d == best_d && (c & 1) == 0)", "(d == best_d && (c & 1) == 1)"),
    "fp8_subnormal_exponent": ("ldexp((double)m, 1 - bias - mbits)", "ldexp((double)m, -bias - mbits)"),
    "fp8_rows_int8_scale": ("amax / (float)oracle_fp8_max(fmt)", "amax / 127.0f"),
    "e2m1_bias_2": ("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)"),
    "e2m1_ties_to_odd": ("if (d < best_d || (d == best_d && (c & 1) == 0)) {", "if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    "nvfp4_tensor_scale_int8": ("float st = amax / (6.0f * 448.0f);", "float st = amax / (6.0f * 127.0f);"),
    "nvfp4_block_scale_over_7": ("oracle_fp8_encode((bmax / 6.0f) / st, 0)", "oracle_fp8_encode((bmax / 7.0f) / st, 0)"),
    "unpack_high_nibble_unmasked": ("codes[n * K + 2 * j + 1] = packed[n * (K / 2) + j] >> 4;",
                                    "codes[n * K + 2 * j + 1] = packed[n * (K / 2) + j] >> 3;"),
    "int8_dequant_group_index": ("(double)s[n * G + k / g] * (double)codes[n * K + k]",
                                 "(double)s[n * G + k % G] * (double)codes[n * K + k]"),
    "int8_zero_scale_kept": ("float s = store_param(amax / 127.0f, mode);\n            if (s == 0.0f) s = 1.0f;",
                             "float s = store_param(amax / 127.0f, mode);"),
    "fp8_rows_zero_scale_kept": ("float s = amax / (float)oracle_fp8_max(fmt);\n        if (s == 0.0f) s = 1.0f;",
                                 "float s = amax / (float)oracle_fp8_max(fmt);"),
    "fp8_no_saturation": ("if (a > oracle_fp8_max(fmt)) a = oracle_fp8_max(fmt);", ";"),
    "e2m1_no_saturation": ("if (!(a <= 6.0)) a = 6.0;", ";"),
    "nvfp4_global_amax_per_row": ("if (fabsf(w[n * ldw + k]) > amax) amax = fabsf(w[n * ldw + k]);",
                                  "if (n == 0 && fabsf(w[n * ldw + k]) > amax) amax = fabsf(w[n * ldw + k]);"),
    "matmul_bound_without_a": ("if (a) a[m * N + n] = aacc;", "if (a) a[m * N + n] = fabs(acc);"),
    "nvfp4_dequant_block_index": ("block_codes[n * (K / 16) + k / 16]", "block_codes[n * (K / 16) + k % (K / 16)]"),
    "nvfp4_dequant_scale_as_e5m2": ("oracle_fp8_decode(block_codes[n * (K / 16) + k / 16], 0)",
                                    "oracle_fp8_decode(block_codes[n * (K / 16) + k / 16], 1)"),
}

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _call_pin(fn):
    import inspect
    params = inspect.signature(fn).parameters
    if not params:
        fn()
        return
    # parametrised pins: run every parameter value the test module declares
    marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
    assert len(marks) == 1
    name, values = marks[0].args
    for v in values:
        fn(**{name: v})


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_mutant(mutant, tmp_path):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) >= 1, f"mutation site for {mutant} not found"
    path_c = os.path.join(tmp_path, "mutant.c")
    path_so = os.path.join(tmp_path, "libmutant.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new, 1))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", path_so, path_c, "-lm"], check=True)
    saved = oracle.swap_library(path_so)
    failures = 0
    try:
        for fn in PINS:
            try:
                _call_pin(fn)
            except Exception:
                failures += 1
    finally:
        oracle.swap_library(None)
        oracle._lib = saved
    assert failures > 0, f"no pin caught mutant {mutant}"
