"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden/, cited there), closed forms, brute force over all
codes on small groups, invariants that hold for any input, and independent
library routines (numpy's binary64 matmul, torch's bf16 rounding).  These are
CPU-only.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from golden import read, scalar

U_BF16 = 2.0 ** -8  # unit roundoff of bf16 (8 significant bits: half an ulp of 2^-7)


# --------------------------------------------------------------------------
# "Quantization for LLM inference ...", "Numerical example"
# --------------------------------------------------------------------------

def _worked():
    sc, rows = read("int4_worked_example.txt")
    w = np.array([[float(r[0]) for r in rows]], dtype=np.float32)
    return sc, rows, w


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_worked_example_codes_scale_zero(mode):
    sc, rows, w = _worked()
    g = int(scalar(sc, "group"))
    codes, s, z = oracle.quantize_int4(w, g, mode)
    assert codes[0].tolist() == [int(r[3]) for r in rows]
    assert [int(r[2]) for r in rows] == [int(r[3]) for r in rows]  # no code was clipped except 15.14
    assert z[0, 0] == scalar(sc, "z_printed")
    # s printed to 4 decimals: 0.1553.  Both the binary32 and the bf16 value round to it.
    assert abs(float(s[0, 0]) - scalar(sc, "s_printed")) < 5e-5
    # range and the unrounded zero-point as printed
    assert abs((w.max() - w.min()) - scalar(sc, "range")) < 1e-6
    assert abs(-w.min() / float(s[0, 0]) - scalar(sc, "z_unrounded_printed")) < 5e-3


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_worked_example_t_column(mode):
    """t = w/s + z, printed to 2 decimals; the garbled -0.91 row uses the recomputed value."""
    sc, rows, w = _worked()
    codes, s, z = oracle.quantize_int4(w, 8, mode)
    t = w[0].astype(np.float64) / float(s[0, 0]) + float(z[0, 0])
    want = np.array([float(r[6]) for r in rows])
    assert np.all(np.abs(t - want) < 0.006), (t, want)
    # the printed value of the garbled row is not what the formula gives
    printed = np.array([float(r[1]) for r in rows])
    assert abs(t[5] - printed[5]) > 0.1 and abs(t[5] - 0.14) < 0.006


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_worked_example_reconstruction_and_mse(mode):
    sc, rows, w = _worked()
    codes, s, z = oracle.quantize_int4(w, 8, mode)
    w_hat = oracle.dequant_int4(codes, s, z, 8)[0]
    printed_hat = np.array([float(r[4]) for r in rows])
    printed_err = np.array([float(r[5]) for r in rows])
    # printed to 3 decimals from s ~ 0.1553; our s differs by < 3e-5, |q - z| <= 9
    assert np.all(np.abs(w_hat - printed_hat) < 1e-3)
    err = w_hat - w[0].astype(np.float64)
    assert np.all(np.abs(err - printed_err) < 1e-3)
    mse = float(np.mean(err ** 2))
    assert abs(mse - scalar(sc, "mse_printed")) < 5e-5  # "MSE ~ 0.0015"


def test_worked_example_storage():
    sc, rows, w = _worked()
    codes, s, z = oracle.quantize_int4(w, 8, oracle.STORED)
    packed = oracle.pack_int4(codes)
    assert packed.nbytes == 4  # 8 x 4 bits
    assert oracle.example_bytes(8, 4, 16, 4) == scalar(sc, "storage_bytes_printed")


# --------------------------------------------------------------------------
# "Quantization Methods Compared ...", "What quantisation does"
# --------------------------------------------------------------------------

def _int8_fixture():
    sc, _ = read("int8_absmax_example.txt")
    w = np.array([[float(v) for v in sc["weights"][0]]], dtype=np.float32)
    return sc, w


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_absmax_int8_example_sub_one_percent(mode):
    sc, w = _int8_fixture()
    codes, s = oracle.quantize_int8(w, w.shape[1], mode)
    # s = max|w| / 127 (bf16-rounded in STORED mode)
    assert abs(float(s[0, 0]) - 0.90 / 127) <= (U_BF16 if mode else 1e-7) * 0.90 / 127
    w_hat = oracle.dequant_int8(codes, s, w.shape[1])[0]
    rel = np.abs(w_hat - w[0]) / np.abs(w[0])
    assert rel.max() * 100 < scalar(sc, "max_rel_error_before_percent_below")
    assert codes[0].tolist() == [17, -71, 47, 127]


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_absmax_int8_outlier_31_percent(mode):
    sc, w = _int8_fixture()
    w5 = np.concatenate([w, [[scalar(sc, "outlier")]]], axis=1).astype(np.float32)
    codes, s = oracle.quantize_int8(w5, w5.shape[1], mode)
    if mode == oracle.EXACT:
        assert abs(float(s[0, 0]) - scalar(sc, "step_with_outlier_printed")) < 5e-5
    else:
        assert abs(float(s[0, 0]) - 20.0 / 127) <= U_BF16 * 20.0 / 127
    w_hat = oracle.dequant_int8(codes, s, w5.shape[1])[0]
    rel = abs(w_hat[0] - 0.12) / 0.12
    assert round(rel * 100) == scalar(sc, "rel_error_after_percent_printed")
    assert codes[0, -1] == 127


def test_storage_accounting():
    sc, _ = read("storage_accounting.txt")
    for b, g, sb, zb, v in sc["bits_per_weight"]:
        assert oracle.bits_per_weight(int(b), int(g), int(sb), int(zb)) == float(v)
    for b, g, sb, zb, v in sc["model_gb_70b"]:
        assert round(oracle.model_gigabytes(70e9, int(b), int(g), int(sb), int(zb)), 1) == float(v)
    for b, g, sb, zb, v in sc["fp16_gb_70b"]:
        assert oracle.model_gigabytes(70e9, int(b), int(g), int(sb), int(zb)) == float(v)
    fp16 = oracle.model_gigabytes(70e9, 16, 1, 0, 0)
    assert round(fp16 / oracle.model_gigabytes(70e9, 4, 16, 8, 0), 2) == 3.56
    for b, n, sb, zb, v in sc["example_bytes"]:
        assert oracle.example_bytes(int(n), int(b), int(sb), int(zb)) == float(v)
    # the library's format carries a bf16 zero-point as well
    assert oracle.bits_per_weight(4, 128, 16, 16) == 4.25
    assert oracle.bits_per_weight(4, 32, 16, 16) == 5.0


@pytest.mark.parametrize("g", [32, 64, 128])
def test_storage_matches_array_bytes(g):
    w = wq_inputs.tiny_weight()
    codes, s, z = oracle.quantize_int4(w.numpy(), g)
    packed = oracle.pack_int4(codes)
    nbytes = packed.nbytes + 2 * s.size + 2 * z.size  # bf16 s and z
    N, K = w.shape
    assert nbytes * 8 == N * K * oracle.bits_per_weight(4, g, 16, 16)


# --------------------------------------------------------------------------
# Error bound: "Test-time quantization ...", "The error of quantising an
# outlier with the wrong scale" -- the rounding error is at most half a scale.
# --------------------------------------------------------------------------

def _groups(seed, n_groups, g):
    gens = [
        wq_inputs.uniform_weight(n_groups, g, seed),
        wq_inputs.heavy_tail_weight(n_groups, g, seed + 1),
        wq_inputs.tiny_weight(seed + 2, N=n_groups, K=g),
        wq_inputs.llm_weight(n_groups, g, seed + 3, outlier_frac=0.01, outlier_mult=20,
                             dtype=torch.float32),
        wq_inputs.uniform_weight(n_groups, g, seed + 4, lo=-1e-3, hi=5.0),
    ]
    return np.concatenate([t.numpy() for t in gens], axis=0)


@pytest.mark.parametrize("g", [8, 32, 128])
def test_int4_error_at_most_half_scale_exact(g):
    w = _groups(11, 2000 // g * 8, g)
    codes, s, z = oracle.quantize_int4(w, g, oracle.EXACT)
    err = np.abs(oracle.dequant_int4(codes, s, z, g) - w.astype(np.float64))
    bound = 0.5 * np.repeat(s.astype(np.float64), g, axis=1) * (1 + 1e-5)
    assert np.all(err <= bound)
    # the bound is tight: some element reaches at least 0.45 s
    assert np.max(err / bound) > 0.9


@pytest.mark.parametrize("g", [8, 32, 128])
def test_int4_error_bound_stored(g):
    """bf16 s can be up to u below the binary32 s, so the clipped top element may exceed s/2 by 15u/(1-u) s."""
    w = _groups(21, 2000 // g * 8, g)
    codes, s, z = oracle.quantize_int4(w, g, oracle.STORED)
    err = np.abs(oracle.dequant_int4(codes, s, z, g) - w.astype(np.float64))
    k = 0.5 + 15 * U_BF16 / (1 - U_BF16)
    bound = k * np.repeat(s.astype(np.float64), g, axis=1) * (1 + 1e-5)
    assert np.all(err <= bound)
    # non-clipped codes are still within half a scale
    inner = (codes > 0) & (codes < 15)
    assert np.all(err[inner] <= 0.5 * np.repeat(s.astype(np.float64), g, axis=1)[inner] * (1 + 1e-5))


def test_int8_error_at_most_half_scale_exact():
    w = _groups(31, 256, 64)
    codes, s = oracle.quantize_int8(w, 64, oracle.EXACT)
    err = np.abs(oracle.dequant_int8(codes, s, 64) - w.astype(np.float64))
    assert np.all(err <= 0.5 * np.repeat(s.astype(np.float64), 64, axis=1) * (1 + 1e-5))


# --------------------------------------------------------------------------
# Brute force on small groups: every code is the nearest level (ties to even).
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_int4_codes_are_nearest_levels(mode):
    w = _groups(41, 400, 8)
    codes, s, z = oracle.quantize_int4(w, 8, mode)
    # the scale and zero-point themselves, by the page's formulas
    mn, mx = w.min(1).astype(np.float64), w.max(1).astype(np.float64)
    s64 = s[:, 0].astype(np.float64)
    rel = 1e-6 if mode == oracle.EXACT else U_BF16 * 1.0001
    assert np.all(np.abs(s64 - (mx - mn) / 15) <= rel * (mx - mn) / 15)
    assert np.all(np.abs(z[:, 0] - np.round(-mn / s64)) <= 1)  # round of binary32 vs binary64 quotient
    assert np.all(z == np.round(z))
    levels = np.arange(16, dtype=np.float64)
    for i in range(w.shape[0]):
        t = w[i].astype(np.float64) / s64[i] + float(z[i, 0])
        d = np.abs(t[:, None] - levels[None, :])
        best = d.min(axis=1)
        chosen = d[np.arange(8), codes[i]]
        assert np.all(chosen <= best + 1e-5), (i, t, codes[i])


def test_int4_ties_round_to_even():
    # min 0, max 15 -> s = 1 and z = 0 exactly; the other values sit on half-integers
    w = np.array([[0.0, 15.0, 2.5, 3.5, 0.5, 1.5, 14.5, 7.5]], dtype=np.float32)
    for mode in (oracle.EXACT, oracle.STORED):
        codes, s, z = oracle.quantize_int4(w, 8, mode)
        assert s[0, 0] == 1.0 and z[0, 0] == 0.0
        assert codes[0].tolist() == [0, 15, 2, 4, 0, 2, 14, 8]


def test_int8_codes_are_nearest_levels():
    w = _groups(51, 200, 8)
    codes, s = oracle.quantize_int8(w, 8, oracle.EXACT)
    levels = np.arange(-127, 128, dtype=np.float64)
    for i in range(w.shape[0]):
        t = w[i].astype(np.float64) / float(s[i, 0])
        d = np.abs(t[:, None] - levels[None, :])
        chosen = d[np.arange(8), codes[i].astype(np.int64) + 127]
        assert np.all(chosen <= d.min(axis=1) + 1e-5)
    # the largest magnitude maps to +-127
    amax_idx = np.abs(w).argmax(axis=1)
    assert np.all(np.abs(codes[np.arange(w.shape[0]), amax_idx]) == 127)


# --------------------------------------------------------------------------
# Degenerate groups (the pages are silent; readings in the design notes)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_degenerate_groups(mode):
    w = np.zeros((4, 32), dtype=np.float32)
    w[1, :] = 0.25
    w[2, :] = -3.0
    w[3, :] = 1.0e-30  # below bf16's smallest normal step for s
    codes, s, z = oracle.quantize_int4(w, 32, mode)
    w_hat = oracle.dequant_int4(codes, s, z, 32)
    assert s[0, 0] == 1.0 and z[0, 0] == 0.0 and np.all(codes[0] == 0)
    assert np.all(w_hat[0] == 0.0)
    assert np.all(w_hat[1] == 0.25) and np.all(w_hat[2] == -3.0)
    assert np.all(np.abs(w_hat[3] - 1e-30) <= 1e-30 * U_BF16)
    c8, s8 = oracle.quantize_int8(w, 32, mode)
    assert s8[0, 0] == 1.0 and np.all(c8[0] == 0)
    assert np.all(c8[1] == 127) and np.all(c8[2] == -127)
    assert np.all(np.abs(oracle.dequant_int8(c8, s8, 32)[1] - 0.25) <= 0.5 * s8[1, 0])


def test_one_signed_groups_keep_codes_in_range():
    w = wq_inputs.one_signed_weight(64, 128, 7).numpy()
    codes, s, z = oracle.quantize_int4(w, 128, oracle.EXACT)
    assert codes.min() >= 0 and codes.max() <= 15
    assert np.all(z < 0)  # min > 0 puts the zero-point below code 0
    err = np.abs(oracle.dequant_int4(codes, s, z, 128) - w.astype(np.float64))
    assert np.all(err <= 0.5 * np.repeat(s.astype(np.float64), 128, axis=1) * (1 + 1e-5))


# --------------------------------------------------------------------------
# Stored parameters, packing and bf16 rounding
# --------------------------------------------------------------------------

def test_stored_params_are_bf16_values():
    w = wq_inputs.llm_weight(64, 512, 3, dtype=torch.float32).numpy()
    codes, s, z = oracle.quantize_int4(w, 128, oracle.STORED)
    for p in (s, z):
        assert np.array_equal(oracle.bf16_value(oracle.bf16_bits(p)), p)
    c8, s8 = oracle.quantize_int8(w, 512, oracle.STORED)
    assert np.array_equal(oracle.bf16_value(oracle.bf16_bits(s8)), s8)


def test_bf16_rounding_matches_torch():
    g = torch.Generator().manual_seed(5)
    v = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-60, 60, (200000,), generator=g).float())
    # exact ties: a kept value plus half a bf16 ulp
    # finite patterns only (inputs are finite by contract); both signs
    base = torch.randint(0, 0x7f7f, (4096,), generator=g).to(torch.int32) << 16
    base[::2] |= torch.tensor(-(1 << 31), dtype=torch.int32)
    ties = (base | 0x8000).view(torch.float32)
    denorm = torch.tensor([1e-40, -3e-39, 1.2e-38, 0.0, -0.0], dtype=torch.float32)
    allv = torch.cat([v, ties, denorm])
    ours = oracle.bf16_bits(allv.numpy())
    theirs = allv.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_pack_unpack_roundtrip_and_order():
    g = torch.Generator().manual_seed(9)
    codes = torch.randint(0, 16, (33, 64), generator=g).to(torch.uint8).numpy()
    packed = oracle.pack_int4(codes)
    assert packed.shape == (33, 32)
    assert np.array_equal(oracle.unpack_int4(packed, 64), codes)
    # code 2j in the low nibble, code 2j+1 in the high nibble
    assert np.array_equal(packed & 0xF, codes[:, 0::2]) and np.array_equal(packed >> 4, codes[:, 1::2])


# --------------------------------------------------------------------------
# The binary64 matmul against numpy, and its closed forms
# --------------------------------------------------------------------------

def test_matmul_against_numpy():
    g = torch.Generator().manual_seed(13)
    M, N, K = 5, 37, 96
    x = torch.randn(M, K, generator=g).double().numpy()
    wh = torch.randn(N, K, generator=g).double().numpy()
    y, a = oracle.matmul(x, wh)
    assert y.shape == (M, N)
    ref = x @ wh.T
    aref = np.abs(x) @ np.abs(wh).T
    assert np.all(np.abs(y - ref) <= 1e-12 * aref)
    assert np.allclose(a, aref, rtol=1e-12, atol=0)


def test_matmul_closed_forms():
    K, N = 64, 9
    g = torch.Generator().manual_seed(17)
    wh = torch.randn(N, K, generator=g).double().numpy()
    x = np.zeros((K, K))
    x[np.arange(K), np.arange(K)] = 1.0  # unit vectors pick out columns of w_hat^T
    y, a = oracle.matmul(x, wh)
    assert np.array_equal(y, wh.T) and np.array_equal(a, np.abs(wh).T)


def test_gemm_w4a16_reference_tiny():
    w = wq_inputs.tiny_weight()
    x = wq_inputs.plain_activations(1, 256, 0)
    codes, s, z = oracle.quantize_int4(w.numpy(), 128)
    y, a = oracle.gemm_w4a16(x.double().numpy(), codes, s, z, 128)
    # independent evaluation: group-wise sum of s * sum x * (q - z), binary64, numpy
    xs = x.double().numpy()[0]
    ref = np.zeros(w.shape[0])
    for gi in range(2):
        sl = slice(gi * 128, (gi + 1) * 128)
        ref += s[:, gi].astype(np.float64) * ((codes[:, sl].astype(np.float64) - z[:, gi:gi + 1]) @ xs[sl])
    assert np.all(np.abs(y[0] - ref) <= 1e-12 * a[0])


# --------------------------------------------------------------------------
# Symmetric INT4 (levels -7..7): "Test-time quantization ...", "The error of
# quantising an outlier with the wrong scale"; the comparison page, "The
# methods compared" (the AWQ example)
# --------------------------------------------------------------------------

def _sym_fixture():
    sc, _ = read("int4_symmetric_examples.txt")
    return sc


def _sym_group(typical, outlier=None, g=32):
    """A group whose typical magnitude is `typical` (values of both signs, the largest exactly `typical`),
    plus one channel of magnitude |outlier| placed on the negative side."""
    base = np.array([1.0, -1.0, 0.75, -0.5, 0.25, -0.875, 0.625, -0.125], dtype=np.float32) * typical
    w = np.resize(base, g).astype(np.float32)
    if outlier is not None:
        w[3] = -outlier
    return w[None, :]


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_sym_int4_shared_scale_with_outlier(mode):
    """One 30x channel sets the scale: s = 30 / 7 (printed 4.29), half a step 2.14, so a value of
    magnitude 1 may be off by up to 214 %; every error stays within half a step."""
    sc = _sym_fixture()
    w = _sym_group(scalar(sc, "typical_magnitude"), scalar(sc, "outlier_magnitude"))
    codes, s = oracle.quantize_int4_sym(w, w.shape[1], mode)
    s0 = float(s[0, 0])
    if mode == oracle.EXACT:
        assert round(s0, 2) == scalar(sc, "s_shared_printed")
        assert round(s0 / 2, 2) == scalar(sc, "half_step_shared_printed")
        assert round(100 * (s0 / 2) / scalar(sc, "typical_magnitude")) == scalar(sc, "rel_error_shared_percent_printed")
    else:
        assert abs(s0 - 30.0 / 7) <= U_BF16 * 30.0 / 7
    q = codes[0].astype(np.int64) - 8
    assert q.min() >= -7 and q.max() <= 7 and q[3] == -7
    w_hat = q * np.float64(s0)
    assert np.all(np.abs(w_hat - w[0]) <= 0.5 * s0 * (1 + 1e-6))
    # the typical values all collapse onto the levels 0 and +-1 of the inflated scale
    assert set(np.unique(np.delete(q, 3))) <= {-1, 0, 1}


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_sym_int4_segregated_scale(mode):
    """Without the outlier (M = 1): s = 1/7 (printed 0.143), half a step 0.071, about 7 % of a value of
    magnitude 1."""
    sc = _sym_fixture()
    w = _sym_group(scalar(sc, "typical_magnitude"))
    codes, s = oracle.quantize_int4_sym(w, w.shape[1], mode)
    s0 = float(s[0, 0])
    if mode == oracle.EXACT:
        assert round(s0, 3) == scalar(sc, "s_segregated_printed")
        assert round(s0 / 2, 3) == scalar(sc, "half_step_segregated_printed")
        assert round(100 * s0 / 2) == scalar(sc, "rel_error_segregated_percent_printed")
    q = codes[0].astype(np.int64) - 8
    assert np.all(np.abs(q * np.float64(s0) - w[0]) <= 0.5 * s0 * (1 + 1e-6))
    assert q[0] == 7 and q[1] == -7  # +-1, the largest magnitude, sit on the end levels


def _awq():
    sc = _sym_fixture()
    w = np.array([[float(v) for v in sc["awq_weights"][0]]], dtype=np.float32)
    x = np.array([float(v) for v in sc["awq_activations"][0]])
    return sc, w, x


def test_sym_int4_awq_example_codes():
    """Codes of the AWQ example (the page's table is lost; recomputed from s = max|w| / 7): within
    the printed range -7..7, the largest weight on the top level."""
    sc, w, x = _awq()
    codes, s = oracle.quantize_int4_sym(w, w.shape[1], oracle.EXACT)
    q = codes[0].astype(np.int64) - 8
    assert q.tolist() == [2, -4, 3, 7]
    assert q.min() >= scalar(sc, "awq_code_min") and q.max() <= scalar(sc, "awq_code_max")
    assert abs(float(s[0, 0]) - 0.90 / 7) < 1e-7


def test_sym_int4_awq_scaling_helps_only_the_salient_channel():
    """Scaling the salient channel (activation 10x the others) up by 2 before quantising and its
    activation down by 2 (the factor the page used is lost; 2 keeps the group maximum): the other
    channels' codes and rounding errors do not change, the salient channel's error in the output falls,
    and so does the output error."""
    sc, w, x = _awq()
    g = w.shape[1]
    codes, s = oracle.quantize_int4_sym(w, g, oracle.EXACT)
    w_hat = (codes[0].astype(np.float64) - 8) * float(s[0, 0])
    f = np.array([2.0, 1.0, 1.0, 1.0])
    ws = (w * f).astype(np.float32)
    codes2, s2 = oracle.quantize_int4_sym(ws, g, oracle.EXACT)
    assert float(s2[0, 0]) == float(s[0, 0])  # the group maximum, 0.90, is unchanged
    w_hat2 = (codes2[0].astype(np.float64) - 8) * float(s2[0, 0]) / f  # effective weights seen by x
    assert codes2[0, 1:].tolist() == codes[0, 1:].tolist()
    assert np.allclose(w_hat2[1:] - w[0, 1:], w_hat[1:] - w[0, 1:])
    assert abs(w_hat2[0] - w[0, 0]) < abs(w_hat[0] - w[0, 0])
    y = float(x @ w[0].astype(np.float64))
    assert abs(float(x @ w_hat2) - y) < abs(float(x @ w_hat) - y)


@pytest.mark.parametrize("g", [8, 32, 128])
def test_sym_int4_error_at_most_half_scale(g):
    w = _groups(61, 2000 // g * 8, g)
    codes, s = oracle.quantize_int4_sym(w, g, oracle.EXACT)
    q = codes.astype(np.float64) - 8
    err = np.abs(q * np.repeat(s.astype(np.float64), g, axis=1) - w.astype(np.float64))
    assert np.all(err <= 0.5 * np.repeat(s.astype(np.float64), g, axis=1) * (1 + 1e-5))
    # the largest magnitude of every group sits on +-7
    idx = np.abs(w).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(w.shape[0]), idx]) == 7)


@pytest.mark.parametrize("mode", [oracle.EXACT, oracle.STORED])
def test_sym_int4_codes_are_nearest_levels(mode):
    w = _groups(71, 300, 8)
    codes, s = oracle.quantize_int4_sym(w, 8, mode)
    amax = np.abs(w).max(1).astype(np.float64)
    rel = 1e-6 if mode == oracle.EXACT else U_BF16 * 1.0001
    assert np.all(np.abs(s[:, 0] - amax / 7) <= rel * amax / 7)
    levels = np.arange(-7, 8, dtype=np.float64)
    for i in range(w.shape[0]):
        t = w[i].astype(np.float64) / float(s[i, 0])
        d = np.abs(t[:, None] - levels[None, :])
        chosen = d[np.arange(8), codes[i].astype(np.int64) - 1]
        assert np.all(chosen <= d.min(axis=1) + 1e-5)


def test_sym_int4_special_groups_and_asymmetric_decode():
    """An all-zero group gets s = 1 and code 8 (q = 0); a constant group sits on +-7; ties go to even;
    and the stored codes decode through the asymmetric INT4 formula with z = 8."""
    w = np.zeros((4, 8), dtype=np.float32)
    w[1, :] = -0.25
    w[2, :] = np.array([7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5])  # s = 1 exactly, halves tie
    w[3, :] = np.array([0.3, -0.1, 0.7, 0.05, -0.6, 0.2, 0.45, -0.35])
    for mode in (oracle.EXACT, oracle.STORED):
        codes, s = oracle.quantize_int4_sym(w, 8, mode)
        q = codes.astype(np.int64) - 8
        assert s[0, 0] == 1.0 and q[0].tolist() == [0] * 8
        assert q[1].tolist() == [-7] * 8
        assert s[2, 0] == 1.0 and q[2].tolist() == [7, 0, 2, 2, 0, -2, -2, 4]
        z = np.full(s.shape, 8.0, dtype=np.float32)
        assert np.array_equal(oracle.dequant_int4(codes, s, z, 8), q * np.repeat(s.astype(np.float64), 8, axis=1))


# --------------------------------------------------------------------------
# KV-cache accounting (groundwork for the KV-cache row)
# --------------------------------------------------------------------------

def test_kv_cache_worked_decode_step():
    from oracle.accounting import kv_cache_bytes, decode_step_speedup
    sc, _ = read("kv_cache_accounting.txt")
    g = lambda k: scalar(sc, k)  # noqa: E731
    kv = kv_cache_bytes(int(g("layers")), int(g("kv_heads")), int(g("head_dim")), int(g("tokens")),
                        int(g("batch")), 2)
    assert round(kv / 1e9, 1) == g("kv_gb_printed")
    gain = decode_step_speedup(g("weights_fp16_gb_printed") * 1e9, g("weights_int4_gb_printed") * 1e9, kv)
    assert round(gain, 2) == g("int4_gain_printed")
    # the KV bytes dwarf the weights at this batch and context
    assert kv > 2 * g("weights_fp16_gb_printed") * 1e9


def test_kv_cache_formats():
    from oracle.accounting import kv_cache_bytes, block_bytes_per_element
    sc, _ = read("kv_cache_accounting.txt")
    bf16 = kv_cache_bytes(80, 8, 128, 1000, 1, 2)
    assert bf16 / kv_cache_bytes(80, 8, 128, 1000, 1, 1) == scalar(sc, "fp8_kv_factor_printed")
    block = int(scalar(sc, "int4_kv_block"))
    # "about 3.5": 16- or 32-bit scales (with or without a zero-point) per block of 128 give 3.56 to 3.88
    factors = [2 / block_bytes_per_element(4, block, p) for p in (16, 32, 64)]
    assert all(3.5 <= f <= 3.9 for f in factors)
    assert min(abs(f - scalar(sc, "int4_kv_factor_printed")) for f in factors) < 0.1
    assert block_bytes_per_element(4, block, 0) == 0.5


# --------------------------------------------------------------------------
# FP8 codec and per-channel FP8 quantisation (groundwork for the FP8 W8A8 row):
# "Quantization for LLM inference ...", "FP8: the Hopper/Blackwell datacenter format"
# --------------------------------------------------------------------------

def _fp8_values(fmt):
    vals = {c: oracle.fp8_decode(c, fmt) for c in range(128)}
    return {c: v for c, v in vals.items() if np.isfinite(v)}


@pytest.mark.parametrize("fmt,key", [(oracle.E4M3, "e4m3"), (oracle.E5M2, "e5m2")])
def test_fp8_ranges_and_structure(fmt, key):
    sc, _ = read("fp8_formats.txt")
    vals = _fp8_values(fmt)
    assert max(vals.values()) == scalar(sc, f"{key}_range_printed") == oracle.fp8_max(fmt)
    ebits, mbits = int(scalar(sc, f"{key}_exponent_bits")), int(scalar(sc, f"{key}_mantissa_bits"))
    bias = 2 ** (ebits - 1) - 1
    assert min(v for v in vals.values() if v > 0) == 2.0 ** (1 - bias - mbits)   # smallest subnormal
    assert oracle.fp8_decode(1 << mbits, fmt) == 2.0 ** (1 - bias)                # smallest normal
    # positive codes are ordered like their values, and negative codes mirror them
    pos = [vals[c] for c in sorted(vals)]
    assert all(a < b for a, b in zip(pos, pos[1:]))
    for c in vals:
        assert oracle.fp8_decode(c | 0x80, fmt) == -vals[c]


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_fp8_encode_nearest_ties_even_saturating(fmt):
    vals = _fp8_values(fmt)
    codes = sorted(vals)
    for c in codes:  # exact values round-trip, with either sign
        assert oracle.fp8_encode(vals[c], fmt) == c
        if vals[c] != 0:
            assert oracle.fp8_encode(-vals[c], fmt) == (c | 0x80)
    for a, b in zip(codes, codes[1:]):  # midpoints go to the even code, neighbours to the nearer value
        lo, hi = vals[a], vals[b]
        mid = np.float32((lo + hi) / 2)
        if float(mid) == (lo + hi) / 2:
            assert oracle.fp8_encode(mid, fmt) == (a if a % 2 == 0 else b)
        assert oracle.fp8_encode(np.nextafter(np.float32((lo + hi) / 2), np.float32(0)), fmt) in (a, b)
        assert oracle.fp8_encode(np.float32(lo + (hi - lo) * 0.25), fmt) == a
        assert oracle.fp8_encode(np.float32(lo + (hi - lo) * 0.75), fmt) == b
    top = max(codes)
    assert oracle.fp8_encode(1e30, fmt) == top and oracle.fp8_encode(-1e30, fmt) == (top | 0x80)


@pytest.mark.parametrize("fmt,dtype", [(oracle.E4M3, torch.float8_e4m3fn), (oracle.E5M2, torch.float8_e5m2)])
def test_fp8_encode_matches_torch(fmt, dtype):
    """torch's conversion to its FP8 types rounds to nearest even as well (it does not saturate, so only
    values within range are compared)."""
    g = torch.Generator().manual_seed(7)
    v = torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 3)
    v = v[v.abs() < oracle.fp8_max(fmt)]
    want = v.to(dtype).view(torch.uint8).numpy()
    got = np.array([oracle.fp8_encode(float(x), fmt) for x in v.numpy()], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_fp8_rows_quantisation():
    w = wq_inputs.llm_weight(64, 256, 501, dtype=torch.float32).numpy()
    w[3] = 0.0
    for fmt in (oracle.E4M3, oracle.E5M2):
        codes, s = oracle.quantize_fp8_rows(w, fmt)
        assert s[3] == 1.0 and np.all(oracle.dequant_fp8_rows(codes, s, fmt)[3] == 0.0)
        amax = np.abs(w).max(1)
        live = amax > 0
        assert np.allclose(s[live], (amax / oracle.fp8_max(fmt))[live], rtol=1e-7)
        w_hat = oracle.dequant_fp8_rows(codes, s, fmt)
        # the largest magnitude of every row lands on +-max; elsewhere the relative error is at most half
        # an ulp of the mantissa (2^-4 for E4M3, 2^-3 for E5M2) where the value is normal in the format
        idx = np.abs(w).argmax(1)
        assert np.allclose(np.abs(w_hat[np.arange(64), idx])[live], amax[live], rtol=1e-6)
        mbits = 3 if fmt == oracle.E4M3 else 2
        min_normal = oracle.fp8_decode(1 << mbits, fmt)
        normal = np.abs(w) / s[:, None] >= min_normal
        rel = np.abs(w_hat - w)[normal] / np.abs(w)[normal]
        assert rel.max() <= 2.0 ** -(mbits + 1) * (1 + 1e-6)


def test_fp8_w8a8_reference():
    """The W8A8 reference: the exact product of the decoded operands; close to the unquantised product
    within the formats' half-ulp (E4M3: 2^-4 relative per operand, so about 2^-3 on sum|x w|)."""
    x = wq_inputs.plain_activations(4, 256, 503).float().numpy()
    w = wq_inputs.llm_weight(32, 256, 504, dtype=torch.float32).numpy()
    y, a = oracle.gemm_w8a8_fp8(x, w)
    xc, sx = oracle.quantize_fp8_tensor(x)
    assert xc.shape == x.shape and sx == np.float32(np.abs(x).max() / 448.0)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    bound = np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T
    assert np.all(np.abs(y - exact) <= 2.0 ** -3 * bound + 1e-12)
    assert np.all(a <= bound * (1 + 2.0 ** -3))


# --------------------------------------------------------------------------
# NVFP4 (groundwork for the NVFP4 row): the comparison page, "Hardware, formats and the roofline", and
# "Quantization for LLM inference ...", "Microscaling: NVFP4 and MXFP4"
# --------------------------------------------------------------------------

def test_e2m1_values_and_rounding():
    mags = [oracle.e2m1_decode(c) for c in range(8)]
    # sign, 2 exponent bits with bias 1, 1 mantissa bit; exponent 0 is subnormal (0 and 0.5)
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert [oracle.e2m1_decode(c | 8) for c in range(8)] == [-m for m in mags]
    for c, v in enumerate(mags):
        assert oracle.e2m1_encode(v) == c
    for a in range(7):  # midpoints to the even code, quarter points to the nearer value
        lo, hi = mags[a], mags[a + 1]
        assert oracle.e2m1_encode((lo + hi) / 2) == (a if a % 2 == 0 else a + 1)
        assert oracle.e2m1_encode(lo + (hi - lo) / 4) == a and oracle.e2m1_encode(lo + 3 * (hi - lo) / 4) == a + 1
    assert oracle.e2m1_encode(100.0) == 7 and oracle.e2m1_encode(-100.0) == 15


def test_nvfp4_blocks_and_scales():
    from oracle.accounting import bits_per_weight
    w = wq_inputs.llm_weight(24, 256, 601, dtype=torch.float32).numpy()
    w[2] = 0.0
    w[5, 16:32] *= 40.0   # one loud block
    codes, blocks, st = oracle.quantize_nvfp4(w)
    assert codes.shape == w.shape and blocks.shape == (24, 256 // 16)
    assert st == np.float32(np.abs(w).max() / (6.0 * 448.0))          # block scales fit E4M3
    w_hat = oracle.dequant_nvfp4(codes, blocks, st)
    assert np.all(w_hat[2] == 0.0)
    S = np.array([[oracle.fp8_decode(b, oracle.E4M3) for b in row] for row in blocks]) * st
    wb = np.abs(w).reshape(24, 16, 16).max(-1)
    live = wb > 0
    # each block scale is its max / 6 up to E4M3 rounding (half an ulp: 2^-4 relative)
    assert np.all(np.abs(S[live] - wb[live] / 6) <= 2.0 ** -4 * wb[live] / 6 * (1 + 1e-6))
    # every block's largest magnitude lands on the top value 6; every error is within one block scale
    vals = np.abs(np.vectorize(oracle.e2m1_decode)(codes)).reshape(24, 16, 16)
    idx = np.abs(w).reshape(24, 16, 16).argmax(-1)
    top = np.take_along_axis(vals, idx[..., None], -1)[..., 0]
    assert np.all(top[live] == 6.0)
    assert np.all(np.abs(w_hat - w) <= np.repeat(S, 16, axis=1) * (1 + 1e-6))
    # 4-bit values plus an 8-bit scale per 16: the printed 4.5 bits per weight
    assert bits_per_weight(4, 16, 8, 0) == 4.5


def test_nvfp4_w4a4_reference():
    """The NVFP4 matmul reference: the binary64 product of operands decoded from their codes with a table
    of the eight E2M1 magnitudes (the microscaling formats' 4-bit element, Rouhani et al., cited by the
    page's "Microscaling: NVFP4 and MXFP4") and torch's E4M3 decode; within one block scale per operand
    of the unquantised product."""
    x = wq_inputs.plain_activations(4, 256, 605).float().numpy()
    w = wq_inputs.llm_weight(32, 256, 606, dtype=torch.float32).numpy()
    y, a = oracle.gemm_nvfp4(x, w)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

    def decode(v):
        c, b, st = oracle.quantize_nvfp4(v)
        vals = np.where(c & 8, -1.0, 1.0) * mags[c & 7]
        S = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy() * st
        return vals * np.repeat(S, 16, axis=1), np.repeat(S, 16, axis=1)

    xd, sx = decode(x)
    wd, sw = decode(w)
    np.testing.assert_allclose(y, xd @ wd.T, rtol=1e-13, atol=1e-13)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    bound = np.abs(x) @ sw.T + sx @ np.abs(w).T + sx @ sw.T
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-9))
    assert np.all(np.abs(y) <= a * (1 + 1e-12))


def test_roofline_closed_forms():
    """[P3] "Hardware, formats and the roofline": ridge 1,000 / 3.3 = 303 flop/B; fp16 intensity = batch
    (memory-bound to about 300); 4-bit intensity 4 x batch (crossing near 76); the worked 70B step at batch
    128 on 8 GPUs computes for about 2.2 ms."""
    from oracle.accounting import crossover_batch, decode_compute_seconds, decode_intensity, ridge_point
    sc, _ = read("roofline_closed_forms.txt")
    ridge = ridge_point(scalar(sc, "tflops_assumed") * 1e12, scalar(sc, "tbs_assumed") * 1e12)
    assert round(ridge) == scalar(sc, "ridge_printed")
    assert decode_intensity(128, 2.0) == 128 and decode_intensity(128, 0.5) == 4 * 128
    assert abs(crossover_batch(ridge, 2.0) - scalar(sc, "fp16_crossover_printed")) < 5   # "about 300"
    assert round(crossover_batch(ridge, 0.5)) == scalar(sc, "int4_crossover_printed")
    n = scalar(sc, "gpus")
    assert round(n * scalar(sc, "tbs_assumed"), 1) == scalar(sc, "aggregate_tbs_printed")
    assert n * scalar(sc, "tflops_assumed") == scalar(sc, "aggregate_tflops_printed")
    t = decode_compute_seconds(scalar(sc, "params"), int(scalar(sc, "batch")),
                               scalar(sc, "aggregate_tflops_printed") * 1e12)
    assert round(t * 1e3, 1) == scalar(sc, "compute_ms_printed")
