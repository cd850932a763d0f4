"""Pins for the KV-cache oracle: the int4 and fp8 cache formats and the decode-attention read.

Each pin checks the oracle against what the pages or the mathematics fix, never against itself:
the page's worked INT4 example laid out as a 128-value cache block, per-block scales recomputed
from the block's own extremes, the page's storage figures, FP8 error bounds and torch's FP8
conversion, and closed forms of attention (a zero query averages, one token returns itself, the
e / (1 + e) two-token case that fixes the 1/sqrt(D) factor, constant values per KV head that fix
the query-head mapping, invariance to what lies beyond a sequence's length, convexity).  The
planted mistakes at the end must each fail at least one pin.  CPU only.
"""
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle
import oracle.kv_cache as kv
from oracle.accounting import block_bytes_per_element
from golden import read, scalar


def _cache(seed, B, T, H, D, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, T, H, D, generator=g) * std).to(torch.bfloat16).float().numpy()


def _bf16(x32):
    return float(torch.tensor(np.float32(x32)).to(torch.bfloat16).float())


def test_int4_block_holds_the_page_example():
    """[P2] "Numerical example": the 8 weights repeated 16 times form one 128-value block with the
    same extremes, so the block takes the page's s, z and codes."""
    sc, rows = read("int4_worked_example.txt")
    w = np.array([float(r[0]) for r in rows], dtype=np.float32)
    cache = np.tile(w, 16).reshape(1, 1, 1, 128)
    codes, s, z = kv.quantize_kv_int4(cache)
    assert codes.shape == (1, 1, 1, 128) and s.shape == (1, 1, 1, 1)
    assert list(codes[0, 0, 0, :8]) == [int(r[3]) for r in rows]
    assert (codes.reshape(16, 8) == codes[0, 0, 0, :8]).all()
    assert z[0, 0, 0, 0] == scalar(sc, "z_printed")
    assert round(float(s[0, 0, 0, 0]), 4) == scalar(sc, "s_printed")
    w_hat = kv.dequant_kv_int4(codes, s, z)
    # the printed w_hat use s = 2.33 / 15; the cache stores s in bf16, which moves 9 s by 5e-4
    assert np.abs(w_hat[0, 0, 0, :8] - [float(r[4]) for r in rows]).max() <= 1.1e-3


def test_int4_blocks_run_along_head_dim():
    """Every (sequence, token, head) vector splits into blocks of 128 along head_dim: each block's
    scale is bf16((max - min) / 15) of that block alone, its zero-point the rounded -min / s, and
    every value decodes within the stored-parameter half-step bound."""
    B, T, H, D = 2, 128, 2, 256
    cache = _cache(11, B, T, H, D)
    cache[0, 3, 1, 130] = 30.0         # an outlier moves one block's scale only
    codes, s, z = kv.quantize_kv_int4(cache)
    assert s.shape == (B, T, H, 2)
    k_hat = kv.dequant_kv_int4(codes, s, z)
    u = 2.0 ** -8
    for b in range(B):
        for t in (0, 3, 77, 127):
            for h in range(H):
                for j in range(2):
                    blk = cache[b, t, h, 128 * j:128 * (j + 1)]
                    mx, mn = np.float32(blk.max()), np.float32(blk.min())
                    want_s = _bf16(np.float32(mx - mn) / np.float32(15.0))
                    assert s[b, t, h, j] == want_s
                    assert z[b, t, h, j] == _bf16(np.rint(np.float32(-mn) / np.float32(want_s)))
                    err = np.abs(k_hat[b, t, h, 128 * j:128 * (j + 1)] - blk)
                    assert err.max() <= (0.5 + 15 * u / (1 - u)) * want_s * (1 + 1e-5)
    assert s[0, 3, 1, 1] > 4 * s[0, 3, 1, 0]


def test_int4_cache_storage_matches_the_page():
    """[P1] "KV cache quantization": half a byte per value plus the block's parameters, dividing a bf16
    cache by about 3.5 (read as 16- to 64-bit parameters per block of 128: 3.56 to 3.88)."""
    sc, _ = read("kv_cache_accounting.txt")
    per_value = kv.cache_bytes_per_value("int4")
    assert per_value == block_bytes_per_element(4, int(scalar(sc, "int4_kv_block")), 32)
    ratio = kv.cache_bytes_per_value("bf16") / per_value
    assert 3.56 <= ratio <= 3.88 and abs(ratio - scalar(sc, "int4_kv_factor_printed")) < 0.4
    assert kv.cache_bytes_per_value("bf16") / kv.cache_bytes_per_value("fp8") == scalar(sc, "fp8_kv_factor_printed")
    cache = _cache(3, 1, 4, 2, 128)
    codes, s, z = kv.quantize_kv_int4(cache)
    stored = codes.size // 2 + 2 * s.size + 2 * z.size      # packed nibbles, bf16 s and z
    assert stored / cache.size == per_value


@pytest.mark.parametrize("fmt,dtype", [(oracle.E4M3, torch.float8_e4m3fn), (oracle.E5M2, torch.float8_e5m2)])
def test_fp8_cache_scale_and_codes(fmt, dtype):
    """One binary32 scale per tensor, max|x| / max_fmt; the codes are torch's FP8 conversion of x / s
    and decode within half a step of x."""
    cache = _cache(5, 2, 16, 2, 128)
    cache[1, 2, 0, 5] = -7.5
    codes, s = kv.quantize_kv_fp8(cache, fmt)
    assert s == np.float32(np.float32(7.5) / np.float32(oracle.fp8_max(fmt)))
    want = torch.from_numpy((cache / np.float32(s)).astype(np.float32)).to(dtype).view(torch.uint8).numpy()
    assert (codes == want).all()
    x_hat = kv.dequant_kv_fp8(codes, s, fmt)
    mbits = 3 if fmt == oracle.E4M3 else 2
    tiny = 2.0 ** (1 - (7 if fmt == oracle.E4M3 else 15)) * float(s)   # smallest normal, scaled
    err = np.abs(x_hat - cache)
    assert (err <= np.maximum(np.abs(cache) * 2.0 ** -(mbits + 1), tiny * 2.0 ** -(mbits + 1)) * (1 + 1e-6)).all()


def test_zero_query_averages_the_values():
    """q = 0 gives equal scores, so every head returns the plain mean of its first len_b values."""
    B, T, H, D = 3, 9, 2, 32
    k, v = _cache(1, B, T, H, D), _cache(2, B, T, H, D)
    lengths = [5, 1, 9]
    o, a = kv.decode_attention(np.zeros((B, 2 * H, D)), k, v, lengths)
    for b in range(B):
        for h in range(2 * H):
            np.testing.assert_allclose(o[b, h], v[b, :lengths[b], h // 2].astype(np.float64).mean(axis=0),
                                       rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(a[b, h], np.abs(v[b, :lengths[b], h // 2].astype(np.float64)).mean(axis=0), rtol=1e-13)


def test_one_token_returns_its_value():
    k, v = _cache(3, 2, 4, 1, 64), _cache(4, 2, 4, 1, 64)
    q = _cache(5, 1, 2, 3, 64)[0]
    o, _ = kv.decode_attention(q, k, v, [1, 1])
    for b in range(2):
        for h in range(3):
            assert (o[b, h] == v[b, 0, 0]).all()


@pytest.mark.parametrize("D", [16, 64, 128])
def test_scores_scaled_by_sqrt_head_dim(D):
    """q = sqrt(D) e0, k0 = e0, k1 = 0: the scores are 1 and 0 only under the 1/sqrt(D) factor, so the
    first token's weight is e / (1 + e)."""
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = math.sqrt(D)
    k = np.zeros((1, 2, 1, D))
    k[0, 0, 0, 0] = 1.0
    v = np.zeros((1, 2, 1, D))
    v[0, 0, 0, :] = 1.0
    o, _ = kv.decode_attention(q, k, v, [2])
    assert np.allclose(o[0, 0], math.e / (1 + math.e), rtol=1e-14, atol=0)


def test_query_heads_share_consecutive_kv_heads():
    """Values constant per KV head (head j holds j + 1 everywhere): with 8 query heads over 2 KV heads,
    query head h must return h // 4 + 1 whatever the keys."""
    B, T, H, D = 2, 6, 2, 16
    k = _cache(6, B, T, H, D)
    v = np.ones((B, T, H, D)) * (np.arange(H) + 1.0)[None, None, :, None]
    o, _ = kv.decode_attention(_cache(7, 1, B, 8, D)[0], k, v, [6, 4])
    for h in range(8):
        assert np.allclose(o[:, h], h // 4 + 1, rtol=1e-14, atol=0)


def test_tokens_beyond_length_are_ignored():
    B, T, H, D = 3, 12, 2, 32
    k, v = _cache(8, B, T, H, D), _cache(9, B, T, H, D)
    q = _cache(10, 1, B, 4, D)[0]
    lengths = [7, 12, 0]
    k2, v2 = k.copy(), v.copy()
    for b, n in enumerate(lengths):
        k2[b, n:] = 1e6
        v2[b, n:] = -1e6
    o1, a1 = kv.decode_attention(q, k, v, lengths)
    o2, a2 = kv.decode_attention(q, k2, v2, lengths)
    assert (o1 == o2).all() and (a1 == a2).all()
    assert (o1[2] == 0).all() and (a1[2] == 0).all()       # an empty sequence reads nothing


def test_large_scores_select_the_best_token():
    """Scores of 800, 600 and -400: softmax puts all weight on the best-matching key, with no overflow."""
    D = 64
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 8.0
    k = np.zeros((1, 3, 1, D))
    k[0, :, 0, 0] = [800.0, 600.0, -400.0]   # exp(800) alone would overflow binary64
    v = _cache(12, 1, 3, 1, D)
    o, a = kv.decode_attention(q, k, v, [3])
    assert np.isfinite(o).all() and (o[0, 0] == v[0, 0, 0]).all()
    assert (a[0, 0] == np.abs(v[0, 0, 0])).all()


def test_output_is_a_convex_combination_and_order_free():
    B, T, H, D = 2, 10, 2, 32
    k, v = _cache(13, B, T, H, D), _cache(14, B, T, H, D)
    q = _cache(15, 1, B, 4, D)[0] * 3
    lengths = [10, 6]
    o, a = kv.decode_attention(q, k, v, lengths)
    for b, n in enumerate(lengths):
        for h in range(4):
            vs = v[b, :n, h // 2]
            assert (o[b, h] >= vs.min(axis=0) - 1e-12).all() and (o[b, h] <= vs.max(axis=0) + 1e-12).all()
    assert (np.abs(o) <= a + 1e-12).all()
    perm = np.random.default_rng(0).permutation(6)
    k2, v2 = k.copy(), v.copy()
    k2[1, :6], v2[1, :6] = k[1, perm], v[1, perm]
    o2, _ = kv.decode_attention(q, k2, v2, lengths)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)


def test_quantised_values_move_the_output_by_at_most_their_error():
    """With exact keys the weights p are unchanged, so |o(v_hat) - o(v)| <= max_t |v_hat - v|, and the
    int4 error is at most about half a block step."""
    B, T, H, D = 2, 32, 1, 128
    k, v = _cache(16, B, T, H, D), _cache(17, B, T, H, D)
    q = _cache(18, 1, B, 2, D)[0]
    codes, s, z = kv.quantize_kv_int4(v)
    v_hat = kv.dequant_kv_int4(codes, s, z)
    o, _ = kv.decode_attention(q, k, v, [32, 20])
    oq, _ = kv.decode_attention(q, k, v_hat, [32, 20])
    assert 0 < np.abs(oq - o).max() <= np.abs(v_hat - v).max() * (1 + 1e-12)
    assert np.abs(v_hat - v).max() <= 0.56 * s.max()


def test_fp8_cache_read_error_and_zero_cache():
    """E4M3 with a per-tensor scale: with exact keys, each output moves by at most the largest value error,
    itself at most 2^-4 relative (half a step of a 3-bit mantissa) above the subnormal range; an all-zero
    cache takes the scale 1 and reads back zeros."""
    B, T, H, D = 2, 24, 1, 128
    k, v = _cache(19, B, T, H, D), _cache(20, B, T, H, D)
    q = _cache(21, 1, B, 2, D)[0]
    codes, s = kv.quantize_kv_fp8(v)
    v_hat = kv.dequant_kv_fp8(codes, s)
    o, _ = kv.decode_attention(q, k, v, [24, 9])
    oq, _ = kv.decode_attention(q, k, v_hat, [24, 9])
    verr = np.abs(v_hat - v)
    assert 0 < np.abs(oq - o).max() <= verr.max() * (1 + 1e-12)
    normal = np.abs(v) >= 2.0 ** -6 * float(s)
    assert (verr[normal] <= 2.0 ** -4 * np.abs(v[normal]) * (1 + 1e-6)).all()
    zc, zs = kv.quantize_kv_fp8(np.zeros((1, 4, 1, D), dtype=np.float32))
    assert zs == 1.0 and not zc.any() and not kv.dequant_kv_fp8(zc, zs).any()


PINS = [test_int4_block_holds_the_page_example, test_int4_blocks_run_along_head_dim,
        test_int4_cache_storage_matches_the_page,
        lambda: [test_fp8_cache_scale_and_codes(f, d) for f, d in
                 ((oracle.E4M3, torch.float8_e4m3fn), (oracle.E5M2, torch.float8_e5m2))],
        test_zero_query_averages_the_values, test_one_token_returns_its_value,
        lambda: [test_scores_scaled_by_sqrt_head_dim(d) for d in (16, 64, 128)],
        test_query_heads_share_consecutive_kv_heads, test_tokens_beyond_length_are_ignored,
        test_large_scores_select_the_best_token, test_output_is_a_convex_combination_and_order_free,
        test_quantised_values_move_the_output_by_at_most_their_error, test_fp8_cache_read_error_and_zero_cache]

MUTANTS = {
    "no_sqrt_scale": ("score = k[b, :n, kv, :] @ q[b, h] / math.sqrt(D)", "score = k[b, :n, kv, :] @ q[b, h]"),
    "scale_by_head_dim": ("/ math.sqrt(D)", "/ D"),
    "query_heads_interleaved": ("kv = h // r", "kv = h % H"),
    "ignores_length": ("n = int(lengths[b])", "n = k.shape[1] if int(lengths[b]) else 0"),
    "no_max_shift": ("np.exp(score - score.max())", "np.exp(score)"),
    "unnormalised_weights": ("p = e / e.sum()", "p = e / e.max()"),
    "bound_drops_abs": ("a[b, h] = p @ np.abs(v[b, :n, kv, :])", "a[b, h] = p @ v[b, :n, kv, :]"),
    "blocks_along_tokens": ("return c.reshape(-1, c.shape[3]), c.shape",
                            "return np.ascontiguousarray(c.transpose(0, 2, 3, 1)).reshape(-1, c.shape[1]), c.shape"),
    "dequant_drops_zero_point": ("np.reshape(s, (-1, nb)), np.reshape(z, (-1, nb))",
                                 "np.reshape(s, (-1, nb)), 0 * np.reshape(z, (-1, nb))"),
    "fp8_wrong_format": ("return oracle.quantize_fp8_tensor(c, fmt)", "return oracle.quantize_fp8_tensor(c, 1 - fmt)"),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_mutant(mutant, monkeypatch):
    src = open(kv.__file__).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, f"mutation site for {mutant} not found"
    mod = types.ModuleType("kv_cache_mutant")
    mod.__file__ = os.path.join(os.path.dirname(kv.__file__), "kv_cache_mutant.py")
    exec(compile(src.replace(old, new), mod.__file__, "exec"), mod.__dict__)
    monkeypatch.setitem(globals(), "kv", mod)
    failures = 0
    with np.errstate(all="ignore"):          # a mutant may overflow; that is one way to fail
        for p in PINS:
            try:
                p()
            except Exception:
                failures += 1
    assert failures > 0, f"no pin caught {mutant}"
