"""KV-cache quantisation and the decode-attention read of a quantised cache (test infrastructure).

Only the test suite may import this; the CUDA library never does, and nothing here imports it.

What the pages fix, cited by page title and section:
  * "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF" -- "KV cache quantization":
    a bf16 cache holds 2 bytes per dimension for every head and head dimension, for K and for V; an
    fp8 cache (E4M3 or E5M2) holds one byte; an int4 cache works in blocks of 128 values, half a
    byte each plus the scale overhead.  Cache and weight quantisation are independent choices.
  * "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization" --
    "Hardware, formats and the roofline": every decode step reads the whole cache of every sequence,
    and at batch 128 with 8,000-token contexts those reads outweigh the weights.

Readings (the pages give neither the cache layout, nor the int4 parameters, nor the read itself):
  * K and V of one layer are each a [B][T][H][D] tensor: B sequences, T token slots, H KV heads,
    D = head_dim.  K and V are quantised alike and independently.
  * int4: every (b, t, h) vector splits into blocks of 128 consecutive values along D (one block at
    head_dim 128), and each block takes the weight format unchanged: asymmetric INT4 with a bf16
    scale and a bf16 zero-point (the same arithmetic as the weight quantiser, applied to the cache
    viewed as rows of D values).  That is 0.5 + 4/128 bytes per value, 3.76x smaller than bf16.
  * fp8: one binary32 scale per tensor, max|x| / max_fmt, and the nearest FP8 code of x / scale.
  * The read is decode attention (scaled dot-product attention, Vaswani et al., "Attention Is All
    You Need", 2017, section 3.2.1) of one new query token per sequence over the first len_b cached
    tokens: score_t = (q . k_t) / sqrt(D), p = softmax(score), o = sum_t p_t v_t.  With grouped
    query heads (Hq = r * H), query head h reads KV head h // r.  A sequence with len_b = 0 reads
    nothing and its output is 0.
All arithmetic after dequantisation is binary64.
"""
from __future__ import annotations

import math

import numpy as np

import oracle

KV_BLOCK = 128


def _rows(cache):
    c = np.ascontiguousarray(cache, dtype=np.float32)
    if c.ndim != 4:
        raise ValueError("kv cache must be [B][T][H][D]")
    return c.reshape(-1, c.shape[3]), c.shape


def quantize_kv_int4(cache, block: int = KV_BLOCK):
    """Asymmetric INT4 per block of `block` values along head_dim.

    Returns (codes uint8 [B][T][H][D] in 0..15, s float32 [B][T][H][D/block], z float32 same)."""
    rows, shape = _rows(cache)
    if shape[3] % block:
        raise ValueError("head_dim must be a multiple of the block")
    codes, s, z = oracle.quantize_int4(rows, block, oracle.STORED)
    nb = shape[3] // block
    return codes.reshape(shape), s.reshape(shape[:3] + (nb,)), z.reshape(shape[:3] + (nb,))


def dequant_kv_int4(codes, s, z, block: int = KV_BLOCK) -> np.ndarray:
    """k_hat = s * (q - z) per block, binary64 [B][T][H][D]."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    shape = c.shape
    nb = shape[3] // block
    out = oracle.dequant_int4(c.reshape(-1, shape[3]), np.reshape(s, (-1, nb)), np.reshape(z, (-1, nb)), block)
    return out.reshape(shape)


def quantize_kv_fp8(cache, fmt: int = oracle.E4M3):
    """One binary32 scale for the tensor, FP8 codes of x / scale.  Returns (codes uint8 [B][T][H][D], s)."""
    c = np.ascontiguousarray(cache, dtype=np.float32)
    return oracle.quantize_fp8_tensor(c, fmt)


def dequant_kv_fp8(codes, s, fmt: int = oracle.E4M3) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = oracle.dequant_fp8_rows(c.reshape(1, -1), np.array([s], dtype=np.float32), fmt)
    return out.reshape(c.shape)


def decode_attention(q, k_hat, v_hat, lengths):
    """One query token per sequence against its first lengths[b] cached tokens.

    q: [B][Hq][D]; k_hat, v_hat: [B][T][H][D] (dequantised, any float type); lengths: [B] ints.
    Returns (o, a), both binary64 [B][Hq][D]: o = sum_t p_t v_t, and a = sum_t p_t |v_t|, the scale
    against which a kernel's rounding error is measured (|o| <= a).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k_hat, dtype=np.float64)
    v = np.asarray(v_hat, dtype=np.float64)
    B, Hq, D = q.shape
    H = k.shape[2]
    if Hq % H:
        raise ValueError("query heads must be a multiple of the KV heads")
    r = Hq // H
    o = np.zeros((B, Hq, D))
    a = np.zeros((B, Hq, D))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        for h in range(Hq):
            kv = h // r
            score = k[b, :n, kv, :] @ q[b, h] / math.sqrt(D)
            e = np.exp(score - score.max())
            p = e / e.sum()
            o[b, h] = p @ v[b, :n, kv, :]
            a[b, h] = p @ np.abs(v[b, :n, kv, :])
    return o, a


def cache_bytes_per_value(kind: str, block: int = KV_BLOCK) -> float:
    """Bytes each cached value occupies in the formats above (scales of the fp8 tensor amortised away)."""
    if kind == "bf16":
        return 2.0
    if kind == "fp8":
        return 1.0
    if kind == "int4":
        return 0.5 + 4.0 / block
    raise ValueError(kind)
