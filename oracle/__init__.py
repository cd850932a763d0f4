"""CPU oracle for group-wise weight quantisation and the weight-only matmul.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library
never imports, links or calls anything here, and nothing here imports the
CUDA library.  The arithmetic lives in ``wq_oracle.c`` (plain C, built with
gcc, binary32 quantisation with round-half-to-even, binary64 dequantisation
and matmul); this module only marshals numpy arrays in and out of it.

Sources, by page title and section:
  * "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF" --
    "The minimum maths: scale and zero-point" (s, z, encode, decode) and
    "Numerical example" (the 8-weight table and the storage count).
  * "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
    Quantization" -- "What quantisation does" (symmetric absmax INT8, the
    outlier example, granularity and bits per weight).
  * "Test-time quantization: quantising on the fly with no calibration
    dataset" -- "The error of quantising an outlier with the wrong scale"
    (rounding error at most half a scale; the symmetric scale M / 7 at 4 bits).
  * The same comparison page -- "The methods compared" (the AWQ example:
    symmetric int4 with codes -7 to 7).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(page values, closed forms, brute force, invariants, an independent binary64
matmul); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .accounting import bits_per_weight, model_gigabytes, example_bytes  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

EXACT = 0   # s and z kept in binary32 (the pages' arithmetic)
STORED = 1  # s and z rounded to bf16 before encoding (the library's format)

_lib = None


def build(force: bool = False) -> str:
    """Compile wq_oracle.c into liboracle.so with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _bind(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_quantize_int4.argtypes = [P, I64, I64, I64, I64, I, P, P, P]
    lib.oracle_quantize_int8.argtypes = [P, I64, I64, I64, I64, I, P, P]
    lib.oracle_quantize_int4_sym.argtypes = [P, I64, I64, I64, I64, I, P, P]
    lib.oracle_fp8_decode.argtypes = [ctypes.c_uint8, I]
    lib.oracle_fp8_decode.restype = ctypes.c_double
    lib.oracle_fp8_encode.argtypes = [ctypes.c_float, I]
    lib.oracle_fp8_encode.restype = ctypes.c_uint8
    lib.oracle_fp8_max.argtypes = [I]
    lib.oracle_fp8_max.restype = ctypes.c_double
    lib.oracle_quantize_fp8_rows.argtypes = [P, I64, I64, I64, I, P, P]
    lib.oracle_dequant_fp8_rows.argtypes = [P, P, I64, I64, I, P]
    lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_decode.restype = ctypes.c_double
    lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
    lib.oracle_e2m1_encode.restype = ctypes.c_uint8
    lib.oracle_quantize_nvfp4.argtypes = [P, I64, I64, I64, P, P, P]
    lib.oracle_dequant_nvfp4.argtypes = [P, P, ctypes.c_float, I64, I64, P]
    lib.oracle_pack_int4.argtypes = [P, I64, I64, P]
    lib.oracle_unpack_int4.argtypes = [P, I64, I64, P]
    lib.oracle_dequant_int4.argtypes = [P, P, P, I64, I64, I64, P]
    lib.oracle_dequant_int8.argtypes = [P, P, I64, I64, I64, P]
    lib.oracle_matmul.argtypes = [P, P, I64, I64, I64, P, P]
    lib.oracle_f32_to_bf16_array.argtypes = [P, I64, P]
    lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_set_threads.argtypes = [I]
    lib.oracle_max_threads.restype = I
    for name in ("oracle_quantize_int4", "oracle_quantize_int8", "oracle_pack_int4",
                 "oracle_unpack_int4", "oracle_dequant_int4", "oracle_dequant_int8",
                 "oracle_matmul"):
        getattr(lib, name).restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def swap_library(path):
    """Make the wrappers call the oracle compiled at ``path`` (None: the default build).

    Returns the previously bound library handle.  Used only by the mutation
    tests, which compile deliberately broken copies of wq_oracle.c and check
    that the pins reject them.
    """
    global _lib
    old = _lib
    _lib = _bind(path) if path is not None else None
    return old


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")


def set_threads(n: int) -> None:
    """Number of OpenMP threads the oracle's outer loops use (rows / outputs)."""
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def bf16_bits(values) -> np.ndarray:
    """binary32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_f32_to_bf16_array(_ptr(v), v.size, _ptr(out))
    return out


def bf16_value(bits) -> np.ndarray:
    """bf16 bit patterns -> binary32 values (exact widening)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def quantize_int4(w, g: int, mode: int = STORED):
    """Asymmetric INT4 per group of ``g`` consecutive weights along a row.

    w: [N][K] binary32 values (bf16 weights widened exactly).
    Returns (codes uint8 [N][K] in 0..15, s float32 [N][K/g], z float32 [N][K/g]);
    s and z are the values the codes were encoded against (bf16-representable in
    STORED mode).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N, K // g), dtype=np.float32)
    z = np.empty((N, K // g), dtype=np.float32)
    _check(_load().oracle_quantize_int4(_ptr(w), N, K, K, g, mode, _ptr(codes), _ptr(s), _ptr(z)),
           "quantize_int4")
    return codes, s, z


def quantize_int4_sym(w, g: int, mode: int = STORED):
    """Symmetric INT4 per group of ``g`` weights: s = max|w| / 7, q = clip(round(w / s), -7, 7).

    Returns (codes uint8 [N][K] holding q + 8 in 1..15, s float32 [N][K/g]); the codes decode as
    s * (code - 8), i.e. as asymmetric INT4 with z = 8.
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N, K // g), dtype=np.float32)
    _check(_load().oracle_quantize_int4_sym(_ptr(w), N, K, K, g, mode, _ptr(codes), _ptr(s)),
           "quantize_int4_sym")
    return codes, s


E4M3 = 0  # FP8 formats
E5M2 = 1


def fp8_decode(code: int, fmt: int) -> float:
    return float(_load().oracle_fp8_decode(int(code) & 0xff, fmt))


def fp8_encode(v: float, fmt: int) -> int:
    return int(_load().oracle_fp8_encode(float(v), fmt))


def fp8_max(fmt: int) -> float:
    return float(_load().oracle_fp8_max(fmt))


def quantize_fp8_rows(w, fmt: int = E4M3):
    """FP8 per output channel: s = max|w| / max_fmt per row, codes = nearest FP8 of w / s.
    Returns (codes uint8 [N][K], s float32 [N])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), dtype=np.uint8)
    s = np.empty(N, dtype=np.float32)
    _check(_load().oracle_quantize_fp8_rows(_ptr(w), N, K, K, fmt, _ptr(codes), _ptr(s)), "quantize_fp8_rows")
    return codes, s


def dequant_fp8_rows(codes, s, fmt: int = E4M3) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    N, K = c.shape
    out = np.empty((N, K), dtype=np.float64)
    _check(_load().oracle_dequant_fp8_rows(_ptr(c), _ptr(s), N, K, fmt, _ptr(out)), "dequant_fp8_rows")
    return out


def quantize_fp8_tensor(x, fmt: int = E4M3):
    """FP8 with one scale for the whole tensor (the pages' dynamic per-tensor scaling of activations):
    s = max|x| / max_fmt.  Returns (codes uint8, s float32 scalar)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes, s = quantize_fp8_rows(x.reshape(1, -1), fmt)
    return codes.reshape(x.shape), s[0]


def gemm_w8a8_fp8(x, w, fmt: int = E4M3):
    """Reference for an FP8 W8A8 matmul: activations quantised per tensor, weights per output channel, the
    products of the decoded values summed in binary64.  Returns (y, a) as matmul does."""
    xc, sx = quantize_fp8_tensor(x, fmt)
    wc, sw = quantize_fp8_rows(w, fmt)
    x_hat = dequant_fp8_rows(xc.reshape(1, -1), np.array([sx], dtype=np.float32), fmt).reshape(np.shape(x))
    return matmul(x_hat, dequant_fp8_rows(wc, sw, fmt))


def e2m1_decode(code: int) -> float:
    return float(_load().oracle_e2m1_decode(int(code) & 0xf))


def e2m1_encode(v: float) -> int:
    return int(_load().oracle_e2m1_encode(float(v)))


def quantize_nvfp4(w):
    """NVFP4: E2M1 values, one E4M3 scale per 16 values of a row, one binary32 tensor scale.
    Returns (codes uint8 [N][K], block_codes uint8 [N][K/16], tensor_scale float)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), dtype=np.uint8)
    blocks = np.empty((N, K // 16), dtype=np.uint8)
    st = np.empty(1, dtype=np.float32)
    _check(_load().oracle_quantize_nvfp4(_ptr(w), N, K, K, _ptr(codes), _ptr(blocks), _ptr(st)), "quantize_nvfp4")
    return codes, blocks, float(st[0])


def dequant_nvfp4(codes, block_codes, tensor_scale: float) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    b = np.ascontiguousarray(block_codes, dtype=np.uint8)
    N, K = c.shape
    out = np.empty((N, K), dtype=np.float64)
    _check(_load().oracle_dequant_nvfp4(_ptr(c), _ptr(b), tensor_scale, N, K, _ptr(out)), "dequant_nvfp4")
    return out


def gemm_nvfp4(x, w):
    """Reference for an NVFP4 W4A4 matmul: activations and weights each quantised to NVFP4 (blocks of 16
    along K, each operand with its own tensor scale), the products of the decoded values summed in
    binary64.  Returns (y, a) as matmul does."""
    xc, xb, xs = quantize_nvfp4(x)
    wc, wb, ws = quantize_nvfp4(w)
    return matmul(dequant_nvfp4(xc, xb, xs), dequant_nvfp4(wc, wb, ws))


def pack_int4(codes) -> np.ndarray:
    """[N][K] codes -> [N][K/2] bytes, code 2j in the low nibble of byte j."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = c.shape
    out = np.empty((N, K // 2), dtype=np.uint8)
    _check(_load().oracle_pack_int4(_ptr(c), N, K, _ptr(out)), "pack_int4")
    return out


def unpack_int4(packed, K: int) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    N = p.shape[0]
    out = np.empty((N, K), dtype=np.uint8)
    _check(_load().oracle_unpack_int4(_ptr(p), N, K, _ptr(out)), "unpack_int4")
    return out


def quantize_int8(w, g: int, mode: int = STORED):
    """Symmetric absmax INT8 per group of ``g`` weights (g = K: per output channel).

    Returns (codes int8 [N][K] in -127..127, s float32 [N][K/g]).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K), dtype=np.int8)
    s = np.empty((N, K // g), dtype=np.float32)
    _check(_load().oracle_quantize_int8(_ptr(w), N, K, K, g, mode, _ptr(codes), _ptr(s)),
           "quantize_int8")
    return codes, s


def dequant_int4(codes, s, z, g: int) -> np.ndarray:
    """w_hat = s * (q - z) in binary64, [N][K]."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    z = np.ascontiguousarray(z, dtype=np.float32)
    N, K = c.shape
    out = np.empty((N, K), dtype=np.float64)
    _check(_load().oracle_dequant_int4(_ptr(c), _ptr(s), _ptr(z), N, K, g, _ptr(out)),
           "dequant_int4")
    return out


def dequant_int8(codes, s, g: int) -> np.ndarray:
    """w_hat = q * s in binary64, [N][K]."""
    c = np.ascontiguousarray(codes, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    N, K = c.shape
    out = np.empty((N, K), dtype=np.float64)
    _check(_load().oracle_dequant_int8(_ptr(c), _ptr(s), N, K, g, _ptr(out)), "dequant_int8")
    return out


def matmul(x, w_hat):
    """y[m][n] = sum_k x[m][k] * w_hat[n][k] and a[m][n] = sum_k |x[m][k] * w_hat[n][k]|, binary64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    w_hat = np.ascontiguousarray(w_hat, dtype=np.float64)
    M, K = x.shape
    N = w_hat.shape[0]
    if w_hat.shape[1] != K:
        raise ValueError("oracle.matmul: K mismatch")
    y = np.empty((M, N), dtype=np.float64)
    a = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_matmul(_ptr(x), _ptr(w_hat), M, N, K, _ptr(y), _ptr(a)), "matmul")
    return y, a


def gemm_w4a16(x, codes, s, z, g: int):
    """Reference for the W4A16 matmul: dequantise, then the binary64 matmul. Returns (y, a)."""
    return matmul(x, dequant_int4(codes, s, z, g))


def gemm_w8a16(x, codes, s, g: int):
    """Reference for the W8A16 matmul: dequantise, then the binary64 matmul. Returns (y, a)."""
    return matmul(x, dequant_int8(codes, s, g))
