"""Python binding of libwq (include/wq.h): group-wise weight quantisation and the
dequant-fused weight-only matmul on NVIDIA B200.

Argument marshalling only.  Every step runs in the CUDA kernels of
``libwq.so``; this module passes device pointers, sizes and the current CUDA
stream through ctypes and allocates output tensors with torch when the
caller does not pass them.  There is no CPU path: the functions require CUDA
tensors and raise if ``libwq.so`` is missing.

bf16 scales and zero-points are returned as ``torch.bfloat16`` tensors (the
C ABI's uint16 bit patterns).  Function names are those of the C ABI.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "wq.h")

WQ_OK = 0
WQ_ERR_ARG = -1
WQ_ERR_SHAPE = -2
WQ_ERR_ALIGN = -3
WQ_ERR_UNSUPPORTED = -4
WQ_ERR_CUDA = -5
WQ_ERR_WORKSPACE = -6
WQ_ERR_DEVICE_TIMEOUT = -7
WQ_F32 = 0
WQ_BF16 = 1
WQ_FP8_E4M3 = 0
WQ_FP8_E5M2 = 1

_lib = None


class WQError(RuntimeError):
    """A libwq call returned a status other than WQ_OK."""

    def __init__(self, status: int, detail: str):
        super().__init__(f"{wq_status_str(status)} ({detail})" if detail else wq_status_str(status))
        self.status = status


def lib():
    """The loaded libwq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libwq.so not found at {LIB_PATH}: build it with "
                               "`python -m group_wise_weight_b200.build` (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.wq_status_str.argtypes = [I]
        L.wq_status_str.restype = ctypes.c_char_p
        L.wq_last_error.argtypes = []
        L.wq_last_error.restype = ctypes.c_char_p
        L.wq_version.restype = I
        L.wq_quantize_int4.argtypes = [P, I, I64, I64, I64, I, P, P, P, P]
        L.wq_quantize_int4.restype = I
        L.wq_quantize_int4_scaled.argtypes = [P, I, I64, I64, I64, I, P, P, P, P, P]
        L.wq_quantize_int4_scaled.restype = I
        L.wq_quantize_int4_sym.argtypes = [P, I, I64, I64, I64, I, P, P, P, P]
        L.wq_quantize_int4_sym.restype = I
        L.wq_quantize_int8.argtypes = [P, I, I64, I64, I64, I, P, P, P]
        L.wq_quantize_int8.restype = I
        L.wq_gemm_workspace_bytes.argtypes = [I64, I64, I64, I, I]
        L.wq_gemm_workspace_bytes.restype = SZ
        L.wq_gemm_w4a16.argtypes = [P, I64, I64, I64, P, P, P, I, P, P, SZ, P]
        L.wq_gemm_w4a16.restype = I
        L.wq_gemm_w8a16.argtypes = [P, I64, I64, I64, P, P, I, P, P, SZ, P]
        L.wq_gemm_w8a16.restype = I
        L.wq_gemm_w4a16_noalloc.argtypes = [P, I64, I64, I64, P, P, P, I, P, P]
        L.wq_gemm_w4a16_noalloc.restype = I
        L.wq_device_status.argtypes = [P]
        L.wq_device_status.restype = I
        L.wq_quantize_fp8.argtypes = [P, I, I64, I64, I64, I, P, P, P]
        L.wq_quantize_fp8.restype = I
        L.wq_quantize_fp8_tensor.argtypes = [P, I, I64, I64, I, P, P, P]
        L.wq_quantize_fp8_tensor.restype = I
        L.wq_gemm_w8a8_fp8_workspace_bytes.argtypes = [I64, I64, I64]
        L.wq_gemm_w8a8_fp8_workspace_bytes.restype = SZ
        L.wq_gemm_w8a8_fp8.argtypes = [P, P, I64, I64, I64, P, P, P, P, SZ, P]
        L.wq_gemm_w8a8_fp8.restype = I
        L.wq_nvfp4_scale_bytes.argtypes = [I64, I64]
        L.wq_nvfp4_scale_bytes.restype = SZ
        L.wq_quantize_nvfp4.argtypes = [P, I, I64, I64, I64, P, P, P, P]
        L.wq_quantize_nvfp4.restype = I
        L.wq_gemm_nvfp4_workspace_bytes.argtypes = [I64, I64, I64]
        L.wq_gemm_nvfp4_workspace_bytes.restype = SZ
        L.wq_gemm_nvfp4.argtypes = [P, P, P, I64, I64, I64, P, P, P, P, P, SZ, P]
        L.wq_gemm_nvfp4.restype = I
        L.wq_gemm_w4a16_colscaled_workspace_bytes.argtypes = [I64, I64, I64, I]
        L.wq_gemm_w4a16_colscaled_workspace_bytes.restype = SZ
        L.wq_gemm_w4a16_colscaled.argtypes = [P, P, I64, I64, I64, P, P, P, I, P, P, SZ, P]
        L.wq_gemm_w4a16_colscaled.restype = I
        L.wq_awq_channel_magnitudes.argtypes = [P, I64, I64, P, P]
        L.wq_awq_channel_magnitudes.restype = I
        L.wq_awq_channel_scales.argtypes = [P, I64, ctypes.c_double, P, P]
        L.wq_awq_channel_scales.restype = I
        L.wq_test_skip_weight_copy.argtypes = [I64]
        L.wq_test_skip_weight_copy.restype = None
        L.wq_decode_attention_workspace_bytes.argtypes = [I64, I64, I64]
        L.wq_decode_attention_workspace_bytes.restype = SZ
        L.wq_decode_attention_int4.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I64, I64, P, P, SZ, P]
        L.wq_decode_attention_int4.restype = I
        L.wq_decode_attention_fp8.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64, I64, P, P, SZ, P]
        L.wq_decode_attention_fp8.restype = I
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/wq.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)))


def wq_status_str(status: int) -> str:
    return lib().wq_status_str(int(status)).decode()


def wq_last_error() -> str:
    return lib().wq_last_error().decode()


def wq_version() -> int:
    return int(lib().wq_version())


def _check(rc: int):
    if rc != WQ_OK:
        raise WQError(rc, wq_last_error())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (libwq has no CPU path)")
    return t.data_ptr()


def _dense(t: torch.Tensor, name: str):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def wq_quantize_int4(w: torch.Tensor, g: int = 128, qweight=None, scales=None, zeros=None, stream=None):
    """Asymmetric INT4 per group of g weights along K.  w: [N][K] (row stride >= K) fp32 or bf16 on CUDA.

    Returns (qweight uint8 [N][K/2], scales bf16 [N][K/g], zeros bf16 [N][K/g]).
    """
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a 2-D tensor with unit stride along K")
    wtype = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16}.get(w.dtype)
    if wtype is None:
        raise TypeError("w must be float32 or bfloat16")
    N, K = w.shape
    dev = w.device
    qweight = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if qweight is None else qweight
    scales = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if scales is None else scales
    zeros = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if zeros is None else zeros
    for t, n in ((qweight, "qweight"), (scales, "scales"), (zeros, "zeros")):
        _dense(t, n)
    _check(lib().wq_quantize_int4(_dev(w, "w"), wtype, N, K, w.stride(0), int(g), _dev(qweight, "qweight"),
                                  _dev(scales, "scales"), _dev(zeros, "zeros"), _stream_handle(stream)))
    return qweight, scales, zeros


def wq_quantize_int4_scaled(w: torch.Tensor, col_scale: torch.Tensor, g: int = 128, qweight=None, scales=None,
                            zeros=None, stream=None):
    """wq_quantize_int4 of w[n][k] * col_scale[k] (binary32 products): the weight side of an activation-aware
    per-input-channel scaling.  col_scale: float32 [K] on CUDA.  Returns (qweight, scales, zeros)."""
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a 2-D tensor with unit stride along K")
    wtype = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16}.get(w.dtype)
    if wtype is None:
        raise TypeError("w must be float32 or bfloat16")
    N, K = w.shape
    if col_scale.dtype != torch.float32 or col_scale.numel() != K:
        raise TypeError("col_scale must be a float32 tensor of K values")
    _dense(col_scale, "col_scale")
    dev = w.device
    qweight = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if qweight is None else qweight
    scales = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if scales is None else scales
    zeros = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if zeros is None else zeros
    for t, n in ((qweight, "qweight"), (scales, "scales"), (zeros, "zeros")):
        _dense(t, n)
    _check(lib().wq_quantize_int4_scaled(_dev(w, "w"), wtype, N, K, w.stride(0), int(g), _dev(col_scale, "col_scale"),
                                         _dev(qweight, "qweight"), _dev(scales, "scales"), _dev(zeros, "zeros"),
                                         _stream_handle(stream)))
    return qweight, scales, zeros


def wq_quantize_int4_sym(w: torch.Tensor, g: int = 128, qweight=None, scales=None, zeros=None, stream=None):
    """Symmetric INT4 (levels -7..7) per group of g weights along K, in the INT4 format of
    wq_quantize_int4 with every zero-point 8 (codes q + 8), ready for wq_gemm_w4a16.

    Returns (qweight uint8 [N][K/2], scales bf16 [N][K/g], zeros bf16 [N][K/g] all 8).
    """
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a 2-D tensor with unit stride along K")
    wtype = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16}.get(w.dtype)
    if wtype is None:
        raise TypeError("w must be float32 or bfloat16")
    N, K = w.shape
    dev = w.device
    qweight = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if qweight is None else qweight
    scales = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if scales is None else scales
    zeros = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if zeros is None else zeros
    for t, n in ((qweight, "qweight"), (scales, "scales"), (zeros, "zeros")):
        _dense(t, n)
    _check(lib().wq_quantize_int4_sym(_dev(w, "w"), wtype, N, K, w.stride(0), int(g), _dev(qweight, "qweight"),
                                      _dev(scales, "scales"), _dev(zeros, "zeros"), _stream_handle(stream)))
    return qweight, scales, zeros


def wq_quantize_int8(w: torch.Tensor, g: int | None = None, qweight=None, scales=None, stream=None):
    """Symmetric absmax INT8 per group of g weights (g=None or K: per output channel).

    Returns (qweight int8 [N][K], scales bf16 [N][K/g]).
    """
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a 2-D tensor with unit stride along K")
    wtype = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16}.get(w.dtype)
    if wtype is None:
        raise TypeError("w must be float32 or bfloat16")
    N, K = w.shape
    g = K if g is None else int(g)
    dev = w.device
    qweight = torch.empty((N, K), dtype=torch.int8, device=dev) if qweight is None else qweight
    scales = torch.empty((N, K // g), dtype=torch.bfloat16, device=dev) if scales is None else scales
    _dense(qweight, "qweight")
    _dense(scales, "scales")
    _check(lib().wq_quantize_int8(_dev(w, "w"), wtype, N, K, w.stride(0), g, _dev(qweight, "qweight"),
                                  _dev(scales, "scales"), _stream_handle(stream)))
    return qweight, scales


def wq_gemm_workspace_bytes(M: int, N: int, K: int, g: int, wbits: int) -> int:
    return int(lib().wq_gemm_workspace_bytes(int(M), int(N), int(K), int(g), int(wbits)))


def _workspace(workspace, need: int, dev):
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    return workspace, workspace.numel() * workspace.element_size()


def wq_gemm_w4a16(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, g: int = 128,
                  y=None, workspace=None, stream=None) -> torch.Tensor:
    """y[M][N] = x[M][K] @ w_hat^T with w_hat = s * (q - z) dequantised in-kernel.  bf16 in, bf16 out."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    _dense(x, "x")
    M, K = x.shape
    N = qweight.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _dense(y, "y")
    need = wq_gemm_workspace_bytes(M, N, K, g, 4)
    workspace, ws_bytes = _workspace(workspace, need, x.device)
    _check(lib().wq_gemm_w4a16(_dev(x, "x"), M, N, K, _dev(qweight, "qweight"), _dev(scales, "scales"),
                               _dev(zeros, "zeros"), int(g), _dev(y, "y"),
                               workspace.data_ptr() if workspace is not None else None, ws_bytes,
                               _stream_handle(stream)))
    return y


def wq_gemm_w8a16(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, g: int | None = None, y=None,
                  workspace=None, stream=None) -> torch.Tensor:
    """y[M][N] = x[M][K] @ w_hat^T with w_hat = q * s dequantised in-kernel.  g=None: per output channel."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    _dense(x, "x")
    M, K = x.shape
    N = qweight.shape[0]
    g = K if g is None else int(g)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _dense(y, "y")
    need = wq_gemm_workspace_bytes(M, N, K, g, 8)
    workspace, ws_bytes = _workspace(workspace, need, x.device)
    _check(lib().wq_gemm_w8a16(_dev(x, "x"), M, N, K, _dev(qweight, "qweight"), _dev(scales, "scales"), g,
                               _dev(y, "y"), workspace.data_ptr() if workspace is not None else None, ws_bytes,
                               _stream_handle(stream)))
    return y


def wq_gemm_w4a16_noalloc(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                          g: int = 128, y=None, stream=None) -> torch.Tensor:
    """wq_gemm_w4a16 for callers that cannot allocate device memory: the C entry point takes no
    workspace and uses the library's fixed 2 MiB scratch array (2 <= M <= 16, g = 128; see wq.h).
    Pass `y` to avoid the output allocation here as well."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    _dense(x, "x")
    M, K = x.shape
    N = qweight.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _dense(y, "y")
    _check(lib().wq_gemm_w4a16_noalloc(_dev(x, "x"), M, N, K, _dev(qweight, "qweight"), _dev(scales, "scales"),
                                       _dev(zeros, "zeros"), int(g), _dev(y, "y"), _stream_handle(stream)))
    return y


def wq_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word as a WQ_* code."""
    return int(lib().wq_device_status(_stream_handle(stream)))


def _wtype(t: torch.Tensor) -> int:
    wtype = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16}.get(t.dtype)
    if wtype is None:
        raise TypeError("input must be float32 or bfloat16")
    return wtype


def wq_quantize_fp8(w: torch.Tensor, fmt: int = WQ_FP8_E4M3, qweight=None, scales=None, stream=None):
    """FP8 per output channel.  w: [N][K] (row stride >= K) fp32 or bf16 on CUDA.

    Returns (qweight uint8 [N][K] FP8 codes, scales float32 [N])."""
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a 2-D tensor with unit stride along K")
    wtype = _wtype(w)
    N, K = w.shape
    qweight = torch.empty((N, K), dtype=torch.uint8, device=w.device) if qweight is None else qweight
    scales = torch.empty((N,), dtype=torch.float32, device=w.device) if scales is None else scales
    _dense(qweight, "qweight")
    _dense(scales, "scales")
    _check(lib().wq_quantize_fp8(_dev(w, "w"), wtype, N, K, w.stride(0), int(fmt), _dev(qweight, "qweight"),
                                 _dev(scales, "scales"), _stream_handle(stream)))
    return qweight, scales


def wq_quantize_fp8_tensor(x: torch.Tensor, fmt: int = WQ_FP8_E4M3, q=None, scale=None, stream=None):
    """FP8 with one scale for the whole tensor.  x: dense [M][K] fp32 or bf16 on CUDA.

    Returns (q uint8 [M][K] FP8 codes, scale float32 [1] on the device)."""
    if x.dim() != 2:
        raise ValueError("x must be a 2-D tensor")
    _dense(x, "x")
    xtype = _wtype(x)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if q is None else q
    scale = torch.empty((1,), dtype=torch.float32, device=x.device) if scale is None else scale
    _dense(q, "q")
    _check(lib().wq_quantize_fp8_tensor(_dev(x, "x"), xtype, M, K, int(fmt), _dev(q, "q"), _dev(scale, "scale"),
                                        _stream_handle(stream)))
    return q, scale


def wq_gemm_w8a8_fp8_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().wq_gemm_w8a8_fp8_workspace_bytes(int(M), int(N), int(K)))


def wq_gemm_w8a8_fp8(xq: torch.Tensor, xscale: torch.Tensor, wq: torch.Tensor, wscales: torch.Tensor, y=None,
                     workspace=None, stream=None) -> torch.Tensor:
    """y[M][N] = (xq . wq^T) * xscale * wscales[n] with E4M3 codes multiplied on the tensor cores.  bf16 out."""
    if xq.dtype != torch.uint8 or wq.dtype != torch.uint8 or xq.dim() != 2 or wq.dim() != 2:
        raise TypeError("xq and wq must be 2-D uint8 tensors of FP8 codes")
    for t, n in ((xq, "xq"), (wq, "wq"), (wscales, "wscales")):
        _dense(t, n)
    M, K = xq.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if y is None else y
    _dense(y, "y")
    need = wq_gemm_w8a8_fp8_workspace_bytes(M, N, K)
    workspace, ws_bytes = _workspace(workspace, need, xq.device)
    _check(lib().wq_gemm_w8a8_fp8(_dev(xq, "xq"), _dev(xscale, "xscale"), M, N, K, _dev(wq, "wq"),
                                  _dev(wscales, "wscales"), _dev(y, "y"),
                                  workspace.data_ptr() if workspace is not None else None, ws_bytes,
                                  _stream_handle(stream)))
    return y


def wq_nvfp4_scale_bytes(N: int, K: int) -> int:
    return int(lib().wq_nvfp4_scale_bytes(int(N), int(K)))


def wq_quantize_nvfp4(w: torch.Tensor, codes=None, block_scales=None, tensor_scale=None, stream=None):
    """NVFP4: E2M1 values, an E4M3 scale per 16 values of a row, one binary32 tensor scale.
    w: [N][K] (row stride >= K) fp32 or bf16 on CUDA.

    Returns (codes uint8 [N][K/2], block_scales uint8 [wq_nvfp4_scale_bytes(N, K)] in the tensor-core
    layout, tensor_scale float32 [1] on the device)."""
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a 2-D tensor with unit stride along K")
    wtype = _wtype(w)
    N, K = w.shape
    dev = w.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    nsb = wq_nvfp4_scale_bytes(N, K)
    block_scales = torch.empty((max(nsb, 1),), dtype=torch.uint8, device=dev) if block_scales is None else block_scales
    tensor_scale = torch.empty((1,), dtype=torch.float32, device=dev) if tensor_scale is None else tensor_scale
    _dense(codes, "codes")
    _check(lib().wq_quantize_nvfp4(_dev(w, "w"), wtype, N, K, w.stride(0), _dev(codes, "codes"),
                                   _dev(block_scales, "block_scales"), _dev(tensor_scale, "tensor_scale"),
                                   _stream_handle(stream)))
    return codes, block_scales, tensor_scale


def wq_gemm_nvfp4_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().wq_gemm_nvfp4_workspace_bytes(int(M), int(N), int(K)))


def wq_gemm_nvfp4(x_codes: torch.Tensor, x_scales: torch.Tensor, x_tscale: torch.Tensor, w_codes: torch.Tensor,
                  w_scales: torch.Tensor, w_tscale: torch.Tensor, y=None, workspace=None, stream=None) -> torch.Tensor:
    """NVFP4 W4A4 matmul with the block scales applied inside the tensor-core MMA.  Operands as returned by
    wq_quantize_nvfp4 (x_codes [M][K/2], w_codes [N][K/2]).  bf16 out [M][N]."""
    if x_codes.dtype != torch.uint8 or w_codes.dtype != torch.uint8 or x_codes.dim() != 2 or w_codes.dim() != 2:
        raise TypeError("codes must be 2-D uint8 tensors")
    for t, n in ((x_codes, "x_codes"), (w_codes, "w_codes")):
        _dense(t, n)
    M, K = x_codes.shape[0], x_codes.shape[1] * 2
    N = w_codes.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device) if y is None else y
    _dense(y, "y")
    need = wq_gemm_nvfp4_workspace_bytes(M, N, K)
    workspace, ws_bytes = _workspace(workspace, need, x_codes.device)
    _check(lib().wq_gemm_nvfp4(_dev(x_codes, "x_codes"), _dev(x_scales, "x_scales"), _dev(x_tscale, "x_tscale"),
                               M, N, K, _dev(w_codes, "w_codes"), _dev(w_scales, "w_scales"),
                               _dev(w_tscale, "w_tscale"), _dev(y, "y"),
                               workspace.data_ptr() if workspace is not None else None, ws_bytes,
                               _stream_handle(stream)))
    return y


def wq_decode_attention_workspace_bytes(B: int, T: int, H: int) -> int:
    return int(lib().wq_decode_attention_workspace_bytes(int(B), int(T), int(H)))


def _attention_out(q: torch.Tensor, lengths: torch.Tensor, o, workspace, B: int, T: int, H: int):
    if q.dtype != torch.bfloat16 or q.dim() != 3:
        raise TypeError("q must be a bfloat16 [B][Hq][D] tensor")
    if lengths.dtype != torch.int32 or lengths.numel() != B:
        raise TypeError("lengths must be an int32 tensor of B values")
    _dense(q, "q")
    _dense(lengths, "lengths")
    o = torch.empty(q.shape, dtype=torch.float32, device=q.device) if o is None else o
    _dense(o, "o")
    need = wq_decode_attention_workspace_bytes(B, T, H)
    workspace = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    return o, workspace


def wq_decode_attention_int4(q: torch.Tensor, k_codes: torch.Tensor, k_scales: torch.Tensor, k_zeros: torch.Tensor,
                             v_codes: torch.Tensor, v_scales: torch.Tensor, v_zeros: torch.Tensor,
                             lengths: torch.Tensor, o=None, workspace=None, stream=None) -> torch.Tensor:
    """Decode attention over an int4 KV cache.  q [B][Hq][128] bf16; codes [B][T][H][64] uint8; scales and
    zero-points [B][T][H] (any shape with B*T*H values) bf16; lengths int32 [B].  Returns o float32
    [B][Hq][128]."""
    B, T, H = k_codes.shape[0], k_codes.shape[1], k_codes.shape[2]
    o, workspace = _attention_out(q, lengths, o, workspace, B, T, H)
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes"), (k_scales, "k_scales"), (k_zeros, "k_zeros"),
                 (v_scales, "v_scales"), (v_zeros, "v_zeros")):
        _dense(t, n)
    _check(lib().wq_decode_attention_int4(_dev(q, "q"), _dev(k_codes, "k_codes"), _dev(k_scales, "k_scales"),
                                          _dev(k_zeros, "k_zeros"), _dev(v_codes, "v_codes"),
                                          _dev(v_scales, "v_scales"), _dev(v_zeros, "v_zeros"),
                                          _dev(lengths, "lengths"), B, T, H, q.shape[1], q.shape[2], _dev(o, "o"),
                                          workspace.data_ptr(), workspace.numel(), _stream_handle(stream)))
    return o


def wq_decode_attention_fp8(q: torch.Tensor, k_codes: torch.Tensor, k_scale: torch.Tensor, v_codes: torch.Tensor,
                            v_scale: torch.Tensor, lengths: torch.Tensor, o=None, workspace=None,
                            stream=None) -> torch.Tensor:
    """Decode attention over an fp8 (E4M3, one scale per tensor) KV cache.  q [B][Hq][128] bf16; codes
    [B][T][H][128] uint8; k_scale, v_scale float32 [1] on the device; lengths int32 [B].  Returns o float32
    [B][Hq][128]."""
    B, T, H = k_codes.shape[0], k_codes.shape[1], k_codes.shape[2]
    o, workspace = _attention_out(q, lengths, o, workspace, B, T, H)
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        _dense(t, n)
    _check(lib().wq_decode_attention_fp8(_dev(q, "q"), _dev(k_codes, "k_codes"), _dev(k_scale, "k_scale"),
                                         _dev(v_codes, "v_codes"), _dev(v_scale, "v_scale"), _dev(lengths, "lengths"),
                                         B, T, H, q.shape[1], q.shape[2], _dev(o, "o"), workspace.data_ptr(),
                                         workspace.numel(), _stream_handle(stream)))
    return o


def wq_gemm_w4a16_colscaled(x: torch.Tensor, col_scale: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                            zeros: torch.Tensor, g: int = 128, y=None, workspace=None, stream=None) -> torch.Tensor:
    """y = bf16(x / col_scale) @ w_hat^T for weights quantised by wq_quantize_int4_scaled with the same col_scale
    (float32 [K] on CUDA).  bf16 in, bf16 out."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    _dense(x, "x")
    M, K = x.shape
    if col_scale.dtype != torch.float32 or col_scale.numel() != K:
        raise TypeError("col_scale must be a float32 tensor of K values")
    _dense(col_scale, "col_scale")
    N = qweight.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _dense(y, "y")
    need = int(lib().wq_gemm_w4a16_colscaled_workspace_bytes(M, N, K, int(g)))
    workspace, ws_bytes = _workspace(workspace, need, x.device)
    _check(lib().wq_gemm_w4a16_colscaled(_dev(x, "x"), _dev(col_scale, "col_scale"), M, N, K,
                                         _dev(qweight, "qweight"), _dev(scales, "scales"), _dev(zeros, "zeros"),
                                         int(g), _dev(y, "y"), workspace.data_ptr() if workspace is not None else None,
                                         ws_bytes, _stream_handle(stream)))
    return y


def wq_awq_channel_magnitudes(x: torch.Tensor, magnitudes=None, stream=None) -> torch.Tensor:
    """Mean |x| per input channel over the rows of x (bf16 [M][K] on CUDA), float64 [K]."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    _dense(x, "x")
    M, K = x.shape
    magnitudes = torch.empty(K, dtype=torch.float64, device=x.device) if magnitudes is None else magnitudes
    _check(lib().wq_awq_channel_magnitudes(_dev(x, "x"), M, K, _dev(magnitudes, "magnitudes"),
                                           _stream_handle(stream)))
    return magnitudes


def wq_awq_channel_scales(magnitudes: torch.Tensor, alpha: float, col_scale=None, stream=None) -> torch.Tensor:
    """s_c = m_c ** alpha normalised to max * min = 1 (float64 magnitudes [K] on CUDA), float32 [K]."""
    if magnitudes.dtype != torch.float64 or magnitudes.dim() != 1:
        raise TypeError("magnitudes must be a 1-D float64 tensor")
    K = magnitudes.numel()
    col_scale = torch.empty(K, dtype=torch.float32, device=magnitudes.device) if col_scale is None else col_scale
    _check(lib().wq_awq_channel_scales(_dev(magnitudes, "magnitudes"), K, float(alpha), _dev(col_scale, "col_scale"),
                                       _stream_handle(stream)))
    return col_scale
