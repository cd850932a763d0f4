"""Storage accounting for group-wise quantised weights (test infrastructure).

Cited by page title and section:
  * "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
    Quantization" -- "What quantisation does": a 16-bit scale per group of g
    weights adds 16/g bits per weight, so 4-bit at g=128 is 4.125 bits and a
    70B model takes 36.1 GB; at g=32 it is 4.5 bits and 39.4 GB.
  * "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF" --
    "Numerical example": 8 weights x 4 bits + a 2-byte bf16 scale + a
    half-byte INT4 zero-point = 6.5 bytes.
The library's own format stores a bf16 zero-point per group too, i.e.
zero_bits = 16: 4.25 bits at g=128 and 5.0 at g=32.
"""


def bits_per_weight(b: int, g: int, scale_bits: int = 16, zero_bits: int = 0) -> float:
    """Code bits plus the per-group parameters spread over the g weights they cover."""
    return b + (scale_bits + zero_bits) / g


def model_gigabytes(n_params: float, b: int, g: int, scale_bits: int = 16, zero_bits: int = 0) -> float:
    """Decimal gigabytes for n_params weights at the given format."""
    return n_params * bits_per_weight(b, g, scale_bits, zero_bits) / 8 / 1e9


def example_bytes(n_weights: int, b: int, scale_bits: int, zero_bits: int) -> float:
    """Bytes for one group of n_weights codes plus one scale and one zero-point."""
    return (n_weights * b + scale_bits + zero_bits) / 8


# ---------------------------------------------------------------------------
# KV cache (the NEXT row on KV-cache quantisation)
#   * "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF" -- "KV cache quantization": a bf16
#     cache holds 2 bytes per dimension x heads x head_dim x 2 (K and V); fp8 holds 1 byte; int4 with
#     blocks of 128 holds half a byte plus the scale overhead and divides the cache by about 3.5.
#   * "Quantization Methods Compared ..." -- "Hardware, formats and the roofline": the worked decode step
#     of the 70B model at batch 128 and 8,000-token contexts reads 140 GB of fp16 weights against 335.5 GB
#     of KV cache, so 4-bit weights (about 36 GB) buy only about 1.28x.
# ---------------------------------------------------------------------------

def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int, batch: int,
                   bytes_per_element: float) -> float:
    """K and V of every layer, head and dimension for tokens x batch positions."""
    return 2 * layers * kv_heads * head_dim * tokens * batch * bytes_per_element


def block_bytes_per_element(bits: int, block: int, param_bits: int) -> float:
    """Bytes per cached element when every block of `block` values carries param_bits of parameters."""
    return bits / 8 + param_bits / 8 / block


def decode_step_speedup(weight_bytes_before: float, weight_bytes_after: float, other_bytes: float) -> float:
    """Memory-bound decode: the step time scales with the bytes read, weights plus everything else."""
    return (weight_bytes_before + other_bytes) / (weight_bytes_after + other_bytes)


# ---------------------------------------------------------------------------
# Roofline of the decode step (the measurement's basis)
#   * "Quantization Methods Compared ..." -- "Hardware, formats and the roofline": a decode step reads every
#     weight once and does 2 x parameters x batch flops; with 1,000 TFLOP/s and 3.3 TB/s the ridge point is
#     1,000 / 3.3 = 303 flop per byte; fp16 weights (2 bytes) give an intensity of batch flop per byte, so
#     decode stays memory-bound until batch about 300; 4-bit weights (0.5 bytes) give 4 x batch and cross the
#     ridge near batch 76.  The worked step (70B, batch 128, 8 GPUs: 26.4 TB/s and 8,000 TFLOP/s together)
#     computes for about 2.2 ms, far below its memory time.
# ---------------------------------------------------------------------------

def ridge_point(flops_per_s: float, bytes_per_s: float) -> float:
    """Arithmetic intensity (flop per byte) above which a kernel is compute-bound."""
    return flops_per_s / bytes_per_s


def decode_intensity(batch: int, bytes_per_weight: float) -> float:
    """Flop per byte of a decode step: 2 x batch flops per weight over the weight's bytes."""
    return 2.0 * batch / bytes_per_weight


def crossover_batch(ridge: float, bytes_per_weight: float) -> float:
    """The batch at which decode_intensity reaches the ridge point."""
    return ridge * bytes_per_weight / 2.0


def decode_compute_seconds(n_params: float, batch: int, flops_per_s: float) -> float:
    """Compute time of one decode step: 2 x parameters x batch flops."""
    return 2.0 * n_params * batch / flops_per_s
