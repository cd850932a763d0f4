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
