"""Exact decoding of the operand codes the indexer consumes (oracle; test infrastructure only).

The ADIndex paper (arXiv 2611.12956v1, §3) fixes no operand precision. The workloads
this oracle checks feed bf16 codes, or FP8-e4m3 codes with one fp32 scale per token; the
oracle decodes both exactly into float64 from the format definitions:

  bf16   1 sign, 8 exponent, 7 mantissa bits = the upper half of an IEEE binary32.
  e4m3   the "FN" variant: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
         subnormals when the exponent field is 0, no infinities, and the single
         exponent-15 / mantissa-7 pattern (0x7F, 0xFF) is NaN. Largest finite: 448.
"""

import numpy as np


def bf16_bits_to_f64(bits):
    """uint16 bf16 codes -> float64 values (exact: widen to the binary32 with the same top half)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes):
    """uint8 e4m3 (FN) codes -> float64 values, from the field definition above."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    exp_field = (c >> 3) & 0xF
    man = (c & 0x7).astype(np.float64)
    normal = (1.0 + man / 8.0) * np.exp2(exp_field.astype(np.float64) - 7.0)
    subnormal = (man / 8.0) * np.exp2(1.0 - 7.0)
    val = sign * np.where(exp_field == 0, subnormal, normal)
    return np.where((exp_field == 15) & ((c & 0x7) == 7), np.nan, val)


def dequantize(codes, scale, dtype):
    """Real operand values: bf16 codes as-is, or e4m3 codes times a per-row fp32 scale.

    ``codes`` has the token (or key) index first; ``scale`` holds one value per index
    along that first axis and broadcasts over the rest.
    """
    if dtype == "bf16":
        return bf16_bits_to_f64(codes)
    if dtype == "e4m3":
        v = e4m3_to_f64(codes)
        s = np.asarray(scale, dtype=np.float32).astype(np.float64)
        return v * s.reshape(s.shape + (1,) * (v.ndim - s.ndim))
    raise ValueError(dtype)
