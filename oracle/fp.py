"""Exact decoding of 16-bit storage formats to float64 (oracle; test infrastructure).

The K/V cache and the queries are stored as IEEE binary16 (fp16) or bfloat16
(bf16).  Every value of either format is exactly representable in float64, so
the oracle works on the exact stored values.

* fp16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.  numpy's
  float16 is that format; widening float16 -> float64 is exact.
* bf16: the upper 16 bits of an IEEE binary32; placing the bits in the high
  half of a 32-bit word gives the binary32 value, and widening binary32 ->
  float64 is exact.
"""
import numpy as np


def f16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return b.view(np.float16).astype(np.float64)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def decode(b: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return f16_bits_to_f64(b)
    if dtype == "bf16":
        return bf16_bits_to_f64(b)
    raise ValueError(dtype)
