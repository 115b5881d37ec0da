"""Exact widening of stored cache values to float64 (oracle; test infrastructure only).

Stored dtypes: "f32" (numpy float32), "f16" (numpy float16) and "bf16" (uint16 bit
patterns: a bfloat16 is the upper half of the float32 with the same bits); "f64"
passes float64 values through (dequantized fp8 caches, see ``oracle.fp8``).  Every
widening here is exact.
"""
import numpy as np


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "f16":
        return np.asarray(x, dtype=np.float16).astype(np.float64)
    if dtype == "bf16":
        bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")
