"""Exact widening of the stored K/V/q formats to float64 (oracle only).

FP8 E4M3 codes (uint8) widen through the code table of ``oracle.fp8``.

fp32 and fp16 widen exactly through numpy.  bf16 values arrive as their
uint16 bit patterns: a bf16 number is the upper half of a float32, so
shifting the pattern 16 bits up and reinterpreting it as float32 gives the
value exactly, and float32 -> float64 is exact too.
"""
import numpy as np

NAN_PATTERN = {"f32": np.float32(np.nan), "f16": np.float16(np.nan), "bf16": np.uint16(0x7FC0),
               "e4m3": np.uint8(0x7F)}
STORAGE_NP = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16, "e4m3": np.uint8}


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Return the float64 values held by storage array ``x``."""
    if dtype == "f32":
        assert x.dtype == np.float32
        return x.astype(np.float64)
    if dtype == "f16":
        assert x.dtype == np.float16
        return x.astype(np.float64)
    if dtype == "bf16":
        assert x.dtype == np.uint16
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "e4m3":  # FP8 codes (oracle.fp8); the cache's scale is applied by the caller
        from .fp8 import e4m3_decode
        assert x.dtype == np.uint8
        return e4m3_decode(x)
    raise ValueError(dtype)


def nan_fill(shape, dtype: str) -> np.ndarray:
    """A storage array of ``shape`` whose every element is a quiet NaN."""
    return np.full(shape, NAN_PATTERN[dtype], dtype=STORAGE_NP[dtype])
