"""FP8 E4M3 codes for an FP8 KV cache (oracle only).

The pages name FP8 only as a low-precision format of TensorRT-LLM's
operators ("vLLM 推理加速：PagedAttention、FlashAttention 与动态批处理",
"TensorRT-LLM"); they fix neither the format's details nor how a KV cache
would be scaled.  Readings taken here:

* the format is OCP FP8 E4M3 ("E4M3FN"): sign, 4 exponent bits (bias 7),
  3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9; no
  infinities; only S.1111.111 is NaN, so the largest finite value is
  1.75 * 2^8 = 448;
* a cache stores code = E4M3(x / scale) with one float32 scale for all of K
  and one for all of V (the plainest granularity), the division done in
  float32 (the precision the device kernel divides in, so both sides round
  the same float32 value), then rounded to the nearest E4M3 value, ties to
  the even code, magnitudes beyond 448 saturating to +-448;
* the stored value is code's value * scale.

Written from the format's definition: the table of every code's value, and
encoding as the nearest table entry.
"""
import numpy as np

NAN_CODE = 0x7F


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code (NaN for S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
# the non-negative finite codes 0x00..0x7E in increasing value
_POS = TABLE[:0x7F]
assert np.all(np.diff(_POS) > 0)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """float64 values of uint8 codes."""
    return TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """uint8 codes of the float values ``x``: nearest E4M3 value, ties to the
    even code, saturating at +-448; NaN -> 0x7F (sign kept).

    The non-negative codes are increasing in value, so the nearest one to
    |x| is one of the two table entries around it (found by bisection)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x).ravel()
    hi = np.searchsorted(_POS, a, side="left")          # first entry >= |x|
    hi = np.clip(hi, 0, len(_POS) - 1)
    lo = np.clip(hi - 1, 0, len(_POS) - 1)
    d_lo, d_hi = np.abs(a - _POS[lo]), np.abs(_POS[hi] - a)
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a > 448.0, 0x7E, pick)               # saturate
    out = pick.astype(np.uint8).reshape(x.shape)
    out = out | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    nan = np.isnan(x)
    out[nan] = NAN_CODE | np.where(np.signbit(x[nan]), 0x80, 0).astype(np.uint8)
    return out


def quantize(x32: np.ndarray, scale: float) -> np.ndarray:
    """Codes of float32 values x32 stored with ``scale``: E4M3(x32 / scale),
    the division in float32."""
    q = (np.asarray(x32, dtype=np.float32) / np.float32(scale)).astype(np.float32)
    return e4m3_encode(q.astype(np.float64))
