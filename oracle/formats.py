"""Number formats of the expert path, decoded from their definitions.

* E2M1 (FP4): the expert weights are "FP4 E2M1" with an "F8_E8M0 block scale,
  one per 32 elements" ("DeepSeek-V4-Flash-SI" model card, 架构特性 /
  低精度计算).  The walkthrough "DeepSeek-V4-Pro-0813-nvfp4-DSpark"
  (关于 MXFP4 的无损种子) decodes them by splitting each int8 into its low and
  high 4 bits and looking the nibble up in an FP4 table.  The table itself is
  not printed; the value set {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit is
  the OCP MX E2M1 format: bit 3 = sign, bits 2..1 = exponent (bias 1),
  bit 0 = mantissa, exponent 0 = subnormal.
* E8M0: unsigned power-of-two scale 2^(b - 127); b = 255 is NaN.
* E4M3 (FP8, "FN" variant without infinities): bit 7 sign, bits 6..3 exponent
  (bias 7), bits 2..0 mantissa; exponent 0 is subnormal (m/8 * 2^-6); the
  pattern S.1111.111 is NaN; the largest finite magnitude is 448.
* bfloat16: the upper 16 bits of an IEEE float32.
"""
from __future__ import annotations

import numpy as np


def e2m1_value(code: int) -> float:
    """Value of one 4-bit E2M1 code, from the field definition."""
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 3
    man = code & 1
    if exp == 0:
        mag = 0.5 * man                       # subnormal: m/2 * 2^(1-1)
    else:
        mag = (1.0 + 0.5 * man) * 2.0 ** (exp - 1)
    return sign * mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def decode_e2m1_packed(packed: np.ndarray) -> np.ndarray:
    """uint8 [..., K/2] -> float64 [..., K]; element 2i is the LOW nibble."""
    packed = np.asarray(packed, dtype=np.uint8)
    lo = E2M1_TABLE[packed & 0xF]
    hi = E2M1_TABLE[packed >> 4]
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.float64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def decode_e8m0(b: np.ndarray) -> np.ndarray:
    """uint8 -> float64 2^(b-127); 255 -> NaN."""
    b = np.asarray(b, dtype=np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 127))


def e4m3_value(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 7
    if exp == 15 and man == 7:
        return float("nan")
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** -6
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite magnitudes, codes 0x00..0x7E, strictly increasing
_E4M3_POS = E4M3_TABLE[:0x7F]
E4M3_MAX = 448.0


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def encode_e4m3_rne_sat(v: np.ndarray) -> np.ndarray:
    """float64 -> E4M3 codes: nearest finite value, ties to the even code,
    magnitudes above 448 saturate to 448 (a finite result is always produced).
    The sign bit is the sign of the input, so negative values that round to
    zero give 0x80."""
    v = np.asarray(v, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("NaN input to E4M3 encoder")
    mag = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, mag, side="left")      # first value >= mag
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_hi = _E4M3_POS[hi] - mag
    d_lo = mag - _E4M3_POS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(mag == _E4M3_POS[hi], hi, code).astype(np.uint8)
    sign = np.signbit(v).astype(np.uint8) << 7
    return (code | sign).astype(np.uint8)


def decode_bf16_bits(b: np.ndarray) -> np.ndarray:
    """uint16 bfloat16 bit patterns -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint32) << np.uint32(16)).view(np.float32)


def encode_bf16_rne(v: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bits, rounding once to nearest even from float64.

    Used only to compare: the CUDA path rounds its float32 result; the test
    tolerance covers the difference."""
    v = np.asarray(v, dtype=np.float64)
    f32 = v.astype(np.float32)
    b = f32.view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)
