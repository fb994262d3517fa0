"""Online FP8 E4M3 quantisation with one power-of-two scale per 128 elements.

Passage: "DeepSeek-V4-Flash-SI" model card -- 架构特性 / 低精度计算 says the
activations are quantised online to FP8 E4M3 in groups of 128 elements with a
power-of-2 scale; the 模型训练 table says the scale is dynamic and ue8m0.

The pages do not spell out the scale rule.  Reading taken (the plainest one
consistent with "power-of-2 scale" and an E4M3 target whose largest finite
value is 448):
  ratio = amax / 448            (float32, IEEE round-to-nearest-even divide)
  k     = ceil(log2(ratio))     (exact, from the float32 value)
  k     = clamp(k, -127, 127);  amax == 0 -> k = 0
  q     = E4M3(x / 2^k)         (round to nearest even, saturate to +-448)
  stored scale byte = k + 127   (E8M0, value 2^k)
x / 2^k is exact (a power-of-two rescale), so only the final rounding loses
information.  Rounding to nearest even matches the half_even rounding named
in the "DeepSeek-V4.1-Flash-Quark-PTPC-FP8" walkthrough (核心参数).
The same rule requantises the SwiGLU output h before the w2 GEMM.
"""
from __future__ import annotations

import numpy as np

from .formats import decode_bf16_bits, decode_e4m3, encode_e4m3_rne_sat

GROUP = 128


def ceil_log2_f32(r: np.ndarray) -> np.ndarray:
    """Exact ceil(log2(r)) for positive float32 r (normal or subnormal)."""
    m, e = np.frexp(np.asarray(r, dtype=np.float32))    # r = m * 2^e, m in [0.5, 1)
    return np.where(m == 0.5, e - 1, e).astype(np.int64)


def pow2_scale_exponent(amax32: np.ndarray) -> np.ndarray:
    """Per-group exponent k from the float32 group maxima."""
    amax32 = np.asarray(amax32, dtype=np.float32)
    ratio = amax32 / np.float32(448.0)                  # float32 IEEE division
    safe = np.where(amax32 > 0, ratio, np.float32(1.0))
    k = np.where(amax32 > 0, ceil_log2_f32(safe), 0)
    return np.clip(k, -127, 127).astype(np.int64)


def quantize_fp8_pow2(x32: np.ndarray, group: int = GROUP):
    """float32 [rows, cols] -> (E4M3 codes uint8 [rows, cols], E8M0 uint8 [rows, cols/group])."""
    x32 = np.asarray(x32, dtype=np.float32)
    rows, cols = x32.shape
    assert cols % group == 0
    g = x32.reshape(rows, cols // group, group)
    amax = np.abs(g).max(axis=-1) if rows else np.zeros((0, cols // group), np.float32)
    k = pow2_scale_exponent(amax)
    y = g.astype(np.float64) * np.ldexp(1.0, -k)[..., None]
    q = encode_e4m3_rne_sat(y).reshape(rows, cols)
    return q, (k + 127).astype(np.uint8)


def quantize_act_fp8(x_bf16_bits: np.ndarray):
    """Step a1: bf16 activations [T, H] -> (xq E4M3 [T, H], sx E8M0 [T, H/128])."""
    return quantize_fp8_pow2(decode_bf16_bits(x_bf16_bits))


def dequantize_fp8_pow2(q: np.ndarray, s: np.ndarray, group: int = GROUP) -> np.ndarray:
    """E4M3 codes + per-group E8M0 -> float64."""
    q = np.asarray(q)
    rows, cols = q.shape
    v = decode_e4m3(q).reshape(rows, cols // group, group)
    scale = np.ldexp(1.0, np.asarray(s, dtype=np.int64) - 127)
    return (v * scale[..., None]).reshape(rows, cols)
