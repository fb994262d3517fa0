"""Weight repacks of the companion path.

MXFP4 -> NVFP4.  "DeepSeek-V4-Pro-0813-nvfp4-DSpark" walkthrough, 阶段三 and
its MXFP4-vs-NVFP4 storage table: the E2M1 nibbles are moved bit for bit
(weight bits are not recomputed); only the block scale is rewritten, from an
E8M0 scale per 32 elements to an E4M3 scale per 16 elements (group_size 16,
only-experts section), so the scale bytes double and the cast is lossless.
Reading of what the page leaves open: an E8M0 scale 2^e becomes two E4M3
scales 2^(e - G); E4M3 holds the powers of two 2^-9 .. 2^8 exactly (subnormals
included), so G = 0 when every block exponent of the matrix lies in [-9, 8],
otherwise G = max_e - 8 when the exponent span is at most 17, otherwise the
matrix is not representable (error -4).  2^G is returned as the per-matrix
float32 global scale; one "matrix" is one (expert, projection) [N, K].
E8M0 byte 255 (NaN) is error -3.

MXFP4 -> symmetric INT4, group 128.  "DeepSeek-V4-Flash-0731-W4AFP8-mt" model
card, 量化方式 / 权重约定: recipe direct-fp4-to-symmetric-int4-group128,
signed INT4 packed two per int8, float32 weight_scale_inv of shape [N, K/128]
(example: w1.weight [2048, 2048] int8 with weight_scale_inv [2048, 32]).
The page gives no formula.  Reading (parity unpinned): per (row, group of
128) dequantise exactly, amax; scale_inv = amax / 7 (float32 IEEE divide);
q = clamp(round_half_even(x / scale_inv), -7, 7) with x / scale_inv a float32
IEEE divide; amax == 0 -> scale_inv = 1, q = 0.  Element 2i is the low
nibble, stored as 4-bit two's complement.  A block whose dequantised values
overflow float32 is error -4; E8M0 255 is error -3.

MXFP4 -> FP8 E4M3 with a [128, 128] block scale.  "DeepSeek-V4-Pro-0813-
nvfp4-DSpark" walkthrough, 关于 MXFP4 的无损种子: cast_e2m1fn_to_e4m3fn splits
the two nibbles of each int8, looks the E2M1 values up and rewrites the scale
per 128-block; the cast is called lossless.  "DeepSeek-V4-Flash-SI" model card,
模型训练 table: weight block size [128, 128].  Readings: one scale per
(128-row, 128-column) block of each matrix, stored as float32 scale_inv [N/128,
K/128] (the dequant multiplier, w = e4m3 * scale_inv); it is the power of two
2^s of the activation rule (oracle.quant) applied to the block: s =
ceil(log2(amax / 448)) for the exact block maximum, clamped to [-127, 127],
amax = 0 -> s = 0; each element is E4M3(value / 2^s), nearest even, sign kept
(so -0 gives 0x80).  The cast is exact unless a nonzero element falls below
E4M3's resolution (a block whose exponents spread too far); then the rounded
codes are still produced and the cast reports error -4.  E8M0 255 is -3.
"""
from __future__ import annotations

import numpy as np

from .formats import decode_e2m1_packed, decode_e4m3, encode_e4m3_rne_sat


class RepackError(Exception):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


def nvfp4_global_exponent(e8m0_matrix: np.ndarray) -> int:
    b = np.asarray(e8m0_matrix, dtype=np.int64)
    if (b == 255).any():
        raise RepackError(-3, "E8M0 NaN scale")
    e = b - 127
    lo, hi = int(e.min()), int(e.max())
    if lo >= -9 and hi <= 8:
        return 0
    if hi - lo <= 17:
        return hi - 8
    raise RepackError(-4, "exponent span not representable in E4M3")


def repack_mxfp4_to_nvfp4(fp4: np.ndarray, e8m0: np.ndarray):
    """fp4 uint8 [M, N, K/2], e8m0 uint8 [M, N, K/32] ->
    (fp4 [M, N, K/2], e4m3 [M, N, K/16], global float32 [M])."""
    fp4 = np.asarray(fp4, dtype=np.uint8)
    e8m0 = np.asarray(e8m0, dtype=np.uint8)
    M = fp4.shape[0]
    out_s = np.empty(e8m0.shape[:-1] + (e8m0.shape[-1] * 2,), np.uint8)
    glob = np.empty(M, np.float32)
    for m in range(M):
        G = nvfp4_global_exponent(e8m0[m])
        s = encode_e4m3_rne_sat(np.ldexp(1.0, e8m0[m].astype(np.int64) - 127 - G))
        out_s[m, ..., 0::2] = s
        out_s[m, ..., 1::2] = s
        glob[m] = np.float32(np.ldexp(1.0, G))
    return fp4.copy(), out_s, glob


def repack_mxfp4_to_int4g128(fp4: np.ndarray, e8m0: np.ndarray):
    """fp4 uint8 [M, N, K/2], e8m0 uint8 [M, N, K/32] ->
    (int4 packed int8 [M, N, K/2], scale_inv float32 [M, N, K/128])."""
    fp4 = np.asarray(fp4, dtype=np.uint8)
    e8m0 = np.asarray(e8m0, dtype=np.uint8)
    if (e8m0 == 255).any():
        raise RepackError(-3, "E8M0 NaN scale")
    lead = fp4.shape[:-1]
    K = fp4.shape[-1] * 2
    v = decode_e2m1_packed(fp4).reshape(*lead, K // 32, 32)
    v = v * np.ldexp(1.0, e8m0.astype(np.int64) - 127)[..., None]
    with np.errstate(over="ignore"):
        v32 = v.reshape(*lead, K).astype(np.float32)
    if not np.isfinite(v32).all():
        raise RepackError(-4, "dequantised value overflows float32")
    g = v32.reshape(*lead, K // 128, 128)
    amax = np.abs(g).max(axis=-1)
    sinv = np.where(amax > 0, amax / np.float32(7.0), np.float32(1.0)).astype(np.float32)
    q = np.rint(g / sinv[..., None])                     # float32 divide, half-even
    q = np.clip(q, -7, 7).astype(np.int64).reshape(*lead, K)
    nib = (q & 0xF).astype(np.uint8)
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8).view(np.int8)
    return packed, sinv


def repack_mxfp4_to_fp8_block128(fp4: np.ndarray, e8m0: np.ndarray):
    """fp4 uint8 [M, N, K/2], e8m0 uint8 [M, N, K/32] ->
    (e4m3 uint8 [M, N, K], scale_inv float32 [M, N/128, K/128], exact: bool).

    exact is False when some nonzero element is not reproduced bit for bit
    (the GPU then records error -4)."""
    fp4 = np.asarray(fp4, dtype=np.uint8)
    e8m0 = np.asarray(e8m0, dtype=np.uint8)
    if (e8m0 == 255).any():
        raise RepackError(-3, "E8M0 NaN scale")
    M, N, k2 = fp4.shape
    K = 2 * k2
    # exact values in float64 (MXFP4 reaches 6 * 2^127, beyond float32)
    v = decode_e2m1_packed(fp4).reshape(M, N, K // 32, 32)
    v = v * np.ldexp(1.0, e8m0.astype(np.int64) - 127)[..., None]
    v = v.reshape(M, N // 128, 128, K // 128, 128)
    amax = np.abs(v).max(axis=(2, 4))                        # [M, N/128, K/128]
    s = np.zeros(amax.shape, np.int64)
    nz = amax > 0
    # ceil(log2(r)) for r = amax / 448 > 0, exactly: frexp gives r = f * 2^x,
    # f in [0.5, 1); r is a power of two iff f == 0.5
    f, x = np.frexp(amax[nz] / 448.0)
    s[nz] = np.where(f == 0.5, x - 1, x)
    s = np.clip(s, -127, 127)
    scaled = v / np.ldexp(1.0, s)[:, :, None, :, None]
    q = encode_e4m3_rne_sat(scaled)
    exact = bool((decode_e4m3(q) == scaled).all())
    scale_inv = np.ldexp(np.float32(1.0), s).astype(np.float32)
    return q.reshape(M, N, K), scale_inv, exact
