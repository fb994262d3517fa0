"""Expert FFN: grouped w1/w3 GEMM, SwiGLU with +-10 clamp, w2 GEMM, combine.

Passages:
  * "DeepSeek-V4-Flash-SI" model card, 架构特性 (Mixture of Experts paragraph):
    routed + shared experts, SwiGLU activation clamped to +-10.0, routing
    scale 1.5; 低精度计算: FP4 E2M1 expert weights with an E8M0 scale per 32
    elements, activations FP8 E4M3 with a power-of-two scale per 128.
  * "DeepSeek-V4-Flash-0731-W4AFP8-mt" model card, 量化方式 / 权重约定: expert
    projections are named w1, w2, w3; weights are [N, K] with K the input
    dimension; the W4AFP8 form holds INT4 weights with a float32
    weight_scale_inv of shape [N, K/128] and dynamic E4M3 activations.
  * FP8 shared expert: "DeepSeek-V4-Pro-0813-nvfp4-DSpark" walkthrough (only-
    experts section: the shared experts stay FP8) and the "DeepSeek-V4-Flash-SI"
    model card (模型训练: weight block size [128, 128]).  Reading: E4M3 weights
    [N, K] with a float32 weight_scale_inv [N/128, K/128] per [128, 128] block
    (w = e4m3 * scale_inv), the same dynamic E4M3 activations.
  * PTPC-FP8: "DeepSeek-V4.1-Flash-Quark-PTPC-FP8" walkthrough, 核心参数
    (quant_scheme ptpc_fp8): E4M3 everywhere; weights per output channel with
    a static scale (ch_axis 0, min-max observer), activations per token with a
    dynamic scale, symmetric, half_even rounding; the routed and shared
    experts are both quantised, from the dequantised base weights.  Readings:
    scale = amax / 448 (float32 IEEE divide; 1.0 when amax == 0); q =
    E4M3(x / scale) with a float32 IEEE divide, nearest even, saturating; the
    GEMM accumulates sum q_a * q_w and multiplies by scale_a[token] *
    scale_w[channel]; h after SwiGLU is requantised per token over its I
    columns.

Readings: w1 = gate, w3 = up, w2 = down; both gate and up are clamped to
[-limit, limit] before silu(gate) * up (which tensors the clamp applies to is
not stated: parity unpinned beyond the closed forms); the router weight is
applied in the combine, after w2; the shared expert has weight 1.0 (no route
scale).  The GEMMs are the plain definition: dequantise both operands exactly
to float64 and multiply (numpy matmul as the library step).  h is rounded to
float32 before requantisation because the quantisation decision is taken in
float32 (the kernels' precision) -- see oracle.quant.
"""
from __future__ import annotations

import numpy as np

from .formats import decode_bf16_bits, decode_e2m1_packed, decode_e4m3, decode_e8m0, encode_e4m3_rne_sat
from .permute import gather_rows, permute
from .quant import dequantize_fp8_pow2, quantize_act_fp8, quantize_fp8_pow2
from .route import route_hash, route_topk


def dequant_mxfp4(packed: np.ndarray, e8m0: np.ndarray) -> np.ndarray:
    """MXFP4 [N, K/2] + E8M0 [N, K/32] -> float64 [N, K]."""
    v = decode_e2m1_packed(packed)
    N, K = v.shape[-2], v.shape[-1]
    s = decode_e8m0(e8m0)
    return (v.reshape(*v.shape[:-1], K // 32, 32) * s[..., None]).reshape(v.shape)


def dequant_int4g128(q_packed: np.ndarray, scale_inv: np.ndarray) -> np.ndarray:
    """Symmetric INT4 [N, K/2] (two's complement, element 2i in the low nibble)
    + float32 scale_inv [N, K/128] -> float64 [N, K]."""
    q_packed = np.asarray(q_packed).view(np.uint8)
    lo = (q_packed & 0xF).astype(np.int64)
    hi = (q_packed >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    q = np.empty(q_packed.shape[:-1] + (q_packed.shape[-1] * 2,), np.float64)
    q[..., 0::2] = lo
    q[..., 1::2] = hi
    N, K = q.shape[-2], q.shape[-1]
    s = np.asarray(scale_inv, dtype=np.float32).astype(np.float64)
    return (q.reshape(*q.shape[:-1], K // 128, 128) * s[..., None]).reshape(q.shape)


def grouped_gemm(a_q, a_s, offsets, w_deq_fn, n_groups):
    """Rows offsets[g]:offsets[g+1] of the FP8 operand times group g's weights^T.

    a_q: E4M3 [R, K]; a_s: E8M0 [R, K/128]; w_deq_fn(g) -> float64 [N, K].
    Returns float64 [R, N]."""
    a = dequantize_fp8_pow2(a_q, a_s)
    out = None
    for g in range(n_groups):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 == r0:
            continue
        w = w_deq_fn(g)
        if out is None:
            out = np.zeros((a.shape[0], w.shape[0]), np.float64)
        out[r0:r1] = a[r0:r1] @ w.T
    if out is None:
        out = np.zeros((a.shape[0], 0), np.float64)
    return out


def _memo(cache, arrays, fn):
    """fn() -- or, with a cache dict, its value stored under the memory
    address and shape of the source arrays: groups whose weights occupy the
    same memory dequantise once (a saving of time, not a change of values)."""
    if cache is None:
        return fn()
    key = tuple((np.asarray(a).__array_interface__["data"][0], np.asarray(a).shape) for a in arrays)
    if key not in cache:
        cache[key] = fn()
    return cache[key]


def grouped_gemm_mxfp4(a_q, a_s, offsets, w_fp4, w_e8m0, cache=None):
    """Steps a4 / a6: FP8 rows x MXFP4 weights [G, N, K/2] -> float64 [R, N]."""
    N = w_fp4.shape[1]
    out = grouped_gemm(a_q, a_s, offsets,
                       lambda g: _memo(cache, (w_fp4[g], w_e8m0[g]), lambda: dequant_mxfp4(w_fp4[g], w_e8m0[g])),
                       w_fp4.shape[0])
    return out if out.shape[1] else np.zeros((a_q.shape[0], N))


def grouped_gemm_w4afp8(a_q, a_s, offsets, w_int4, w_scale_inv, cache=None):
    """Step a10: FP8 rows x INT4-g128 weights [G, N, K/2] -> float64 [R, N]."""
    N = w_int4.shape[1]
    out = grouped_gemm(a_q, a_s, offsets,
                       lambda g: _memo(cache, (w_int4[g], w_scale_inv[g]),
                                       lambda: dequant_int4g128(w_int4[g], w_scale_inv[g])),
                       w_int4.shape[0])
    return out if out.shape[1] else np.zeros((a_q.shape[0], N))


def dequant_fp8_block128(q: np.ndarray, scale_inv: np.ndarray) -> np.ndarray:
    """E4M3 [N, K] + float32 scale_inv [N/128, K/128] -> float64 [N, K]."""
    v = decode_e4m3(q)
    s = np.asarray(scale_inv, dtype=np.float32).astype(np.float64)
    return v * np.repeat(np.repeat(s, 128, axis=-2), 128, axis=-1)


def grouped_gemm_fp8_block128(a_q, a_s, offsets, w_q, w_scale_inv):
    """FP8 rows x FP8 [128, 128]-block weights [G, N, K] -> float64 [R, N]."""
    N = w_q.shape[1]
    out = grouped_gemm(a_q, a_s, offsets, lambda g: dequant_fp8_block128(w_q[g], w_scale_inv[g]), w_q.shape[0])
    return out if out.shape[1] else np.zeros((a_q.shape[0], N))


def quantize_fp8_per_row(x: np.ndarray):
    """float32 [rows, cols] -> (E4M3 [rows, cols], float32 scale [rows]):
    scale = amax / 448 (float32 divide, 1 when amax == 0), q = E4M3(x / scale)
    with a float32 divide, nearest even (PTPC-FP8 per-token / per-channel rule,
    "DeepSeek-V4.1-Flash-Quark-PTPC-FP8" walkthrough, 核心参数: symmetric,
    half_even).  Parity unpinned: the page names the scheme, not the scale
    formula; amax / 448 is the plain symmetric reading."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.abs(x32).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    q = encode_e4m3_rne_sat((x32 / scale[..., None]).astype(np.float64))
    return q, scale


def ptpc_weights(fp4: np.ndarray, e8m0: np.ndarray):
    """MXFP4 [G, N, K/2] + E8M0 -> (E4M3 [G, N, K], float32 per-channel scale [G, N]):
    the per-row rule applied to the exact float32 dequantisation."""
    w = dequant_mxfp4(fp4, e8m0).astype(np.float32)
    return quantize_fp8_per_row(w)


def grouped_gemm_ptpc(a_q, a_scale, offsets, w_q, w_scale):
    """E4M3 rows [R, K] with per-row scales [R] x E4M3 weights [G, N, K] with
    per-channel scales [G, N] -> float64 [R, N]."""
    a = decode_e4m3(a_q) * np.asarray(a_scale, np.float32).astype(np.float64)[:, None]
    N = w_q.shape[1]
    out = np.zeros((a.shape[0], N), np.float64)
    for g in range(w_q.shape[0]):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 > r0:
            w = decode_e4m3(w_q[g]) * np.asarray(w_scale[g], np.float32).astype(np.float64)[:, None]
            out[r0:r1] = a[r0:r1] @ w.T
    return out


def moe_layer_ptpc(x_bf16, logits, w13_q, w13_scale, w2_q, w2_scale, topk, route_scale=1.5,
                   swiglu_limit=10.0, has_shared=1, route_norm=1, tokens=None):
    """The expert path with PTPC-FP8 weights (w13_q [G, 2I, H] + [G, 2I], w2_q
    [G, H, I] + [G, H]; G = E + has_shared) and per-token dynamic activations."""
    x_bf16 = np.asarray(x_bf16)
    logits = np.asarray(logits, dtype=np.float32)
    if tokens is not None:
        x_bf16 = x_bf16[tokens]
        logits = logits[tokens]
    T, H = x_bf16.shape
    E = logits.shape[1]
    I = w2_q.shape[2]
    xq, sx = quantize_fp8_per_row(decode_bf16_bits(x_bf16))
    idx, w = route_topk(logits, topk, route_scale, route_norm)
    counts, offsets, perm, inv, src = permute(idx, E, has_shared)
    xq_p, sx_p = xq[src], sx[src]
    gu = grouped_gemm_ptpc(xq_p, sx_p, offsets, w13_q, w13_scale)
    h = swiglu_clamp(gu, I, swiglu_limit).astype(np.float32)
    hq, sh = quantize_fp8_per_row(h)
    o = grouped_gemm_ptpc(hq, sh, offsets, w2_q, w2_scale)
    y = combine(o, inv, w, offsets, has_shared)
    return dict(xq=xq, sx=sx, idx=idx, w=w, offsets=offsets, inv=inv, gu=gu, h=h, hq=hq, sh=sh, o=o, y=y)


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def swiglu_clamp(gu: np.ndarray, I: int, limit: float = 10.0) -> np.ndarray:
    """Step a5 (activation): gu float [R, 2I] (gate | up) -> h float64 [R, I]."""
    gu = np.asarray(gu, dtype=np.float64)
    g = np.clip(gu[:, :I], -limit, limit)
    u = np.clip(gu[:, I:2 * I], -limit, limit)
    return silu(g) * u


def swiglu_quant(gu: np.ndarray, I: int, limit: float = 10.0):
    """Step a5: SwiGLU then the per-128 power-of-two FP8 requantisation."""
    h = swiglu_clamp(gu, I, limit)
    return quantize_fp8_pow2(h.astype(np.float32))


def combine(o: np.ndarray, inv: np.ndarray, w: np.ndarray, offsets: np.ndarray,
            has_shared: int = 1) -> np.ndarray:
    """Step a7: y[t] = sum_j w[t, j] * o[inv[t, j]] + o[shared row of t] (float64)."""
    T, k = w.shape
    y = np.zeros((T, o.shape[1]), np.float64)
    invr = np.asarray(inv).reshape(T, k)
    for j in range(k):
        y += np.asarray(w[:, j], np.float64)[:, None] * o[invr[:, j]]
    if has_shared:
        E = len(offsets) - 2
        y += o[int(offsets[E]) + np.arange(T)]
    return y


def moe_layer(x_bf16, logits, w13, w13_e8m0, w2, w2_e8m0, topk, route_scale=1.5,
              swiglu_limit=10.0, has_shared=1, route_norm=1, weights="mxfp4",
              w13_int4=None, w13_sinv=None, w2_int4=None, w2_sinv=None, tokens=None,
              shared_fp8=None, token_ids=None, tid2eid=None, cache=None):
    """The whole expert path (a1 -> a7) for the tokens listed in ``tokens``
    (all tokens when None).  Token outputs are independent given the routing,
    so a subset gives exactly those rows of the full result.

    tid2eid / token_ids: hash routing (oracle.route.route_hash) in place of
    the top-k router: the experts of token t are tid2eid[token_ids[t]].

    cache: optional dict in which dequantised expert weights are kept, keyed
    by the memory of their source arrays (experts sharing memory dequantise
    once; the arithmetic is unchanged).

    shared_fp8: optional (w13_q, w13_scale_inv, w2_q, w2_scale_inv) of the
    shared expert in FP8 with [128, 128] block scales ([2I, H], [2I/128,
    H/128], [H, I], [H/128, I/128]); the shared group then uses these instead
    of group E of the routed weight arrays.

    Returns a dict of the intermediates (indices refer to the subset)."""
    x_bf16 = np.asarray(x_bf16)
    logits = np.asarray(logits, dtype=np.float32)
    if tokens is not None:
        x_bf16 = x_bf16[tokens]
        logits = logits[tokens]
        if token_ids is not None:
            token_ids = np.asarray(token_ids)[tokens]
    T, H = x_bf16.shape
    E = logits.shape[1]
    I = (w2 if weights == "mxfp4" else w2_int4).shape[2] * 2
    xq, sx = quantize_act_fp8(x_bf16)
    if tid2eid is not None:
        assert np.asarray(tid2eid).shape[1] == topk
        idx, w = route_hash(token_ids, tid2eid, logits, route_scale, route_norm)
    else:
        idx, w = route_topk(logits, topk, route_scale, route_norm)
    counts, offsets, perm, inv, src = permute(idx, E, has_shared)
    xq_p, sx_p = gather_rows(xq, sx, src)
    if weights == "mxfp4":
        gu = grouped_gemm_mxfp4(xq_p, sx_p, offsets, w13, w13_e8m0, cache)
    else:
        gu = grouped_gemm_w4afp8(xq_p, sx_p, offsets, w13_int4, w13_sinv, cache)
    shared = shared_fp8 is not None and has_shared
    r0, r1 = (int(offsets[E]), int(offsets[E + 1])) if shared else (0, 0)
    if r1 > r0:      # the shared group with its FP8 weights
        gu[r0:r1] = dequantize_fp8_pow2(xq_p[r0:r1], sx_p[r0:r1]) @ \
            dequant_fp8_block128(shared_fp8[0], shared_fp8[1]).T
    hq, sh = swiglu_quant(gu, I, swiglu_limit)
    if weights == "mxfp4":
        o = grouped_gemm_mxfp4(hq, sh, offsets, w2, w2_e8m0, cache)
    else:
        o = grouped_gemm_w4afp8(hq, sh, offsets, w2_int4, w2_sinv, cache)
    if r1 > r0:
        o[r0:r1] = dequantize_fp8_pow2(hq[r0:r1], sh[r0:r1]) @ dequant_fp8_block128(shared_fp8[2], shared_fp8[3]).T
    y = combine(o, inv, w, offsets, has_shared)
    return dict(xq=xq, sx=sx, idx=idx, w=w, counts=counts, offsets=offsets, perm=perm,
                inv=inv, xq_perm=xq_p, sx_perm=sx_p, gu=gu, hq=hq, sh=sh, o=o, y=y)
