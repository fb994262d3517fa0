"""Pins of the expert FFN oracle (a4-a7, a10): pure-Python loops on tiny
shapes, integer-exact special cases, the E=1/k=1 reduction and the SwiGLU
closed forms."""
import numpy as np

import synth
from oracle import ffn
from oracle import formats as F
from oracle import quant as Q


def test_dequant_mxfp4_loop():
    w, s = synth.quantize_mxfp4(synth.normal(0, 31, 4 * 64).reshape(4, 64) * 0.02)
    d = ffn.dequant_mxfp4(w, s)
    for n in range(4):
        for kk in range(64):
            byte = int(w[n, kk // 2])
            nib = (byte & 0xF) if kk % 2 == 0 else (byte >> 4)
            assert d[n, kk] == F.E2M1_TABLE[nib] * 2.0 ** (int(s[n, kk // 32]) - 127)


def test_grouped_gemm_matches_python_loop():
    R, K, N, G = 9, 256, 3, 3
    aq = synth.random_e4m3(1, 1, (R, K), max_code=0x60)
    as_ = synth.random_bytes(1, 2, (R, K // 128), 120, 134)
    wq = synth.random_bytes(1, 3, (G, N, K // 2))
    ws = synth.random_bytes(1, 4, (G, N, K // 32), 118, 130)
    offsets = np.array([0, 4, 4, 9])
    out = ffn.grouped_gemm_mxfp4(aq, as_, offsets, wq, ws)
    for g in range(G):
        for r in range(offsets[g], offsets[g + 1]):
            for n in range(N):
                acc = 0.0
                for kk in range(K):
                    a = F.E4M3_TABLE[aq[r, kk]] * 2.0 ** (int(as_[r, kk // 128]) - 127)
                    byte = int(wq[g, n, kk // 2])
                    nib = (byte & 0xF) if kk % 2 == 0 else (byte >> 4)
                    acc += a * F.E2M1_TABLE[nib] * 2.0 ** (int(ws[g, n, kk // 32]) - 127)
                assert abs(out[r, n] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_integer_exact_case():
    R, K, N = 5, 512, 4
    aq = synth.small_int_e4m3(2, 1, (R, K))
    wq = synth.small_int_fp4(2, 2, (1, N, K // 2))
    out = ffn.grouped_gemm_mxfp4(aq, np.full((R, K // 128), 127, np.uint8), [0, R], wq,
                                 np.full((1, N, K // 32), 127, np.uint8))
    a = F.decode_e4m3(aq)
    w = F.decode_e2m1_packed(wq[0])
    assert (a == np.round(a)).all() and (w == np.round(w)).all()
    assert (out == (a.astype(np.int64) @ w.astype(np.int64).T)).all()


def test_swiglu_closed_forms():
    I = 128
    gu = np.zeros((4, 2 * I))
    gu[1, :I], gu[1, I:] = 50.0, 50.0                     # both clamp to 10
    gu[2, :I], gu[2, I:] = -50.0, 3.0                     # gate clamps to -10
    gu[3, :I], gu[3, I:] = 2.0, -1.0
    h = ffn.swiglu_clamp(gu, I)
    assert (h[0] == 0).all()
    np.testing.assert_allclose(h[1], 10.0 / (1 + np.exp(-10.0)) * 10.0, rtol=1e-15)
    np.testing.assert_allclose(h[2], -10.0 / (1 + np.exp(10.0)) * 3.0, rtol=1e-15)
    np.testing.assert_allclose(h[3], -2.0 / (1 + np.exp(-2.0)), rtol=1e-15)


def test_single_expert_reduction():
    """E = 1, k = 1, normalised: the router weight is exactly 1.5, so
    y = 1.5 * FFN_0(x) + FFN_shared(x) with FFN the plain dense expert."""
    T, H, I = 6, 256, 128
    x = synth.to_bf16_bits(synth.normal(3, 1, T * H).reshape(T, H))
    logits = synth.uniform_logits(3, T, 1)
    w13, s13, w2, s2 = synth.expert_weights(3, 2, H, I)
    r = ffn.moe_layer(x, logits, w13, s13, w2, s2, topk=1)
    assert np.allclose(r["w"], 1.5)

    def dense(e):
        xq, sx = Q.quantize_act_fp8(x)
        a = Q.dequantize_fp8_pow2(xq, sx)
        gu = a @ ffn.dequant_mxfp4(w13[e], s13[e]).T
        g, u = np.clip(gu[:, :I], -10, 10), np.clip(gu[:, I:], -10, 10)
        hq, sh = Q.quantize_fp8_pow2((g / (1 + np.exp(-g)) * u).astype(np.float32))
        return Q.dequantize_fp8_pow2(hq, sh) @ ffn.dequant_mxfp4(w2[e], s2[e]).T

    np.testing.assert_allclose(r["y"], 1.5 * dense(0) + dense(1), rtol=1e-12, atol=1e-15)


def test_combine_k3_hand_built():
    """Combine at k = 3 with the shared expert and a grouping whose inv is not
    the identity, checked against values worked out by hand.  Tokens 0, 1 pick
    experts [2, 0, 3] and [0, 1, 2] (E = 4), so pairs p = 0..5 go to experts
    2, 0, 3, 0, 1, 2; grouped in ascending pair id per expert, the rows are
    e0: p1, p3 | e1: p4 | e2: p0, p5 | e3: p2 | shared: t0, t1, hence
    inv = [3, 0, 5, 1, 2, 4] and perm = [1, 3, 4, 0, 5, 2, 6, 7].
    With o[r] = [r + 1, 10 (r + 1)]:
      y[0] = 0.5 o[3] + 0.25 o[0] + 0.75 o[5] + o[6] = 2 + 0.25 + 4.5 + 7
      y[1] = 1.0 o[1] + 0.125 o[2] + 0.375 o[4] + o[7] = 2 + 0.375 + 1.875 + 8
    (indexing o by perm gives 12.75 for y[0, 0]; reversing the slot weights
    of token 0 gives 13.25)."""
    from oracle import permute as Pm
    idx = np.array([[2, 0, 3], [0, 1, 2]], np.int32)
    counts, offsets, perm, inv, src = Pm.permute(idx, 4, 1)
    assert counts.tolist() == [2, 1, 2, 1, 2] and offsets.tolist() == [0, 2, 3, 5, 6, 8]
    assert inv.tolist() == [3, 0, 5, 1, 2, 4] and perm.tolist() == [1, 3, 4, 0, 5, 2, 6, 7]
    assert src.tolist() == [0, 1, 1, 0, 1, 0, 0, 1]
    o = np.array([[r + 1, 10.0 * (r + 1)] for r in range(8)])
    w = np.array([[0.5, 0.25, 0.75], [1.0, 0.125, 0.375]])
    y = ffn.combine(o, inv, w, offsets, has_shared=1)
    assert y.tolist() == [[13.75, 137.5], [12.25, 122.5]]
    # the same sum as a plain loop over tokens, slots and columns
    for t in range(2):
        for c in range(2):
            acc = o[offsets[4] + t, c]
            for j in range(3):
                acc += w[t, j] * o[inv[t * 3 + j], c]
            assert y[t, c] == acc
    # without the shared expert the shared rows are not added
    y0 = ffn.combine(o[:6], inv, w, np.array([0, 2, 3, 5, 6, 6]), has_shared=0)
    assert y0.tolist() == [[6.75, 67.5], [4.25, 42.5]]


def test_token_subset_equals_full_rows():
    wl = synth.tiny_layer(0)
    full = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    sub = [3, 7, 11]
    part = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk,
                         tokens=sub)
    np.testing.assert_array_equal(part["y"], full["y"][sub])


def test_layer_hash_routing_with_topk_table_equals_topk_layer():
    """The hash-routed layer whose table rows hold each token's top-k experts
    (one vocabulary entry per token) is the top-k routed layer, bit for bit."""
    from oracle import route as R
    wl = synth.tiny_layer(7)
    idx, _ = R.route_topk(wl.logits, wl.topk)
    ref = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    got = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk,
                        token_ids=np.arange(wl.T), tid2eid=idx)
    np.testing.assert_array_equal(got["y"], ref["y"])
    sub = [2, 9]
    part = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk,
                         token_ids=np.arange(wl.T), tid2eid=idx, tokens=sub)
    np.testing.assert_array_equal(part["y"], ref["y"][sub])


def test_w4afp8_dequant_loop():
    q = np.array([[0x7F, 0x98] + [0] * 62], np.uint8).view(np.int8)   # nibbles 15,7,8,9
    d = ffn.dequant_int4g128(q, np.array([[0.5]], np.float32))
    assert d[0, :4].tolist() == [-0.5, 3.5, -4.0, -3.5]


# ------------------------- FP8 [128, 128]-block weights (shared expert) -------------------------
def test_fp8_block_dequant_closed_forms():
    """Code 0x38 is 1.0; every [128, 128] block takes its own scale_inv."""
    q = np.full((256, 256), 0x38, np.uint8)
    sinv = np.array([[1.0, 2.0], [0.25, 8.0]], np.float32)
    w = ffn.dequant_fp8_block128(q, sinv)
    assert (w[:128, :128] == 1.0).all() and (w[:128, 128:] == 2.0).all()
    assert (w[128:, :128] == 0.25).all() and (w[128:, 128:] == 8.0).all()


def test_fp8_gemm_matches_mxfp4_gemm_after_lossless_cast():
    """Weights cast losslessly to FP8 [128, 128] blocks give the MXFP4 GEMM's
    result exactly (an independent path to the same dequantised weights)."""
    from oracle import repack as Rp
    G, N, K = 2, 256, 384
    w = synth.random_bytes(12, 1, (G, N, K // 2))
    ws = synth.random_bytes(12, 2, (G, N, K // 32), 119, 126)
    q, sinv, exact = Rp.repack_mxfp4_to_fp8_block128(w, ws)
    assert exact
    offsets = np.array([0, 5, 40], np.int32)
    a = synth.random_e4m3(12, 3, (40, K))
    asc = synth.random_bytes(12, 4, (40, K // 128), 120, 130)
    np.testing.assert_array_equal(ffn.grouped_gemm_fp8_block128(a, asc, offsets, q, sinv),
                                  ffn.grouped_gemm_mxfp4(a, asc, offsets, w, ws))


def test_layer_shared_fp8_equals_mxfp4_shared_after_cast():
    """The tiny layer with its shared expert cast losslessly to FP8 gives the
    same output as with the MXFP4 shared expert."""
    from oracle import repack as Rp
    wl = synth.tiny_layer(4)
    E = wl.E
    q13, s13, ok13 = Rp.repack_mxfp4_to_fp8_block128(wl.w13[E:E + 1], wl.w13_e8m0[E:E + 1])
    q2, s2, ok2 = Rp.repack_mxfp4_to_fp8_block128(wl.w2[E:E + 1], wl.w2_e8m0[E:E + 1])
    assert ok13 and ok2
    ref = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    got = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk,
                        shared_fp8=(q13[0], s13[0], q2[0], s2[0]))
    np.testing.assert_array_equal(got["y"], ref["y"])


def test_fp8_block_scale_is_linear_per_block():
    """Doubling one block's scale_inv doubles exactly that block's contribution."""
    K = 256
    q = synth.small_int_e4m3(13, 1, (128, K))
    a = synth.small_int_e4m3(13, 2, (8, K))
    asc = np.full((8, K // 128), 127, np.uint8)
    off = np.array([0, 8], np.int32)
    s1 = np.array([[1.0, 1.0]], np.float32)
    s2 = np.array([[1.0, 2.0]], np.float32)
    base = ffn.grouped_gemm_fp8_block128(a, asc, off, q[None], s1[None])
    twice = ffn.grouped_gemm_fp8_block128(a, asc, off, q[None], s2[None])
    hi = ffn.grouped_gemm_fp8_block128(a[:, :], asc, off, np.where(np.arange(K) >= 128, q, 0)[None], s1[None])
    np.testing.assert_array_equal(twice, base + hi)


# --------------------------------- PTPC-FP8 ---------------------------------------
def test_ptpc_per_row_closed_forms():
    # amax 3.5 -> scale 3.5 / 448 = 2^-7 exactly; 3.5 -> 448 (0x7E), 1.0 -> 128 (0x70)
    q, s = ffn.quantize_fp8_per_row(np.array([[3.5, 1.0, -1.0, 0.0]], np.float32))
    assert s[0] == np.float32(2.0 ** -7)
    assert list(q[0]) == [0x7E, 0x70, 0xF0, 0x00]
    # an all-zero row: scale 1, codes 0
    q, s = ffn.quantize_fp8_per_row(np.zeros((1, 8), np.float32))
    assert s[0] == 1.0 and (q == 0).all()


def test_ptpc_per_row_error_bound():
    """|dequant - x| <= 2^-4 |x| for normal E4M3 codes, <= 2^-10 * scale below."""
    x = (synth.normal(21, 1, 64 * 512) * 3).astype(np.float32).reshape(64, 512)
    q, s = ffn.quantize_fp8_per_row(x)
    back = F.decode_e4m3(q) * s[:, None].astype(np.float64)
    err = np.abs(back - x)
    assert (err <= np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s[:, None])).all()
    # the row maximum lands on 448 up to the float32 divide
    assert (np.abs(F.decode_e4m3(q)).max(axis=1) == 448.0).all()


def test_ptpc_gemm_integer_case():
    """Unit scales and small-integer E4M3 codes: the result is the integer
    matmul, computed here in int64."""
    a = synth.small_int_e4m3(22, 1, (30, 256))
    w = synth.small_int_e4m3(22, 2, (2, 128, 256))
    off = np.array([0, 11, 30], np.int32)
    got = ffn.grouped_gemm_ptpc(a, np.ones(30, np.float32), off, w, np.ones((2, 128), np.float32))
    ai = F.decode_e4m3(a).astype(np.int64)
    wi = F.decode_e4m3(w).astype(np.int64)
    ref = np.concatenate([ai[:11] @ wi[0].T, ai[11:] @ wi[1].T])
    np.testing.assert_array_equal(got, ref.astype(np.float64))


def test_ptpc_scale_is_pow2_equivariant():
    """Scaling a row by 2^j scales its per-row scale by 2^j and keeps the codes."""
    x = (synth.normal(23, 1, 4 * 256) * 0.7).astype(np.float32).reshape(4, 256)
    q, s = ffn.quantize_fp8_per_row(x)
    q2, s2 = ffn.quantize_fp8_per_row(x * np.float32(8.0))
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s2, s * np.float32(8.0))


def test_ptpc_layer_token_subset():
    wl = synth.tiny_layer(6)
    q13, s13 = ffn.ptpc_weights(wl.w13, wl.w13_e8m0)
    q2, s2 = ffn.ptpc_weights(wl.w2, wl.w2_e8m0)
    full = ffn.moe_layer_ptpc(wl.x_bf16, wl.logits, q13, s13, q2, s2, wl.topk)
    toks = np.array([1, 4, 9])
    sub = ffn.moe_layer_ptpc(wl.x_bf16, wl.logits, q13, s13, q2, s2, wl.topk, tokens=toks)
    np.testing.assert_allclose(sub["y"], full["y"][toks], rtol=0, atol=1e-12 * np.abs(full["y"]).max())


def test_ptpc_weights_per_output_channel():
    """The weight scale is per output channel (row of [N, K]): rows with very
    different magnitudes each reach code 448 and dequantise within the E4M3
    bound of their own scale; the scale is amax/448 of the exact MXFP4 values."""
    N, K = 6, 64
    fp4 = synth.random_bytes(24, 1, (1, N, K // 2))
    e8 = np.repeat((np.arange(N, dtype=np.uint8) * 9 + 100)[:, None], K // 32, axis=1)[None]
    q, s = ffn.ptpc_weights(fp4, e8)
    w = ffn.dequant_mxfp4(fp4, e8)[0]
    amax = np.abs(w).max(axis=1)
    np.testing.assert_array_equal(s[0], (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    assert (np.abs(F.decode_e4m3(q[0])).max(axis=1) == 448.0).all()
    back = F.decode_e4m3(q[0]) * s[0][:, None].astype(np.float64)
    assert (np.abs(back - w) <= np.maximum(2.0 ** -4 * np.abs(w), 2.0 ** -10 * s[0][:, None])).all()


def test_dequant_cache_changes_no_value():
    """The optional dequantisation memo gives the uncached result bit for bit,
    on experts that share memory (repeated prototypes) and on distinct ones."""
    wl = synth.tiny_layer(8)
    views = synth.expert_views(8, wl.E + 1, wl.H, wl.I, n_proto=3)
    full = [v.materialize() for v in views]
    cache = {}
    a = ffn.moe_layer(wl.x_bf16, wl.logits, *views, wl.topk, cache=cache)
    b = ffn.moe_layer(wl.x_bf16, wl.logits, *full, wl.topk)
    np.testing.assert_array_equal(a["y"], b["y"])
    assert 0 < len(cache) <= 6            # at most 3 prototypes x (w13, w2)
    c = ffn.moe_layer(wl.x_bf16, wl.logits, *full, wl.topk, cache={})
    np.testing.assert_array_equal(c["y"], b["y"])
