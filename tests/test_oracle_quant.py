"""Pins of the per-128 power-of-two FP8 activation quantisation (step a1 and
the a5 requantisation): hand-derived cases, closed forms and invariants."""
import numpy as np

import synth
from oracle import formats as F
from oracle import quant as Q
from tests.conftest import golden_lines


def _group(elems):
    x = np.zeros((1, 128), np.float32)
    for item in elems:
        i, v = item.split(":")
        x[0, int(i)] = np.float32(float(v))
    return x


def test_hand_cases():
    for ln in golden_lines("act_quant_cases.txt"):
        name, ins, sbyte, outs = [p.strip() for p in ln.split("|")]
        x = _group(ins.split())
        # the inputs are bf16 values: they must survive a bf16 round trip
        assert (F.decode_bf16_bits(synth.to_bf16_bits(x)) == x).all(), name
        q, s = Q.quantize_act_fp8(synth.to_bf16_bits(x))
        assert s[0, 0] == int(sbyte), (name, s[0, 0])
        for item in outs.split():
            i, c = item.split(":")
            assert q[0, int(i)] == int(c, 16), (name, i, hex(q[0, int(i)]), c)


def test_ceil_log2_exact():
    for e in range(-149, 128):
        v = np.float32(2.0 ** e)
        assert Q.ceil_log2_f32(np.array([v]))[0] == e
        nxt = np.nextafter(v, np.float32(np.inf))
        if np.isfinite(nxt):
            assert Q.ceil_log2_f32(np.array([nxt]))[0] == e + 1


def test_amax_lands_in_top_binade():
    mag = 10.0 ** np.repeat(np.arange(-4, 4), 8)[:, None]          # 64 rows, 8 decades
    x = synth.bf16_bits_to_f32(synth.to_bf16_bits(synth.normal(0, 7, 64 * 512).reshape(64, 512) * mag))
    q, s = Q.quantize_fp8_pow2(x)
    k = s.astype(np.int64) - 127
    amax = np.abs(x.reshape(64, 4, 128)).max(-1)
    r = amax / np.ldexp(1.0, k)
    assert ((r > 224) & (r <= 448)).all()


def test_idempotent_and_error_bound():
    x = synth.normal(0, 8, 32 * 1024).reshape(32, 1024).astype(np.float32)
    q, s = Q.quantize_fp8_pow2(x)
    d = Q.dequantize_fp8_pow2(q, s)
    q2, s2 = Q.quantize_fp8_pow2(d.astype(np.float32))
    # values are reproduced exactly; the scale may drop by one when the group
    # maximum rounded down to 224 * 2^k
    assert (Q.dequantize_fp8_pow2(q2, s2) == d).all()
    assert ((s.astype(int) - s2.astype(int)) >= 0).all() and ((s.astype(int) - s2.astype(int)) <= 1).all()
    # |error| <= half an E4M3 step at the element's binade (relative 2^-4)
    k = np.repeat(s.astype(np.int64) - 127, 128, axis=1)
    y = np.abs(x.astype(np.float64)) / np.ldexp(1.0, k)
    step = np.where(y < 2.0 ** -6, 2.0 ** -9, np.ldexp(1.0, np.floor(np.log2(np.maximum(y, 1e-300))).astype(int) - 3))
    assert (np.abs(d - x) <= 0.5 * step * np.ldexp(1.0, k) + 0.0).all()


def test_pow2_equivariance():
    x = synth.normal(0, 9, 8 * 256).reshape(8, 256).astype(np.float32)
    q, s = Q.quantize_fp8_pow2(x)
    for j in (-20, -3, 5, 40):
        q2, s2 = Q.quantize_fp8_pow2((x * np.float32(2.0 ** j)).astype(np.float32))
        assert (q2 == q).all() and (s2.astype(int) == s.astype(int) + j).all()


def test_exhaustive_bf16_single_element_groups():
    # every finite bf16 value alone in a group: the code must be the nearest
    # E4M3 value of x / 2^k, with x / 2^k in (224, 448]
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = F.decode_bf16_bits(b)
    b = b[np.isfinite(v) & (v != 0)]
    x = np.zeros((len(b), 128), np.uint16)
    x[:, 5] = b
    q, s = Q.quantize_act_fp8(x)
    xv = F.decode_bf16_bits(b).astype(np.float64)
    k = s[:, 0].astype(np.int64) - 127
    y = xv / np.ldexp(1.0, k)
    ok = (k == -127) | ((np.abs(y) > 224) & (np.abs(y) <= 448))
    assert ok.all()
    deq = F.decode_e4m3(q[:, 5])
    finite = F.E4M3_TABLE[:0x7F]
    best = np.abs(np.abs(y)[:, None] - finite[None, :]).min(axis=1)
    assert (np.abs(np.abs(deq) - np.abs(y)) == best).all()
    assert (q[:, [0, 127]] == 0).all()
