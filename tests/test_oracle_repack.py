"""Pins of the repack oracles (a8, a9): the lossless property of the NVFP4
cast (exhaustive over codes x exponents), the storage-table facts, the INT4
shape example of the W4AFP8 card, error bounds and the error codes."""
import numpy as np
import pytest

import synth
from oracle import ffn
from oracle import formats as F
from oracle import repack as Rp
from tests.conftest import golden_lines


def _nvfp4_dequant(fp4, e4m3, glob):
    v = F.decode_e2m1_packed(fp4)
    s = F.decode_e4m3(e4m3)
    K = v.shape[-1]
    return (v.reshape(*v.shape[:-1], K // 16, 16) * s[..., None]).reshape(v.shape) * glob


def test_nvfp4_lossless_exhaustive():
    # every code (16) in every byte position against every exponent span that
    # fits: blocks with exponents lo .. lo+17 for several lo
    for lo in (-127, -40, -9, -3, 0, 100, 109):
        exps = np.arange(lo, lo + 18)
        N = len(exps)
        e8 = np.repeat((exps + 127)[:, None], 2, axis=1).astype(np.uint8)   # K = 64
        fp4 = np.tile(np.arange(256, dtype=np.uint8)[None, :32], (N, 1))    # all nibble pairs
        out_fp4, out_s, glob = Rp.repack_mxfp4_to_nvfp4(fp4[None], e8[None])
        assert (out_fp4 == fp4[None]).all()
        assert out_s.shape[-1] == 2 * e8.shape[-1]
        src = ffn.dequant_mxfp4(fp4, e8)
        dst = _nvfp4_dequant(out_fp4[0], out_s[0], np.float64(glob[0]))
        assert (src == dst).all()


def test_nvfp4_storage_table():
    facts = {ln.split()[0]: ln.split()[1:] for ln in golden_lines("nvfp4_storage.txt")}
    assert facts["elements_per_scale"] == ["32", "16"]
    fp4, s = synth.quantize_mxfp4(synth.normal(0, 41, 8 * 256).reshape(1, 8, 256) * 0.02)
    out_fp4, out_s, glob = Rp.repack_mxfp4_to_nvfp4(fp4, s)
    assert out_s.nbytes == 2 * s.nbytes and out_fp4.nbytes == fp4.nbytes
    assert glob[0] == 1.0                                # N(0,0.02) blocks fit in [-9, 8]


def test_nvfp4_errors():
    e8 = np.full((1, 2, 2), 127, np.uint8)
    e8[0, 1, 1] = 255
    with pytest.raises(Rp.RepackError) as ex:
        Rp.repack_mxfp4_to_nvfp4(np.zeros((1, 2, 32), np.uint8), e8)
    assert ex.value.code == -3
    e8[0, 1, 1] = 127 + 9
    e8[0, 0, 0] = 127 - 9                                 # span 18 > 17
    with pytest.raises(Rp.RepackError) as ex:
        Rp.repack_mxfp4_to_nvfp4(np.zeros((1, 2, 32), np.uint8), e8)
    assert ex.value.code == -4


def test_int4_shape_example():
    (name, n, k, pshape, sshape), = [ln.split() for ln in golden_lines("w4afp8_shapes.txt")]
    n, k = int(n), int(k)
    fp4, s = synth.quantize_mxfp4(synth.normal(0, 51, n * k).reshape(1, n, k) * 0.02)
    q, sinv = Rp.repack_mxfp4_to_int4g128(fp4, s)
    assert "x".join(map(str, q.shape[1:])) == pshape and q.dtype == np.int8
    assert "x".join(map(str, sinv.shape[1:])) == sshape and sinv.dtype == np.float32


def test_int4_error_bound_and_grid_roundtrip():
    fp4, s = synth.quantize_mxfp4(synth.normal(0, 52, 16 * 512).reshape(1, 16, 512) * 0.02)
    q, sinv = Rp.repack_mxfp4_to_int4g128(fp4, s)
    src = ffn.dequant_mxfp4(fp4[0], s[0])
    deq = ffn.dequant_int4g128(q[0], sinv[0])
    bound = np.repeat(sinv[0].astype(np.float64), 128, axis=1) * (0.5 + 1e-6)
    assert (np.abs(deq - src) <= bound).all()
    qq = q.view(np.uint8)
    nib = np.stack([qq & 0xF, qq >> 4], -1).reshape(-1)
    assert not (nib == 8).any()                           # -8 is never used
    # closed form: a group holding only 0 and +-amax maps to q in {0, +-7}
    # with scale_inv = fp32(amax / 7)
    blk = np.zeros((1, 1, 64), np.uint8)
    codes = np.array([0x0, 0x6, 0xE, 0x6] * 32, np.uint8)        # 0, 4, -4, 4
    blk[0, 0] = codes[0::2] | (codes[1::2] << 4)
    q1, s1 = Rp.repack_mxfp4_to_int4g128(blk, np.full((1, 1, 4), 127 + 3, np.uint8))
    assert s1[0, 0, 0] == np.float32(32.0) / np.float32(7.0)
    v = ffn.dequant_int4g128(q1[0], np.ones((1, 1), np.float32))[0]
    assert v.tolist() == [0, 7, -7, 7] * 32


def test_int4_zero_group_and_errors():
    q, s = Rp.repack_mxfp4_to_int4g128(np.zeros((1, 1, 64), np.uint8), np.full((1, 1, 4), 127, np.uint8))
    assert s[0, 0, 0] == 1.0 and (q == 0).all()
    with pytest.raises(Rp.RepackError) as ex:
        Rp.repack_mxfp4_to_int4g128(np.zeros((1, 1, 64), np.uint8), np.full((1, 1, 4), 255, np.uint8))
    assert ex.value.code == -3
    big = np.full((1, 1, 64), 0x77, np.uint8)
    with pytest.raises(Rp.RepackError) as ex:
        Rp.repack_mxfp4_to_int4g128(big, np.full((1, 1, 4), 254, np.uint8))
    assert ex.value.code == -4


# ---------------- MXFP4 -> FP8 E4M3 with a [128, 128] block scale ----------------
def _block(codes_row, exps, N=128, K=128):
    """One [N, K] matrix: every row holds codes_row (K nibble codes), 32-element
    block j of every row has E8M0 byte exps[j]."""
    codes = np.tile(np.asarray(codes_row, np.uint8), (N, 1))
    fp4 = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)[None]
    e8 = np.tile(np.asarray(exps, np.uint8), (N, 1))[None]
    return fp4, e8


def test_fp8_block_cast_lossless_roundtrip():
    """Exponent spread <= 8 inside every [128, 128] block: decoding the codes
    and multiplying by scale_inv gives back the MXFP4 values exactly."""
    M, N, K = 2, 256, 512
    fp4 = synth.random_bytes(7, 1, (M, N, K // 2))
    e8 = synth.random_bytes(7, 2, (M, N, K // 32), 118, 126)
    q, sinv, exact = Rp.repack_mxfp4_to_fp8_block128(fp4, e8)
    assert exact and q.shape == (M, N, K) and sinv.shape == (M, N // 128, K // 128)
    ref = ffn.dequant_mxfp4(fp4, e8)
    back = F.decode_e4m3(q) * np.repeat(np.repeat(sinv.astype(np.float64), 128, 1), 128, 2)
    np.testing.assert_array_equal(back, ref)


def test_fp8_block_cast_closed_forms():
    # block maximum 6 * 2^e -> scale 2^(e-6); 6 -> 384 (0x7C), 0.5 -> 32 (0x60)
    row = [7] + [1] * 127                         # codes 7 (6.0) and 1 (0.5)
    e = 5
    q, sinv, exact = Rp.repack_mxfp4_to_fp8_block128(*_block(row, [127 + e] * 4))
    assert exact and sinv[0, 0, 0] == np.float32(2.0 ** (e - 6))
    assert q[0, 0, 0] == 0x7C and q[0, 0, 1] == 0x60
    # block maximum 1.0 * 2^e -> scale 2^(e-8); 1.0 -> 256 (0x78)
    q, sinv, _ = Rp.repack_mxfp4_to_fp8_block128(*_block([2] * 128, [127 + e] * 4))
    assert sinv[0, 0, 0] == np.float32(2.0 ** (e - 8)) and (q == 0x78).all()
    # all-zero block: scale 1, codes 0; negative zero keeps its sign
    q, sinv, exact = Rp.repack_mxfp4_to_fp8_block128(*_block([0, 8] * 64, [200] * 4))
    assert exact and sinv[0, 0, 0] == 1.0 and (q[..., 0::2] == 0).all() and (q[..., 1::2] == 0x80).all()


def test_fp8_block_scale_is_the_activation_rule():
    """The block exponent is the activation quantiser's exponent of the block
    maximum (oracle.quant, float32 ratio) wherever that maximum is a float32."""
    from oracle import quant as Q
    for code in range(1, 8):
        for e in range(-126, 125, 7):
            q, sinv, _ = Rp.repack_mxfp4_to_fp8_block128(*_block([code] + [0] * 127, [127 + e] * 4))
            amax = np.float32(F.e2m1_value(code) * 2.0 ** e)
            k = int(Q.pow2_scale_exponent(np.array([amax]))[0])
            assert sinv[0, 0, 0] == np.float32(np.ldexp(1.0, k)), (code, e)


def test_fp8_block_cast_lossy_edge_and_errors():
    # spread 14 with the smallest codes: still exact (0.5 * 2^-14 * 2^6 = 2^-9)
    row = [7] * 32 + [1] * 32 + [3] * 32 + [0] * 32
    q, sinv, exact = Rp.repack_mxfp4_to_fp8_block128(*_block(row, [140, 126, 126, 126]))
    assert exact
    # spread 15: 0.5 -> 2^-10 rounds to 0 (tie to even), 1.5 -> 1.5 * 2^-9 rounds to 2^-8
    q, sinv, exact = Rp.repack_mxfp4_to_fp8_block128(*_block(row, [140, 125, 125, 125]))
    assert not exact
    assert (q[0, :, 32:64] == 0x00).all() and (q[0, :, 64:96] == 0x02).all()
    with pytest.raises(Rp.RepackError) as ex:
        Rp.repack_mxfp4_to_fp8_block128(*_block([1] * 128, [127, 255, 127, 127]))
    assert ex.value.code == -3
