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
