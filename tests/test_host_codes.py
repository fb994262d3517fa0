"""Host-side checks of the code tricks the W4AFP8 converter relies on for
token tiles of at most 32 rows (no GPU needed):

* flipping the top bit of a two's-complement INT4 nibble n gives u = n + 8,
  and the byte u (0..15) is the E4M3 code of u * 2^-9 (checked against the
  oracle's E4M3 decoder, itself pinned to the format's tables);
* sum(x * n) = sum(x * u) - 8 * sum(x), the correction the promotion applies;
* the converter's masks and byte-permute selectors put element k of a packed
  word at byte k (a CPU model of the byte permute's selection rule).
"""
import numpy as np

from oracle import formats as F
import synth


def test_offset_bytes_are_scaled_integers():
    u = np.arange(16, dtype=np.uint8)
    assert (F.decode_e4m3(u) == u.astype(np.float64) * 2.0 ** -9).all()
    n = np.arange(-8, 8)
    nib = (n & 0xF).astype(np.uint8)
    assert ((nib ^ 0x8).astype(np.int64) == n + 8).all()


def test_offset_identity_on_random_steps():
    x = F.decode_e4m3(synth.random_e4m3(7, 1, (64, 128)))
    n = (synth.random_bytes(7, 2, (64, 128)).astype(np.int64) & 0xF)
    n = np.where(n >= 8, n - 16, n)
    u = n + 8
    lhs = (x * n).sum(axis=1)
    rhs = (x * u).sum(axis=1) - 8.0 * x.sum(axis=1)
    assert np.array_equal(lhs, rhs)     # every term is a dyadic rational: float64 is exact here


def _byte_perm(a: int, b: int, sel: int) -> int:
    src = (a & 0xFFFFFFFF) | ((b & 0xFFFFFFFF) << 32)
    out = 0
    for i in range(4):
        k = (sel >> (4 * i)) & 0x7
        out |= ((src >> (8 * k)) & 0xFF) << (8 * i)
    return out


def test_converter_interleave_order():
    words = synth.random_bytes(11, 1, (256, 4)).view(np.uint32).ravel()
    for w in words.tolist():
        ev = (w & 0x0F0F0F0F) ^ 0x08080808
        od = ((w >> 4) & 0x0F0F0F0F) ^ 0x08080808
        lo4, hi4 = _byte_perm(ev, od, 0x5140), _byte_perm(ev, od, 0x7362)
        got = [(lo4 >> (8 * i)) & 0xFF for i in range(4)] + [(hi4 >> (8 * i)) & 0xFF for i in range(4)]
        want = [((w >> (4 * k)) & 0xF) ^ 0x8 for k in range(8)]
        assert got == want, hex(w)
