"""Pins of the oracle's number formats against the pages' fixed points and the
format definitions (see tests/golden/*.txt for the cited sources)."""
import numpy as np

from oracle import formats as F
from tests.conftest import golden_lines


def test_e2m1_table_matches_value_set():
    for ln in golden_lines("e2m1_values.txt"):
        code, val = ln.split()
        v = F.E2M1_TABLE[int(code)]
        assert v == float(val) and np.signbit(v) == np.signbit(float(val)), (code, v, val)
    mags = sorted(set(abs(v) for v in F.E2M1_TABLE))
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_packed_low_nibble_first():
    # byte 0x72: low nibble 2 (1.0) is element 0, high nibble 7 (6.0) is element 1
    out = F.decode_e2m1_packed(np.array([[0x72, 0xF0]], np.uint8))
    assert out.tolist() == [[1.0, 6.0, 0.0, -6.0]]


def test_e8m0_exhaustive_closed_form():
    b = np.arange(256)
    v = F.decode_e8m0(b)
    assert np.isnan(v[255])
    for i in range(255):
        assert v[i] == 2.0 ** (i - 127)


def test_e4m3_table_properties():
    t = F.E4M3_TABLE
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    pos = t[:0x7F]
    assert (np.diff(pos) > 0).all()                     # monotone codes
    assert (t[0x80:0xFF] == -pos).all()
    # every finite value has at most 4 significant bits
    for v in pos[1:]:
        m, e = np.frexp(v)
        assert (m * 16) == int(m * 16)


def test_e4m3_encode_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    back = F.encode_e4m3_rne_sat(F.decode_e4m3(codes))
    assert (back == codes).all()


def test_e4m3_hand_cases():
    for ln in golden_lines("e4m3_cases.txt"):
        val, code = ln.split()[:2]
        got = F.encode_e4m3_rne_sat(np.array([float(val)]))[0]
        assert got == int(code, 16), (val, hex(got), code)


def test_e4m3_encode_is_nearest_brute_force():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(2000) * 10 ** rng.uniform(-4, 3, 2000)])
    q = F.encode_e4m3_rne_sat(v)
    finite = F.E4M3_TABLE[np.isfinite(F.E4M3_TABLE)]
    for x, c in zip(v, q):
        d = np.abs(finite - min(abs(x), 448.0) * np.sign(x))
        assert abs(F.E4M3_TABLE[c] - np.clip(x, -448, 448)) <= d.min() + 0.0


def test_bf16_decode():
    assert F.decode_bf16_bits(np.array([0x3F80, 0xC000, 0x0001], np.uint16)).tolist() == \
        [1.0, -2.0, np.float32(2.0 ** -133)]
