"""The shared input generators: determinism, the published splitmix64 value,
and the MXFP4 synthesis invariant (re-quantising a dequantised block gives
back the same bytes)."""
import numpy as np

import synth
from oracle import ffn


def test_splitmix64_reference_value():
    # first output of splitmix64 from state 0 (Vigna's reference generator)
    assert int(synth.splitmix64(0, 0, 1)[0]) == 0xE220A8397B1DCDAF


def test_streams_independent_and_deterministic():
    a = synth.normal(0, 1, 1000)
    assert (a == synth.normal(0, 1, 1000)).all()
    assert not (a == synth.normal(0, 2, 1000)).all()
    assert abs(a.mean()) < 0.1 and abs(a.std() - 1) < 0.1


def test_mxfp4_synthesis_roundtrip():
    w = synth.normal(0, 5, 64 * 256).reshape(64, 256) * 0.02
    p, s = synth.quantize_mxfp4(w)
    d = ffn.dequant_mxfp4(p, s)
    p2, s2 = synth.quantize_mxfp4(d)
    # the values come back exactly (a block whose maximum rounded down to
    # 3 * 2^e may be re-expressed with the next lower exponent)
    assert (ffn.dequant_mxfp4(p2, s2) == d).all()
    blk = np.abs(d.reshape(64, 8, 32)).max(-1) / 2.0 ** (s.astype(int) - 127)
    assert ((blk >= 3) & (blk <= 6)).all()


def test_zipf_loads_are_skewed():
    z = synth.zipf_logits(0, 4096, 256)
    top = np.argsort(-z, axis=1, kind="stable")[:, :6]
    load = np.bincount(top.reshape(-1), minlength=256)
    assert load[0] > 3000 and load[-1] < 40 and load.sum() == 4096 * 6


def test_hash_table_rows_distinct_and_in_range():
    t = synth.hash_table(0, 2000, 256, 6)
    assert t.shape == (2000, 6) and t.dtype == np.int32
    assert ((t >= 0) & (t < 256)).all()
    assert all(len(set(r)) == 6 for r in t.tolist())
    # every expert is used, roughly uniformly (12000 draws over 256 experts)
    c = np.bincount(t.reshape(-1), minlength=256)
    assert c.min() > 15 and c.max() < 80
    np.testing.assert_array_equal(t, synth.hash_table(0, 2000, 256, 6))
    ids = synth.token_ids(0, 1000, 2000)
    assert ids.dtype == np.int32 and ids.min() >= 0 and ids.max() < 2000


def test_activation_rows_equal_full_batch_rows():
    full = synth.decode_activations(5, 40, 256)
    rows = np.array([0, 17, 39, 17])
    np.testing.assert_array_equal(synth.decode_activations(5, 40, 256, rows=rows), full[rows])


def test_repeated_expert_views_equal_repeated_arrays():
    full = synth.expert_weights(1, 7, 256, 128, n_proto=3)
    views = synth.expert_views(1, 7, 256, 128, n_proto=3)
    for f, v in zip(full, views):
        assert v.shape == f.shape
        np.testing.assert_array_equal(v.materialize(), f)
        np.testing.assert_array_equal(v[5], f[5])
        np.testing.assert_array_equal(v[2:6], f[2:6])
