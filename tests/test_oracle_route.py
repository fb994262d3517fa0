"""Pins of the router oracle (step a2): brute force over all k-subsets on
tiny inputs, closed forms of sqrtsoftplus, the route-scale sum."""
import itertools

import numpy as np

import synth
from oracle import route as R


def _brute_topk(z, k):
    """Largest k logits, ties to the lower index, by enumerating all subsets:
    the chosen subset is the one whose (value desc, index asc) key list is
    lexicographically best."""
    E = len(z)
    best = None
    for sub in itertools.combinations(range(E), k):
        key = sorted(((-float(z[i]), i) for i in sub))
        if best is None or key < best[0]:
            best = (key, [i for _, i in key])
    return best[1]


def test_topk_brute_force_tiny():
    for seed in range(20):
        E = 3 + seed % 6
        k = 1 + seed % min(E, 4)
        z = (synth.uniform(seed, 11, 5 * E) * 4 - 2).astype(np.float32).reshape(5, E)
        z[:, ::2] = np.round(z[:, ::2])                  # plenty of ties
        idx, w = R.route_topk(z, k)
        for t in range(5):
            assert idx[t].tolist() == _brute_topk(z[t], k)


def test_weights_closed_forms():
    z = np.array([[0.0, -50.0, 30.0, 1.0]], np.float32)
    s = R.sqrtsoftplus(z[0])
    assert abs(s[0] - np.sqrt(np.log(2.0))) < 1e-15
    assert abs(s[2] - np.sqrt(30.0)) < 1e-12               # softplus(z) -> z
    assert abs(s[1] - np.sqrt(np.exp(-50.0))) < 1e-30       # softplus(z) -> e^z
    idx, w = R.route_topk(z, 2)
    assert idx.tolist() == [[2, 3]]
    s3 = np.sqrt(np.log1p(np.e))
    np.testing.assert_allclose(w[0], 1.5 * np.array([np.sqrt(30.0), s3]) / (np.sqrt(30.0) + s3), rtol=1e-14)


def test_weights_sum_to_route_scale():
    z = synth.uniform_logits(0, 64, 256)
    idx, w = R.route_topk(z, 6)
    np.testing.assert_allclose(w.sum(1), 1.5, rtol=1e-14)
    assert (np.diff(np.take_along_axis(z, idx, 1), axis=1) <= 0).all()
    _, w0 = R.route_topk(z, 6, route_norm=0)
    np.testing.assert_allclose(w0, 1.5 * R.sqrtsoftplus(np.take_along_axis(z, idx, 1)), rtol=1e-14)


def test_softplus_monotone_so_logit_order_is_score_order():
    z = np.linspace(-40, 40, 20001)
    assert (np.diff(R.sqrtsoftplus(z)) > 0).all()


# ------------------------------ hash routing ------------------------------
def test_hash_route_is_the_table_lookup():
    """idx[t, j] is entry j of the token's table row, checked element by element."""
    V, E, k, T = 50, 16, 4, 40
    table = synth.hash_table(3, V, E, k)
    tok = synth.token_ids(3, T, V)
    z = synth.uniform_logits(3, T, E)
    idx, w = R.route_hash(tok, table, z)
    for t in range(T):
        for j in range(k):
            assert idx[t, j] == table[tok[t], j]
    assert idx.dtype == np.int32


def test_hash_route_weights_closed_forms():
    """Equal logits at the chosen experts give 1.5 / k each; logit 0 scores
    sqrt(ln 2); unnormalised weights are 1.5 * sqrt(softplus(z))."""
    table = np.array([[2, 0, 3], [1, 3, 0]], np.int32)
    z = np.array([[0.0, 9.0, 0.0, 0.0], [0.0, 30.0, -7.0, 0.0]], np.float32)
    idx, w = R.route_hash(np.array([0, 0]), table, z)
    assert idx.tolist() == [[2, 0, 3], [2, 0, 3]]
    np.testing.assert_allclose(w[0], [0.5, 0.5, 0.5], rtol=1e-15)
    _, w0 = R.route_hash(np.array([1]), table, z[1:], route_norm=0)
    np.testing.assert_allclose(w0[0], 1.5 * np.array([np.sqrt(30.0), np.sqrt(np.log(2.0)), np.sqrt(np.log(2.0))]),
                               rtol=1e-12)


def test_hash_route_ignores_unchosen_logits():
    """Only the logits of the looked-up experts enter the weights."""
    V, E, k, T = 30, 12, 3, 20
    table = synth.hash_table(4, V, E, k)
    tok = synth.token_ids(4, T, V)
    z = synth.uniform_logits(4, T, E)
    idx, w = R.route_hash(tok, table, z)
    z2 = z.copy()
    mask = np.ones_like(z2, bool)
    np.put_along_axis(mask, idx.astype(np.int64), False, axis=1)
    z2[mask] = 99.0
    idx2, w2 = R.route_hash(tok, table, z2)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_array_equal(w, w2)
    np.testing.assert_allclose(w.sum(1), 1.5, rtol=1e-14)


def test_hash_route_equals_topk_when_table_holds_the_topk():
    """A table whose row for token t lists that token's k largest logits in
    order gives exactly the top-k router's result (pinned by brute force)."""
    T, E, k = 10, 9, 3
    z = synth.uniform_logits(5, T, E)
    table = np.array([_brute_topk(z[t], k) for t in range(T)], np.int32)
    idx_h, w_h = R.route_hash(np.arange(T), table, z)
    idx_t, w_t = R.route_topk(z, k)
    np.testing.assert_array_equal(idx_h, idx_t)
    np.testing.assert_array_equal(w_h, w_t)
