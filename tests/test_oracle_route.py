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
