"""Pins of the grouping oracle (step a3): invariants and a pure-Python brute force."""
import numpy as np

import synth
from oracle import permute as Pm


def _brute(idx, E, has_shared):
    T, k = idx.shape
    rows = []
    for g in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == g:
                    rows.append(t * k + j)
    if has_shared:
        rows += [T * k + t for t in range(T)]
    return rows


def test_brute_force_and_invariants():
    for seed in range(12):
        T, E, k = 1 + seed * 3, 2 + seed % 7, 1 + seed % 3
        k = min(k, E)
        idx = (synth.splitmix64(seed, 21, T * k) % np.uint64(E)).astype(np.int32).reshape(T, k)
        for has_shared in (0, 1):
            counts, offsets, perm, inv, src = Pm.permute(idx, E, has_shared)
            assert perm.tolist() == _brute(idx, E, has_shared)
            P = T * k
            assert counts.sum() == P + (T if has_shared else 0)
            assert (offsets[1:] - offsets[:-1] == counts).all() and offsets[0] == 0
            assert (perm[inv] == np.arange(P)).all()
            for g in range(E):
                seg = perm[offsets[g]:offsets[g + 1]]
                assert (np.diff(seg) > 0).all()
                assert (idx.reshape(-1)[seg] == g).all()
            if has_shared:
                assert (src[offsets[E]:] == np.arange(T)).all()


def test_empty():
    counts, offsets, perm, inv, src = Pm.permute(np.zeros((0, 6), np.int32), 8, 1)
    assert counts.sum() == 0 and len(perm) == 0 and len(inv) == 0
