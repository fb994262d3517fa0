"""Hash routing (row f2) on the GPU against the oracle, through the C ABI:
indices bit-exact (a table lookup), weights within 1e-6 relative (the
device's expf / log1pf / sqrtf against float64), the error path for
out-of-range ids, and a whole hash-routed layer."""
import numpy as np
import pytest
import torch

import synth
from fp8_block_scaled_pow2_b200.layer import MoeLayer
from oracle import ffn
from oracle import route as R

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


@pytest.mark.parametrize("T,V,E,k", [(1, 10, 8, 2), (1000, 5000, 256, 6), (333, 129, 385, 6),
                                     (70, 40, 1024, 16), (4096, 100000, 256, 6)])
def test_route_hash(lib, T, V, E, k):
    table = synth.hash_table(T + V, V, E, k)
    tok = synth.token_ids(T + V, T, V)
    z = (synth.uniform(T + E, 4, T * E) * 60 - 30).astype(np.float32).reshape(T, E)   # softplus branches
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    for norm in (1, 0):
        lib.moe_route_hash(dev(tok), dev(table), dev(z), idx, w, 1.5, norm)
        i_ref, w_ref = R.route_hash(tok, table, z, 1.5, norm)
        np.testing.assert_array_equal(host(idx), i_ref)
        np.testing.assert_allclose(host(w), w_ref, rtol=1e-6, atol=0)
    assert lib.moe_get_device_error() == 0


def test_route_hash_rejects_out_of_range_ids(lib):
    """A token id past the vocabulary blanks its row; a table entry past E
    blanks its slot; both record MOE_ERR_INVALID; other tokens are unaffected."""
    V, E, k = 8, 16, 3
    table = synth.hash_table(1, V, E, k)
    table[5, 1] = E                                   # bad entry in row 5
    tok = np.array([0, 9, 5, 3, -1], np.int32)        # 9 and -1 are outside [0, V)
    z = synth.uniform_logits(1, 5, E)
    idx = torch.empty((5, k), dtype=torch.int32, device="cuda")
    w = torch.empty((5, k), dtype=torch.float32, device="cuda")
    lib.moe_route_hash(dev(tok), dev(table), dev(z), idx, w)
    assert lib.moe_get_device_error() == -1          # MOE_ERR_INVALID
    i, ww = host(idx), host(w)
    assert (i[1] == -1).all() and (ww[1] == 0).all() and (i[4] == -1).all() and (ww[4] == 0).all()
    assert i[2].tolist() == [table[5, 0], -1, table[5, 2]] and ww[2, 1] == 0
    s = R.sqrtsoftplus(z[2, [table[5, 0], table[5, 2]]])
    np.testing.assert_allclose(ww[2, [0, 2]], 1.5 * s / s.sum(), rtol=1e-6)
    for t, v in ((0, 0), (3, 3)):
        i_ref, w_ref = R.route_hash(np.array([0]), table[[v]], z[[t]])
        assert i[t].tolist() == i_ref[0].tolist()
        np.testing.assert_allclose(ww[t], w_ref[0], rtol=1e-6)
    assert lib.moe_get_device_error() == 0            # the word was cleared by the read


def test_hash_routed_layer(lib):
    """The tiny layer hash-routed through a synthetic token-id table, against
    the oracle's hash-routed layer."""
    wl = synth.tiny_layer(3)
    V = 64
    table = synth.hash_table(3, V, wl.E, wl.topk)
    tok = synth.token_ids(3, wl.T, V)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, tid2eid=table)
    buf = layer.alloc(wl.T)
    y = layer.forward(dev(wl.x_bf16.view(np.int16)), dev(wl.logits), buf, token_ids=dev(tok))
    ref = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk,
                        token_ids=tok, tid2eid=table)
    np.testing.assert_array_equal(host(buf.idx), ref["idx"])
    np.testing.assert_array_equal(host(buf.perm), ref["perm"])
    got = host(y.float()).astype(np.float64)
    err = np.abs(got - ref["y"])
    assert err.max() <= 1e-2 * np.abs(ref["y"]).max()
    assert err.sum() / np.abs(ref["y"]).sum() <= 2e-3
    assert lib.moe_get_device_error() == 0
