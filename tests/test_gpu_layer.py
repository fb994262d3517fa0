"""End-to-end parity of the MoE layer (a1 -> a7) against the oracle.

Tolerance (the layer's floating-point output): max |gpu - oracle| <=
1e-2 * max |oracle| and mean relative error sum|gpu - oracle| / sum|oracle|
<= 2e-3, the oracle being the float64 result before any bf16 rounding.
Intermediates that are integer decisions on exact data (quantised x, routing
indices, grouping) must match bit for bit.  At full sizes the oracle
evaluates a seeded sample of tokens; token outputs are independent given the
routing, so the sample is exact.
"""
import numpy as np
import pytest
import torch

import synth
from fp8_block_scaled_pow2_b200.layer import MoeLayer
from oracle import ffn

pytestmark = pytest.mark.gpu

MAX_TOL, MEAN_TOL = 1e-2, 2e-3


def check_y(y_gpu, y_ref):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    assert err.max() <= MAX_TOL * np.abs(y_ref).max(), (err.max(), np.abs(y_ref).max())
    assert err.sum() / np.abs(y_ref).sum() <= MEAN_TOL, err.sum() / np.abs(y_ref).sum()


def run_layer(x, logits, w13, s13, w2, s2, topk, block_n=0):
    layer = MoeLayer(w13, s13, w2, s2, topk)
    buf = layer.alloc(x.shape[0], block_n)
    y = layer.forward(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(logits).cuda(), buf)
    torch.cuda.synchronize()
    return layer, buf, y.float().cpu().numpy()


@pytest.mark.parametrize("block_n", [0, 16, 128])
def test_tiny_layer(lib, block_n):
    wl = synth.tiny_layer(0)
    layer, buf, y = run_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, block_n)
    ref = ffn.moe_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    np.testing.assert_array_equal(buf.xq.cpu().numpy(), ref["xq"])
    np.testing.assert_array_equal(buf.idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(buf.perm.cpu().numpy(), ref["perm"])
    check_y(y, ref["y"])
    assert lib.moe_get_device_error() == 0


def test_layer_deterministic(lib):
    wl = synth.tiny_layer(1)
    _, _, y1 = run_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    _, _, y2 = run_layer(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    np.testing.assert_array_equal(y1, y2)


def _full_size(T, logits_fn, E=256, n_proto=4, sample=12, seed=0):
    H, I, k = 4096, 2048, 6
    w13, s13, w2, s2 = synth.expert_weights(seed, E + 1, H, I, n_proto=n_proto)
    x = synth.decode_activations(seed, T, H)
    logits = logits_fn(seed, T, E)
    layer, buf, y = run_layer(x, logits, w13, s13, w2, s2, k)
    toks = np.sort((synth.splitmix64(seed, 77, sample) % np.uint64(T)).astype(np.int64))
    ref = ffn.moe_layer(x, logits, w13, s13, w2, s2, k, tokens=toks)
    np.testing.assert_array_equal(buf.idx.cpu().numpy()[toks], ref["idx"])
    check_y(y[toks], ref["y"])


def test_decode_layer_full_size(lib):
    """Hidden 4096, intermediate 2048, 256 routed + 1 shared, top-6, 64 tokens."""
    _full_size(64, synth.uniform_logits)


def test_prefill_layer_full_size(lib):
    """Same shapes, 4096 tokens with Zipf(1.1) expert loads."""
    _full_size(4096, synth.zipf_logits, sample=8)
