"""End-to-end parity of the MoE layer (a1 -> a7) against the oracle.

Tolerance (the layer's floating-point output): max |gpu - oracle| <=
1e-2 * max |oracle| and mean relative error sum|gpu - oracle| / sum|oracle|
<= 2e-3, the oracle being the float64 result before any bf16 rounding.
Intermediates that are integer decisions on exact data (quantised x, routing
indices, grouping) must match bit for bit.  At full sizes the oracle
evaluates a seeded sample of tokens; token outputs are independent given the
routing, so the sample is exact.  The benchmark's full-size MXFP4 and W4AFP8
layers are checked in test_gpu_full_size.py.
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


def _w4a_ref(x, logits, w13, s13, w2, s2, k, tokens=None, n_proto=None):
    """Oracle W4AFP8 layer: the oracle's INT4 repack of the experts, then its FFN.
    With n_proto set (expert e holds the values of expert e % n_proto) only
    the prototypes the sampled tokens reach are repacked."""
    from oracle import repack as Rp
    from oracle import route as R
    G = w13.shape[0]
    q13 = np.zeros(w13.shape, np.int8)
    i13 = np.ones(w13.shape[:2] + (w13.shape[2] * 2 // 128,), np.float32)
    q2 = np.zeros(w2.shape, np.int8)
    i2 = np.ones(w2.shape[:2] + (w2.shape[2] * 2 // 128,), np.float32)
    lg = logits if tokens is None else logits[tokens]
    used = sorted(set(R.route_topk(lg, k)[0].reshape(-1).tolist()) | {G - 1})
    done = {}
    for e in used:
        p = e if n_proto is None else e % n_proto
        if p not in done:
            done[p] = (Rp.repack_mxfp4_to_int4g128(w13[p:p + 1], s13[p:p + 1]),
                       Rp.repack_mxfp4_to_int4g128(w2[p:p + 1], s2[p:p + 1]))
        (a, b), (c, d) = done[p]
        q13[e], i13[e], q2[e], i2[e] = a[0], b[0], c[0], d[0]
    return ffn.moe_layer(x, logits, None, None, None, None, k, weights="w4afp8", w13_int4=q13, w13_sinv=i13,
                         w2_int4=q2, w2_sinv=i2, tokens=tokens)


@pytest.mark.parametrize("block_n", [0, 16])
def test_tiny_layer_w4afp8(lib, block_n):
    """The W4AFP8 path: experts repacked to INT4 group-128 on the GPU, then the
    INT4 x FP8 GEMMs; compared with the oracle's repack and FFN."""
    wl = synth.tiny_layer(0)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, weights="w4afp8")
    buf = layer.alloc(wl.T, block_n)
    y = layer.forward(torch.from_numpy(wl.x_bf16.view(np.int16)).cuda(), torch.from_numpy(wl.logits).cuda(), buf)
    ref = _w4a_ref(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    check_y(y.float().cpu().numpy(), ref["y"])
    assert lib.moe_get_device_error() == 0


@pytest.mark.parametrize("shared", ["mxfp4", "fp8"])
def test_segment_graphs_match_eager(lib, shared):
    """The forward pass captured as four CUDA graphs (one per segment, as the
    decode benchmark replays it) gives the eager result bit for bit, also
    after new inputs are copied into the captured buffers; with the FP8
    shared expert the capture holds its side-stream GEMMs too."""
    wl = synth.tiny_layer(2)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, shared=shared)
    buf = layer.alloc(wl.T)
    x = torch.from_numpy(wl.x_bf16.view(np.int16)).cuda()
    lg = torch.from_numpy(wl.logits).cuda()
    segs = layer.segments(x, lg, buf)
    for f in segs:
        f()
    torch.cuda.synchronize()
    graphs = []
    for f in segs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            f()
        graphs.append(g)
    wl2 = synth.tiny_layer(3)
    for src_x, src_l in ((wl.x_bf16, wl.logits), (wl2.x_bf16, wl2.logits)):
        x.copy_(torch.from_numpy(src_x.view(np.int16)))
        lg.copy_(torch.from_numpy(src_l))
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
        y_graph = buf.y.clone()
        layer.forward(x, lg, buf)
        torch.cuda.synchronize()
        assert torch.equal(y_graph.view(torch.int16), buf.y.view(torch.int16))
    assert lib.moe_get_device_error() == 0
    del graphs


def _shared_fp8_ref(x, logits, w13, s13, w2, s2, k, tokens=None):
    """Oracle layer with the shared expert (group E) cast to FP8 [128, 128]
    blocks by the oracle's cast."""
    from oracle import repack as Rp
    E = w13.shape[0] - 1
    q13, i13, _ = Rp.repack_mxfp4_to_fp8_block128(w13[E:E + 1], s13[E:E + 1])
    q2, i2, _ = Rp.repack_mxfp4_to_fp8_block128(w2[E:E + 1], s2[E:E + 1])
    return ffn.moe_layer(x, logits, w13, s13, w2, s2, k, tokens=tokens, shared_fp8=(q13[0], i13[0], q2[0], i2[0]))


@pytest.mark.parametrize("weights", ["mxfp4", "w4afp8"])
def test_tiny_layer_shared_fp8(lib, weights):
    """Routed experts in MXFP4 (or W4AFP8), the shared expert as FP8 with
    [128, 128] block scales through moe_grouped_gemm_fp8_block128."""
    wl = synth.tiny_layer(5)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, weights=weights, shared="fp8")
    buf = layer.alloc(wl.T)
    y = layer.forward(torch.from_numpy(wl.x_bf16.view(np.int16)).cuda(), torch.from_numpy(wl.logits).cuda(), buf)
    if weights == "mxfp4":
        ref = _shared_fp8_ref(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    else:
        from oracle import repack as Rp
        E = wl.E
        q13, i13 = Rp.repack_mxfp4_to_int4g128(wl.w13, wl.w13_e8m0)
        q2, i2 = Rp.repack_mxfp4_to_int4g128(wl.w2, wl.w2_e8m0)
        f13, g13, _ = Rp.repack_mxfp4_to_fp8_block128(wl.w13[E:E + 1], wl.w13_e8m0[E:E + 1])
        f2, g2, _ = Rp.repack_mxfp4_to_fp8_block128(wl.w2[E:E + 1], wl.w2_e8m0[E:E + 1])
        ref = ffn.moe_layer(wl.x_bf16, wl.logits, None, None, None, None, wl.topk, weights="w4afp8",
                            w13_int4=q13, w13_sinv=i13, w2_int4=q2, w2_sinv=i2,
                            shared_fp8=(f13[0], g13[0], f2[0], g2[0]))
    check_y(y.float().cpu().numpy(), ref["y"])
    assert lib.moe_get_device_error() == 0


def test_decode_layer_shared_fp8_full_size(lib):
    """Decode configuration (64 tokens, 256 + 1 experts) with the FP8 shared
    expert; sampled tokens against the oracle."""
    T, H, I, E, k = 64, 4096, 2048, 256, 6
    w13, s13, w2, s2 = synth.expert_weights(0, E + 1, H, I, n_proto=4)
    x = synth.decode_activations(0, T, H)
    logits = synth.uniform_logits(0, T, E)
    layer = MoeLayer(w13, s13, w2, s2, k, shared="fp8")
    buf = layer.alloc(T)
    y = layer.forward(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(logits).cuda(), buf)
    toks = np.sort((synth.splitmix64(0, 79, 8) % np.uint64(T)).astype(np.int64))
    ref = _shared_fp8_ref(x, logits, w13, s13, w2, s2, k, tokens=toks)
    check_y(y.float().cpu().numpy()[toks], ref["y"])
    assert lib.moe_get_device_error() == 0


class _ProtoWeights:
    """[G, ...] view whose entry g is prototype g % n_proto of a smaller array
    (the synthetic weights repeat n_proto experts), so the oracle repacks only
    the prototypes."""

    def __init__(self, protos, G):
        self.protos, self.shape = protos, (G,) + protos.shape[1:]

    def __getitem__(self, g):
        return self.protos[g % len(self.protos)]


def _ptpc_ref(x, logits, w13, s13, w2, s2, k, tokens=None, n_proto=None):
    """Oracle PTPC-FP8 layer: the oracle's per-channel cast of the experts,
    then its FFN with per-token activations."""
    G = w13.shape[0]
    n = G if n_proto is None else n_proto
    q13, i13 = ffn.ptpc_weights(w13[:n], s13[:n])
    q2, i2 = ffn.ptpc_weights(w2[:n], s2[:n])
    return ffn.moe_layer_ptpc(x, logits, _ProtoWeights(q13, G), _ProtoWeights(i13, G), _ProtoWeights(q2, G),
                              _ProtoWeights(i2, G), k, tokens=tokens)


@pytest.mark.parametrize("block_n", [0, 16, 128])
def test_tiny_layer_ptpc(lib, block_n):
    """PTPC-FP8: experts cast per channel on the GPU, activations quantised
    per token; the per-token quantisation of x is bit-exact."""
    wl = synth.tiny_layer(6)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, weights="ptpc")
    buf = layer.alloc(wl.T, block_n)
    y = layer.forward(torch.from_numpy(wl.x_bf16.view(np.int16)).cuda(), torch.from_numpy(wl.logits).cuda(), buf)
    ref = _ptpc_ref(wl.x_bf16, wl.logits, wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(buf.xq.cpu().numpy(), ref["xq"])
    np.testing.assert_array_equal(buf.sxf.cpu().numpy().view(np.uint32), ref["sx"].view(np.uint32))
    np.testing.assert_array_equal(buf.idx.cpu().numpy(), ref["idx"])
    check_y(y.float().cpu().numpy(), ref["y"])
    assert lib.moe_get_device_error() == 0


def test_decode_layer_ptpc_full_size(lib):
    """Decode configuration (64 tokens, hidden 4096, intermediate 2048, 256 + 1
    experts, top-6) in PTPC-FP8; sampled tokens against the oracle."""
    T, H, I, E, k = 64, 4096, 2048, 256, 6
    w13, s13, w2, s2 = synth.expert_weights(0, E + 1, H, I, n_proto=2)
    x = synth.decode_activations(0, T, H)
    logits = synth.uniform_logits(0, T, E)
    layer = MoeLayer(w13, s13, w2, s2, k, weights="ptpc")
    buf = layer.alloc(T)
    y = layer.forward(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(logits).cuda(), buf)
    toks = np.sort((synth.splitmix64(0, 80, 8) % np.uint64(T)).astype(np.int64))
    ref = _ptpc_ref(x, logits, w13, s13, w2, s2, k, tokens=toks, n_proto=2)
    check_y(y.float().cpu().numpy()[toks], ref["y"])
    assert lib.moe_get_device_error() == 0


@pytest.mark.parametrize("weights", ["mxfp4", "w4afp8", "ptpc"])
def test_empty_batch(lib, weights):
    """Zero tokens: every call of the step is a no-op that returns MOE_OK (the
    grouping still writes all-zero counts and offsets), y is [0, H]."""
    wl = synth.tiny_layer(7)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk, weights=weights)
    buf = layer.alloc(0)
    x = torch.empty((0, layer.H), dtype=torch.int16, device="cuda")
    lg = torch.empty((0, wl.E), dtype=torch.float32, device="cuda")
    y = layer.forward(x, lg, buf)
    torch.cuda.synchronize()
    assert tuple(y.shape) == (0, layer.H)
    assert (buf.counts.cpu().numpy() == 0).all() and (buf.offsets.cpu().numpy() == 0).all()
    assert lib.moe_get_device_error() == 0


@pytest.mark.parametrize("graphs,input_sets", [(True, 2), (False, 2), (True, 1)])
def test_step_runner_overlapped_copies(lib, graphs, input_sets):
    """StepRunner (host copies overlapped with the neighbouring steps on
    their own streams, into one or two device copies of the inputs) gives,
    step after step with changing inputs, the eager forward's y bit for
    bit."""
    from fp8_block_scaled_pow2_b200.runner import StepRunner, pinned_inputs
    wl = synth.tiny_layer(8)
    layer = MoeLayer(wl.w13, wl.w13_e8m0, wl.w2, wl.w2_e8m0, wl.topk)
    runner = StepRunner(layer, wl.T, graphs=graphs, input_sets=input_sets)
    steps = [synth.tiny_layer(20 + i) for i in range(4)]
    hosts = [pinned_inputs(s.x_bf16, s.logits) for s in steps]
    for xh, lh, yh in hosts:
        runner.submit(xh, lh, yh)
    runner.synchronize()
    ref_buf = layer.alloc(wl.T)
    for s, (xh, lh, yh) in zip(steps, hosts):
        y = layer.forward(torch.from_numpy(s.x_bf16.view(np.int16)).cuda(), torch.from_numpy(s.logits).cuda(),
                          ref_buf)
        torch.cuda.synchronize()
        assert torch.equal(yh.view(torch.int16), y.cpu().view(torch.int16))
    runner.close()
    assert lib.moe_get_device_error() == 0


def test_prefill_layer_ptpc_sampled(lib):
    """Prefill configuration (4096 tokens, Zipf loads, 256 + 1 experts) in
    PTPC-FP8, the launch configuration the benchmark times (128-token tiles
    with gate and up pairs); sampled tokens against the oracle."""
    T, H, I, E, k = 4096, 4096, 2048, 256, 6
    w13, s13, w2, s2 = synth.expert_weights(0, E + 1, H, I, n_proto=2)
    x = synth.decode_activations(0, T, H)
    logits = synth.zipf_logits(0, T, E)
    layer = MoeLayer(w13, s13, w2, s2, k, weights="ptpc")
    buf = layer.alloc(T)
    y = layer.forward(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(logits).cuda(), buf)
    toks = np.sort((synth.splitmix64(0, 81, 6) % np.uint64(T)).astype(np.int64))
    ref = _ptpc_ref(x, logits, w13, s13, w2, s2, k, tokens=toks, n_proto=2)
    check_y(y.float().cpu().numpy()[toks], ref["y"])
    assert lib.moe_get_device_error() == 0
