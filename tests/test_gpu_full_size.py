"""Layer parity at the benchmark's full sizes, in the launch configuration
bench.py times (block_n chosen by the library, CUDA graphs not needed for
parity): the decode layer (64 tokens, 256 + 1 experts, all tokens checked),
the prefill layer (4096 tokens, Zipf loads) and the long-prefill layer
(16384 tokens, 384 + 1 experts) on the MXFP4 and W4AFP8 paths, and the
weight-repack sweep shapes.

At the prefill sizes the oracle evaluates: routing and grouping of every
token (bit-exact); y of 256 seeded random tokens plus every token of the two
coldest experts that received rows (their ragged tiles); and, for the two
hottest experts, the w2 output o of every row of their group (each row is
the expert's FFN of its source token, so the rows are independent).
Tolerances are the layer's: max |gpu - oracle| <= 1e-2 * max |oracle| and
sum |gpu - oracle| / sum |oracle| <= 2e-3 over each compared set.  Expert e
holds prototype e % 4 (synthetic weights), so the oracle dequantises each
prototype once (ffn's cache argument)."""
import numpy as np
import pytest
import torch

import synth
from fp8_block_scaled_pow2_b200.layer import MoeLayer
from oracle import ffn
from oracle import permute as Pm
from oracle import quant as Q
from oracle import repack as Rp
from oracle import route as R

pytestmark = pytest.mark.gpu

MAX_TOL, MEAN_TOL = 1e-2, 2e-3
H, I, K_TOP = 4096, 2048, 6


def check(got, ref):
    err = np.abs(np.asarray(got, np.float64) - ref)
    assert err.max() <= MAX_TOL * np.abs(ref).max(), (err.max(), np.abs(ref).max())
    assert err.sum() / np.abs(ref).sum() <= MEAN_TOL, err.sum() / np.abs(ref).sum()


def on_device(view):
    protos = torch.from_numpy(np.ascontiguousarray(view.protos)).cuda()
    return protos[torch.arange(view.shape[0], device="cuda") % protos.shape[0]].contiguous()


def int4_views(views):
    """The oracle's INT4 group-128 repack of each prototype, as views."""
    E1 = views[0].shape[0]
    q13, i13 = Rp.repack_mxfp4_to_int4g128(views[0].protos, views[1].protos)
    q2, i2 = Rp.repack_mxfp4_to_int4g128(views[2].protos, views[3].protos)
    return tuple(synth.RepeatedExperts(p, E1) for p in (q13, i13, q2, i2))


def run_full(T, E, logits_fn, weights="mxfp4", seed=0):
    views = synth.expert_views(seed, E + 1, H, I, n_proto=4)
    x = synth.decode_activations(seed, T, H)
    logits = logits_fn(seed, T, E)
    layer = MoeLayer(*(on_device(v) for v in views), K_TOP, weights=weights)
    torch.cuda.empty_cache()
    buf = layer.alloc(T)
    y = layer.forward(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(logits).cuda(), buf)
    torch.cuda.synchronize()
    return views, x, logits, layer, buf, y.float().cpu().numpy()


def oracle_kwargs(views, weights, wq):
    if weights == "mxfp4":
        return dict(w13=views[0], w13_e8m0=views[1], w2=views[2], w2_e8m0=views[3])
    return dict(w13=None, w13_e8m0=None, w2=None, w2_e8m0=None, weights="w4afp8", w13_int4=wq[0],
                w13_sinv=wq[1], w2_int4=wq[2], w2_sinv=wq[3])


def expert_rows_ref(x_rows, e, views, weights, wq, cache):
    """o = FFN_e(x) for the given token rows (the w2 output of those rows)."""
    xq, sx = Q.quantize_act_fp8(x_rows)
    off = np.array([0, len(x_rows)])
    if weights == "mxfp4":
        gu = ffn.grouped_gemm_mxfp4(xq, sx, off, views[0][e][None], views[1][e][None], cache)
        hq, sh = ffn.swiglu_quant(gu, I)
        return ffn.grouped_gemm_mxfp4(hq, sh, off, views[2][e][None], views[3][e][None], cache)
    gu = ffn.grouped_gemm_w4afp8(xq, sx, off, wq[0][e][None], wq[1][e][None], cache)
    hq, sh = ffn.swiglu_quant(gu, I)
    return ffn.grouped_gemm_w4afp8(hq, sh, off, wq[2][e][None], wq[3][e][None], cache)


def sampled_parity(T, E, logits_fn, weights, n_random=256, seed=0):
    views, x, logits, layer, buf, y = run_full(T, E, logits_fn, weights, seed)
    wq = int4_views(views) if weights == "w4afp8" else None
    # routing and grouping of every token, bit-exact
    idx_ref, _ = R.route_topk(logits, K_TOP)
    idx = buf.idx.cpu().numpy()
    np.testing.assert_array_equal(idx, idx_ref)
    counts, offsets, perm, inv, _ = Pm.permute(idx_ref, E, 1)
    np.testing.assert_array_equal(buf.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(buf.perm.cpu().numpy(), perm)
    np.testing.assert_array_equal(buf.inv.cpu().numpy(), inv)
    routed = counts[:E]
    active = np.flatnonzero(routed)
    by_load = active[np.argsort(routed[active], kind="stable")]
    cold, hot = by_load[:2], by_load[-2:]
    # y of random tokens plus every token of the coldest experts
    rnd = (synth.splitmix64(seed, 90, n_random) % np.uint64(T)).astype(np.int64)
    cold_toks = np.flatnonzero(np.isin(idx_ref, cold).any(axis=1))
    toks = np.unique(np.concatenate([rnd, cold_toks]))
    cache = {}
    ref = ffn.moe_layer(x, logits, topk=K_TOP, tokens=toks, cache=cache, **oracle_kwargs(views, weights, wq))
    check(y[toks], ref["y"])
    # every row of the hottest experts' groups, at the w2 output
    for e in hot:
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        src = perm[r0:r1] // K_TOP
        o = buf.o[r0:r1].cpu().numpy()
        check(o, expert_rows_ref(x[src], int(e), views, weights, wq, cache))
    assert layer and int(routed[hot[-1]]) > 0
    from fp8_block_scaled_pow2_b200 import moe
    assert moe.moe_get_device_error() == 0
    return routed[cold], routed[hot]


def test_decode_layer_full_size_all_tokens(lib):
    """Hidden 4096, intermediate 2048, 256 routed + 1 shared, top-6, 64 tokens
    (uniform logits): every token against the oracle."""
    T, E = 64, 256
    views, x, logits, layer, buf, y = run_full(T, E, synth.uniform_logits)
    ref = ffn.moe_layer(x, logits, *views, K_TOP, cache={})
    np.testing.assert_array_equal(buf.idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(buf.xq.cpu().numpy(), ref["xq"])
    check(y, ref["y"])
    assert lib.moe_get_device_error() == 0


def test_prefill_layer_full_size(lib):
    """4096 tokens, Zipf(1.1) loads over 256 + 1 experts, MXFP4."""
    cold, hot = sampled_parity(4096, 256, synth.zipf_logits, "mxfp4")
    assert cold.max() < 64 and hot.min() > 1000


def test_long_prefill_layer_full_size_mxfp4(lib):
    """16384 tokens, Zipf(1.1) loads over 384 + 1 experts, MXFP4."""
    cold, hot = sampled_parity(16384, 384, synth.zipf_logits, "mxfp4")
    assert cold.max() < 128 and hot.min() > 4000


def test_long_prefill_layer_full_size_w4afp8(lib):
    """16384 tokens, 384 + 1 experts, the W4AFP8 path (experts repacked to
    INT4 group 128 on the GPU; the oracle repacks its prototypes)."""
    sampled_parity(16384, 384, synth.zipf_logits, "w4afp8", n_random=64)


def test_repack_sweep_full_shapes(lib):
    """The repack sweep's shapes: 256 experts of w1, w3 [2048, 4096] and w2
    [4096, 2048] through the three repacks in one launch per matrix set, as
    bench.py runs them.  Every expert's outputs equal those of its prototype
    (e % 4, compared on the device, the last expert included), and the four
    prototypes' outputs equal the oracle's repacks bit for bit."""
    E = 256
    views = synth.expert_views(0, E, H, I, n_proto=4)
    w13, s13, w2, s2 = (on_device(v) for v in views)
    sets = [(w13.reshape(2 * E, I, H // 2), s13.reshape(2 * E, I, H // 32), views[0].protos.reshape(8, I, H // 2),
             views[1].protos.reshape(8, I, H // 32)),
            (w2, s2, views[2].protos, views[3].protos)]
    for fp4, e8, p4, p8 in sets:
        M, N, k2 = fp4.shape
        K = 2 * k2
        per = M // E                                  # matrices per expert (2 for w13, 1 for w2)
        nv = (torch.empty_like(fp4), torch.empty((M, N, K // 16), dtype=torch.uint8, device="cuda"),
              torch.empty(M, dtype=torch.float32, device="cuda"))
        i4 = (torch.empty((M, N, k2), dtype=torch.int8, device="cuda"),
              torch.empty((M, N, K // 128), dtype=torch.float32, device="cuda"))
        f8 = (torch.empty((M, N, K), dtype=torch.uint8, device="cuda"),
              torch.empty((M, N // 128, K // 128), dtype=torch.float32, device="cuda"))
        lib.repack_mxfp4_to_nvfp4(fp4, e8, *nv)
        lib.repack_mxfp4_to_int4g128(fp4, e8, *i4)
        lib.repack_mxfp4_to_fp8_block128(fp4, e8, *f8)
        torch.cuda.synchronize()
        assert lib.moe_get_device_error() == 0
        outs = nv + i4 + f8
        # every expert equals its prototype, on the device
        for t in outs:
            v = t.view(E // 4, 4 * per, -1)
            assert bool((v == v[:1]).all())
        # the prototypes against the oracle
        ref_nv = Rp.repack_mxfp4_to_nvfp4(p4, p8)
        ref_i4 = Rp.repack_mxfp4_to_int4g128(p4, p8)
        ref_f8 = Rp.repack_mxfp4_to_fp8_block128(p4, p8)
        last = slice(M - 4 * per, M)                  # the last 4 experts (prototypes 0..3)
        np.testing.assert_array_equal(nv[0][last].cpu().numpy(), p4)
        np.testing.assert_array_equal(nv[1][last].cpu().numpy(), ref_nv[1])
        np.testing.assert_array_equal(nv[2][last].cpu().numpy(), ref_nv[2])
        np.testing.assert_array_equal(i4[0][last].cpu().numpy(), ref_i4[0])
        np.testing.assert_array_equal(i4[1][last].cpu().numpy().view(np.uint32), ref_i4[1].view(np.uint32))
        assert ref_f8[2]
        np.testing.assert_array_equal(f8[0][last].cpu().numpy(), ref_f8[0])
        np.testing.assert_array_equal(f8[1][last].cpu().numpy().view(np.uint32),
                                      np.asarray(ref_f8[1], np.float32).view(np.uint32))
