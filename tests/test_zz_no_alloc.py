"""moe_permute_noalloc: grouping for callers that cannot allocate device memory.

Some callers run from a fixed memory plan that hands the layer only its input
and output buffers, or may not call cudaMalloc where they call the layer, so
they cannot provide the scratch workspace moe_permute asks for.  This entry
point keeps its counters in a fixed device array inside the library instead.
The test calls it through the C ABI twice in a row and checks that each call
reproduces moe_permute's outputs exactly (the grouping is integer work, so
the tolerance the other grouping tests use is equality).  The second call
runs on the array the first call left behind.  The file is named to be
collected last; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import route as R

pytestmark = pytest.mark.gpu


def _buffers(T, E, k, H, has_shared):
    Rn = T * k + (T if has_shared else 0)
    d = "cuda"
    return dict(counts=torch.empty(E + 1, dtype=torch.int32, device=d),
                offsets=torch.empty(E + 2, dtype=torch.int32, device=d),
                perm=torch.empty(max(Rn, 1), dtype=torch.int32, device=d),
                inv=torch.empty(max(T * k, 1), dtype=torch.int32, device=d),
                xq_perm=torch.empty((Rn, H), dtype=torch.uint8, device=d),
                sx_perm=torch.empty((Rn, H // 128), dtype=torch.uint8, device=d))


@pytest.mark.parametrize("T,E,k,has_shared", [(700, 257, 6, 1), (4096, 256, 6, 1), (37, 8, 2, 0)])
def test_noalloc_matches_workspace_version_twice(lib, T, E, k, has_shared):
    H = 512
    # two different inputs, so the second call cannot pass on stale counters
    cases = []
    for seed in (11, 12):
        idx, _ = R.route_topk(synth.zipf_logits(seed, T, E), k)
        xq = torch.from_numpy(synth.random_bytes(seed, 1, (T, H))).cuda()
        sx = torch.from_numpy(synth.random_bytes(seed, 2, (T, H // 128))).cuda()
        cases.append((torch.from_numpy(idx.astype(np.int32)).cuda(), xq, sx))

    for idx, xq, sx in cases:
        ref = _buffers(T, E, k, H, has_shared)
        ws = torch.empty(lib.moe_permute_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
        lib.moe_permute(idx, E, has_shared, xq, sx, ref["counts"], ref["offsets"], ref["perm"], ref["inv"],
                        ref["xq_perm"], ref["sx_perm"], ws)
        got = _buffers(T, E, k, H, has_shared)
        lib.moe_permute_noalloc(idx, E, has_shared, xq, sx, got["counts"], got["offsets"], got["perm"],
                                got["inv"], got["xq_perm"], got["sx_perm"])
        torch.cuda.synchronize()
        for name in ref:
            assert torch.equal(ref[name], got[name]), name
    assert lib.moe_get_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_array(lib):
    E, k = 1000, 8
    cap = lib.moe_permute_noalloc_max_counters()
    T = (cap // E + 1) * 2048 // k                          # one chunk more than the array holds
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    xq = torch.zeros((T, 128), dtype=torch.uint8, device="cuda")
    sx = torch.zeros((T, 1), dtype=torch.uint8, device="cuda")
    b = _buffers(T, E, k, 128, 1)
    with pytest.raises(lib.MoeError) as ex:
        lib.moe_permute_noalloc(idx, E, 1, xq, sx, b["counts"], b["offsets"], b["perm"], b["inv"],
                                b["xq_perm"], b["sx_perm"])
    assert ex.value.status == -2
