"""Failure detection on the GPU without faulting it: a bounded device wait on
a barrier that nothing arrives at gives up, reports MOE_ERR_TIMEOUT through
the device error word, and the context keeps working."""
import numpy as np
import pytest
import torch

import synth
from oracle import quant as Q

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(lib):
    assert lib.moe_get_device_error() == 0
    lib.moe_selftest_wait_timeout(10_000_000)            # 10 ms
    assert lib.moe_get_device_error() == -6
    assert lib.moe_get_device_error() == 0               # cleared by the read
    x = synth.decode_activations(1, 8, 256)
    xq = torch.empty((8, 256), dtype=torch.uint8, device="cuda")
    sx = torch.empty((8, 2), dtype=torch.uint8, device="cuda")
    lib.moe_quantize_act_fp8(torch.from_numpy(x.view(np.int16)).cuda(), xq, sx)
    q_ref, s_ref = Q.quantize_act_fp8(x)
    assert (xq.cpu().numpy() == q_ref).all() and (sx.cpu().numpy() == s_ref).all()


def test_invalid_arguments_raise_before_launch(lib):
    with pytest.raises(lib.MoeError) as ex:
        lib.moe_selftest_wait_timeout(0)
    assert ex.value.status == -1
    x = torch.zeros((4, 100), dtype=torch.int16, device="cuda")
    with pytest.raises(lib.MoeError):
        lib.moe_quantize_act_fp8(x, torch.empty((4, 100), dtype=torch.uint8, device="cuda"),
                                 torch.empty((4, 1), dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("T", [4, 600])
def test_out_of_range_expert_id_is_flagged(lib, T):
    """An expert id outside [0, E) is flagged; that pair gets no row, its inv
    entry is -1, and the combine leaves it out.  T = 4 runs the one-block
    grouping, T = 600 (2400 pairs) the chunked passes."""
    E, k, H = 8, 4, 128
    idx_np = (np.arange(T * k, dtype=np.int32) % E).reshape(T, k)
    bad = (1, 3) if T == 4 else (577, 2)
    idx_np[bad] = 9                                                           # 9 >= E
    idx = torch.from_numpy(idx_np).cuda()
    xq = torch.zeros((T, H), dtype=torch.uint8, device="cuda")
    sx = torch.zeros((T, 1), dtype=torch.uint8, device="cuda")
    R = T * k + T
    counts, offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda"), torch.empty(E + 2, dtype=torch.int32,
                                                                                          device="cuda")
    perm, inv = torch.empty(R, dtype=torch.int32, device="cuda"), torch.empty(T * k, dtype=torch.int32, device="cuda")
    xqp, sxp = torch.empty((R, H), dtype=torch.uint8, device="cuda"), torch.empty((R, 1), dtype=torch.uint8, device="cuda")
    ws = torch.empty(lib.moe_permute_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    lib.moe_permute(idx, E, 1, xq, sx, counts, offsets, perm, inv, xqp, sxp, ws)
    torch.cuda.synchronize()
    assert lib.moe_get_device_error() == -1
    p_bad = bad[0] * k + bad[1]
    inv_h = inv.cpu().numpy()
    assert inv_h[p_bad] == -1
    assert int(counts[:E].sum()) == T * k - 1
    good = np.delete(np.arange(T * k), p_bad)
    np.testing.assert_array_equal(np.sort(inv_h[good]), np.arange(T * k - 1))
    # combine over rows o[r] = r: the rejected slot adds nothing
    o = torch.arange(R, dtype=torch.float32, device="cuda")[:, None].repeat(1, H).contiguous()
    w = torch.ones((T, k), dtype=torch.float32, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    lib.moe_combine(o, inv, w, 1, offsets, E, y)
    torch.cuda.synchronize()
    off_h = offsets.cpu().numpy()
    t = bad[0]
    expect = sum(float(inv_h[t * k + j]) for j in range(k) if j != bad[1]) + float(off_h[E] + t)
    assert float(y[t, 0]) == float(torch.tensor(expect).to(torch.bfloat16))
    assert lib.moe_get_device_error() == 0


@pytest.mark.parametrize("bad", ["past_rows", "decreasing", "negative_start"])
def test_invalid_group_offsets_plan_no_work(lib, bad):
    """Offsets that are not nondecreasing from >= 0 up to at most a_rows (device
    data the host cannot check) are caught by the GEMM's plan: it records
    MOE_ERR_INVALID and plans no work, so the output keeps its contents and
    no tile reads or writes outside the operands."""
    G, N, K, R = 3, 256, 256, 40
    offsets = {"past_rows": [0, 10, 20, 41], "decreasing": [0, 30, 10, 40],
               "negative_start": [-5, 10, 20, 40]}[bad]
    a = torch.zeros((R, K), dtype=torch.uint8, device="cuda")
    asc = torch.full((R, K // 128), 127, dtype=torch.uint8, device="cuda")
    w = torch.zeros((G, N, K // 2), dtype=torch.uint8, device="cuda")
    wsc = torch.full((G, N, K // 32), 127, dtype=torch.uint8, device="cuda")
    wp = torch.empty(lib.moe_prepared_weights_size(G, N, K), dtype=torch.uint8, device="cuda")
    lib.moe_prepare_weights(w, wsc, wp)
    ws = torch.empty(lib.moe_gemm_workspace_size(R, G, K, 16), dtype=torch.uint8, device="cuda")
    out = torch.full((R, N), 7.0, dtype=torch.float32, device="cuda")
    off = torch.tensor(offsets, dtype=torch.int32, device="cuda")
    lib.moe_grouped_gemm_mxfp4(a, asc, off, wp, G, N, lib.MOE_EPI_STORE_F32, out, None, ws, 10.0, 16)
    torch.cuda.synchronize()
    assert lib.moe_get_device_error() == -1
    assert (out == 7.0).all()
    off_ok = torch.tensor([0, 10, 20, 40], dtype=torch.int32, device="cuda")
    lib.moe_grouped_gemm_mxfp4(a, asc, off_ok, wp, G, N, lib.MOE_EPI_STORE_F32, out, None, ws, 10.0, 16)
    torch.cuda.synchronize()
    assert lib.moe_get_device_error() == 0
    assert (out == 0.0).all()


@pytest.mark.parametrize("gemm", ["w4afp8", "fp8_block128", "fp8_ptpc"])
@pytest.mark.parametrize("bad", ["past_rows", "decreasing"])
def test_invalid_group_offsets_other_gemms(lib, gemm, bad):
    """The same plan check guards the INT4, FP8-block and PTPC-FP8 GEMMs:
    invalid offsets record MOE_ERR_INVALID and leave the output untouched."""
    G, N, K, R = 3, 256, 256, 40
    offsets = {"past_rows": [0, 10, 20, 41], "decreasing": [0, 30, 10, 40]}[bad]
    a = torch.zeros((R, K), dtype=torch.uint8, device="cuda")
    asc = torch.full((R, K // 128), 127, dtype=torch.uint8, device="cuda")
    ws = torch.empty(lib.moe_gemm_workspace_size(R, G, K, 16), dtype=torch.uint8, device="cuda")
    out = torch.full((R, N), 7.0, dtype=torch.float32, device="cuda")

    def run(off):
        if gemm == "w4afp8":
            q = torch.zeros((G, N, K // 2), dtype=torch.int8, device="cuda")
            s = torch.ones((G, N, K // 128), dtype=torch.float32, device="cuda")
            lib.moe_grouped_gemm_w4afp8(a, asc, off, q, s, lib.MOE_EPI_STORE_F32, out, None, ws, 10.0, 16)
        elif gemm == "fp8_block128":
            q = torch.zeros((G, N, K), dtype=torch.uint8, device="cuda")
            s = torch.ones((G, N // 128, K // 128), dtype=torch.float32, device="cuda")
            lib.moe_grouped_gemm_fp8_block128(a, asc, off, q, s, lib.MOE_EPI_STORE_F32, out, None, ws, 10.0, 16)
        else:
            q = torch.zeros((G, N, K), dtype=torch.uint8, device="cuda")
            s = torch.ones((G, N), dtype=torch.float32, device="cuda")
            sa = torch.ones(R, dtype=torch.float32, device="cuda")
            lib.moe_grouped_gemm_fp8_ptpc(a, sa, off, q, s, lib.MOE_EPI_STORE_F32, out, ws, 10.0, 16)
        torch.cuda.synchronize()

    run(torch.tensor(offsets, dtype=torch.int32, device="cuda"))
    assert lib.moe_get_device_error() == -1
    assert (out == 7.0).all()
    run(torch.tensor([0, 10, 20, 40], dtype=torch.int32, device="cuda"))
    assert lib.moe_get_device_error() == 0
    assert (out == 0.0).all()
