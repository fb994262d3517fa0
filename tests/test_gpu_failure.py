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


def test_out_of_range_expert_id_is_flagged(lib):
    T, E, k, H = 4, 8, 2, 128
    idx = torch.tensor([[0, 1], [2, 9], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")   # 9 >= E
    xq = torch.zeros((T, H), dtype=torch.uint8, device="cuda")
    sx = torch.zeros((T, 1), dtype=torch.uint8, device="cuda")
    R = T * k + T
    out = [torch.empty(E + 1, dtype=torch.int32, device="cuda"), torch.empty(E + 2, dtype=torch.int32, device="cuda"),
           torch.empty(R, dtype=torch.int32, device="cuda"), torch.empty(T * k, dtype=torch.int32, device="cuda"),
           torch.empty((R, H), dtype=torch.uint8, device="cuda"), torch.empty((R, 1), dtype=torch.uint8, device="cuda")]
    ws = torch.empty(lib.moe_permute_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    lib.moe_permute(idx, E, 1, xq, sx, *out, ws)
    assert lib.moe_get_device_error() == -1


@pytest.mark.parametrize("bad", ["past_rows", "decreasing", "nonzero_start"])
def test_invalid_group_offsets_plan_no_work(lib, bad):
    """Offsets that are not nondecreasing from 0 up to at most a_rows (device
    data the host cannot check) are caught by the GEMM's plan: it records
    MOE_ERR_INVALID and plans no work, so the output keeps its contents and
    no tile reads or writes outside the operands."""
    G, N, K, R = 3, 256, 256, 40
    offsets = {"past_rows": [0, 10, 20, 41], "decreasing": [0, 30, 10, 40],
               "nonzero_start": [5, 10, 20, 40]}[bad]
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
