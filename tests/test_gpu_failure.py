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
