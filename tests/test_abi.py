"""The C ABI library loads on a machine without a GPU and exports every entry
point include/moe_fp8_pow2.h declares (no compute calls here)."""
import ctypes
import os
import re

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe_fp8_pow2.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ["moe_quantize_act_fp8", "moe_route_topk", "moe_permute", "moe_grouped_gemm_mxfp4",
              "moe_swiglu_clamp", "moe_combine", "repack_mxfp4_to_nvfp4", "repack_mxfp4_to_int4g128"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    from fp8_block_scaled_pow2_b200 import build
    build.build()
    lib = ctypes.CDLL(build.LIB)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_signatures_cover_header():
    from fp8_block_scaled_pow2_b200 import _lib
    assert set(declared_functions()) <= set(_lib.SIGNATURES)


def test_status_strings_without_gpu():
    from fp8_block_scaled_pow2_b200 import _lib
    lib = _lib.load()
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(-6).startswith(b"bounded")
    assert lib.moe_version() >= 200


def test_argument_validation_without_gpu():
    """Invalid shapes are rejected on the host before any CUDA call."""
    from fp8_block_scaled_pow2_b200 import _lib
    lib = _lib.load()
    assert lib.moe_quantize_act_fp8(None, 4, 100, None, None, None) == -1      # cols % 128
    assert lib.moe_quantize_act_fp8(None, 0, 128, None, None, None) == 0       # empty: no-op
    assert lib.moe_route_topk(None, 4, 8, 9, ctypes.c_float(1.5), 1, None, None, None) == -1
    # hash routing: k > 16, an empty vocabulary and null pointers are rejected; T = 0 is a no-op
    assert lib.moe_route_hash(None, 4, None, 100, None, 256, 17, ctypes.c_float(1.5), 1, None, None, None) == -1
    assert lib.moe_route_hash(None, 4, None, 0, None, 256, 6, ctypes.c_float(1.5), 1, None, None, None) == -1
    assert lib.moe_route_hash(None, 4, None, 100, None, 256, 6, ctypes.c_float(1.5), 1, None, None, None) == -1
    assert lib.moe_route_hash(None, 0, None, 100, None, 256, 6, ctypes.c_float(1.5), 1, None, None, None) == 0
    assert lib.moe_grouped_gemm_mxfp4(None, None, 4, None, 2, None, 256, 100, 0,
                                      ctypes.c_float(10), 0, None, None, None, 0, None) == -1
    assert lib.moe_grouped_gemm_mxfp4(None, None, 4, None, 2, None, 256, 128, 0,
                                      ctypes.c_float(10), 48, None, None, None, 0, None) == -2
    # the SM-pair kernel (block_n 256) needs N % 256 == 0
    assert lib.moe_grouped_gemm_mxfp4(None, None, 4, None, 2, None, 384, 128, 0,
                                      ctypes.c_float(10), 256, None, None, None, 0, None) == -2
    assert lib.moe_prepared_weights_size(3, 256, 512) == 3 * 2 * 4 * 8704
    assert lib.repack_mxfp4_to_int4g128(None, None, 1, 8, 96, None, None, None) == -1
    assert lib.repack_mxfp4_to_fp8_block128(None, None, 1, 100, 128, None, None, None) == -1   # N % 128
    # PTPC-FP8 entry points
    assert lib.moe_quantize_fp8_per_token(None, 0, 4, 100, None, None, None) == -1     # cols % 8
    assert lib.moe_quantize_fp8_per_token(None, 1, 0, 128, None, None, None) == 0      # empty: no-op
    assert lib.repack_mxfp4_to_fp8_per_channel(None, None, 1, 8, 48, None, None, None) == -1   # K % 32
    assert lib.moe_gather_row_scales(None, 0, 6, None, 8, None, None, None) == 0       # no rows
    assert lib.moe_grouped_gemm_fp8_ptpc(None, None, 4, None, 2, None, None, 256, 128, 2,
                                         ctypes.c_float(10), 16, None, None, 0, None) == -1   # pow2 epilogue
    assert lib.moe_grouped_gemm_fp8_ptpc(None, None, 4, None, 2, None, None, 384, 128, 3,
                                         ctypes.c_float(10), 16, None, None, 0, None) == -1   # N % 256
    assert lib.moe_grouped_gemm_fp8_ptpc(None, None, 4, None, 2, None, None, 256, 128, 3,
                                         ctypes.c_float(10), 48, None, None, 0, None) == -2   # block_n 48
    assert lib.moe_grouped_gemm_fp8_ptpc(None, None, 4, None, 2, None, None, 256, 128, 3,
                                         ctypes.c_float(10), 128, None, None, 0, None) == -1  # null pointers
    # the block-scaled GEMMs take no float32 SwiGLU epilogue
    assert lib.moe_grouped_gemm_fp8_block128(None, None, 4, None, 2, None, None, 256, 128, 3,
                                             ctypes.c_float(10), 16, None, None, None, 0, None) == -1


def test_layer_workspace_size_without_gpu():
    """moe_workspace_size covers moe_permute and every grouped GEMM of the
    step, for every token tile, and rejects invalid configurations."""
    from fp8_block_scaled_pow2_b200 import moe
    lib = moe._lib()
    T, H, I, E, k = 4096, 4096, 2048, 256, 6
    ws = moe.moe_workspace_size(T, H, I, E, k)
    R, G = T * k + T, E + 1
    need = [lib.moe_permute_workspace_size(T, E, k)]
    need += [lib.moe_gemm_workspace_size(R, G, K, bn) for K in (H, I) for bn in (0, 16, 32, 64, 128, 256)]
    assert ws >= max(need) and ws % 256 == 0
    assert moe.moe_workspace_size(T, H, I, E, k, path=moe.MOE_PATH_PTPC) == ws
    assert moe.moe_workspace_size(T, 100, I, E, k) == 0            # H % 128
    assert moe.moe_workspace_size(T, H, I, E, 7, path=3) == 0      # unknown path
    assert moe.moe_workspace_size(T, H, I, 4, 6) == 0              # topk > E
    assert moe.moe_workspace_size(0, H, I, E, k) > 0               # empty batch still valid


def test_split_gemm_workspace_without_gpu():
    """With block_n = 0 a prefill-sized call (128-row tiles) may split its
    groups between the swap-AB and the SM-pair kernel: its workspace holds
    both plans; decode-sized calls keep one plan."""
    from fp8_block_scaled_pow2_b200 import moe
    R, G, K = 28672, 257, 4096
    w128, w256 = moe.moe_gemm_workspace_size(R, G, K, 128), moe.moe_gemm_workspace_size(R, G, K, 256)
    assert w256 > 0 and moe.moe_gemm_workspace_size(R, G, K, 0) == (w128 + 255) // 256 * 256 + w256
    assert moe.moe_gemm_workspace_size(384, 257, K, 0) == moe.moe_gemm_workspace_size(384, 257, K, 16)


def test_w4afp8_workspace_sizes_without_gpu():
    """The E4M3 weight copy is G * N * K bytes on top of the plan for token
    tiles of 64 rows or more, nothing for narrower ones; the layer's W4AFP8
    workspace covers the copy of w1/w3 [2I, H] and of w2 [H, I]."""
    from fp8_block_scaled_pow2_b200 import moe
    plan = moe.moe_gemm_workspace_size(1000, 9, 4096, 64)
    assert moe.moe_w4afp8_workspace_size(1000, 9, 4096, 4096, 64) == plan + 9 * 4096 * 4096
    assert moe.moe_w4afp8_workspace_size(1000, 9, 4096, 4096, 32) == moe.moe_gemm_workspace_size(1000, 9, 4096, 32)
    # block_n 0 covers the plan of every tile width the call may pick (96 included)
    assert moe.moe_w4afp8_workspace_size(1000, 9, 4096, 4096, 0) >= moe.moe_gemm_workspace_size(1000, 9, 4096, 96)
    T, H, I, E, k = 16384, 4096, 2048, 384, 6
    R, G = T * k + T, E + 1
    ws = moe.moe_workspace_size(T, H, I, E, k, path=moe.MOE_PATH_W4AFP8)
    assert ws >= moe.moe_w4afp8_workspace_size(R, G, 2 * I, H, 0) >= G * 2 * I * H
    assert moe.moe_workspace_size(T, H, I, E, k, path=moe.MOE_PATH_MXFP4) < G * 2 * I * H
