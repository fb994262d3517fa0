"""Loads libmoe.so (built in-tree by fp8_block_scaled_pow2_b200.build) and
declares the C signatures.  Fails loudly when the library is missing: there
is no CPU or framework fallback for any step."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY may point at another build of the same C ABI (e.g. a debug build)
LIB_PATH = os.environ.get("MOE_LIBRARY") or os.path.join(_HERE, "libmoe.so")

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float



class MoeConfig(ctypes.Structure):
    """The C struct MoeConfig (one layer's configuration)."""
    _fields_ = [("T", _I), ("H", _I), ("I", _I), ("E", _I), ("topk", _I), ("route_scale", _F),
                ("swiglu_limit", _F), ("has_shared", _I), ("route_norm", _I)]


# name -> (restype, argtypes)
SIGNATURES = {
    "moe_workspace_size": (_SZ, [ctypes.POINTER(MoeConfig), _I]),
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_version": (_I, []),
    "moe_get_device_error": (_I, [ctypes.POINTER(_I), _P]),
    "moe_selftest_wait_timeout": (_I, [_I64, _P]),
    "moe_quantize_act_fp8": (_I, [_P, _I, _I, _P, _P, _P]),
    "moe_route_topk": (_I, [_P, _I, _I, _I, _F, _I, _P, _P, _P]),
    "moe_route_hash": (_I, [_P, _I, _P, _I, _P, _I, _I, _F, _I, _P, _P, _P]),
    "moe_permute_workspace_size": (_SZ, [_I, _I, _I]),
    "moe_permute": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_permute_noalloc_max_counters": (_I64, []),
    "moe_permute_noalloc": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "moe_prepared_weights_size": (_SZ, [_I64, _I, _I]),
    "moe_prepare_weights": (_I, [_P, _P, _I64, _I, _I, _I, _P, _P]),
    "moe_gemm_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "moe_w4afp8_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "moe_grouped_gemm_mxfp4": (_I, [_P, _P, _I, _P, _I, _P, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _P]),
    "moe_grouped_gemm_w4afp8": (_I, [_P, _P, _I, _P, _I, _P, _P, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _P]),
    "moe_grouped_gemm_fp8_block128": (_I, [_P, _P, _I, _P, _I, _P, _P, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _P]),
    "moe_swiglu_clamp": (_I, [_P, _I, _I, _F, _P, _P, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P]),
    "repack_mxfp4_to_nvfp4": (_I, [_P, _P, _I64, _I, _I, _P, _P, _P, _P]),
    "repack_mxfp4_to_int4g128": (_I, [_P, _P, _I64, _I, _I, _P, _P, _P]),
    "repack_mxfp4_to_fp8_block128": (_I, [_P, _P, _I64, _I, _I, _P, _P, _P]),
    "moe_quantize_fp8_per_token": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_gather_row_scales": (_I, [_P, _I, _I, _P, _I, _P, _P, _P]),
    "moe_grouped_gemm_fp8_ptpc": (_I, [_P, _P, _I, _P, _I, _P, _P, _I, _I, _I, _F, _I, _P, _P, _SZ, _P]),
    "repack_mxfp4_to_fp8_per_channel": (_I, [_P, _P, _I64, _I, _I, _P, _P, _P]),
}

_lib = None


def load(path: str = LIB_PATH):
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libmoe.so not found at {path}; build it with `python -m fp8_block_scaled_pow2_b200.build` "
            "(the CUDA library is required: there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
