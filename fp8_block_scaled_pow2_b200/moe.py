"""Python binding of libmoe (the C ABI declared in include/moe_fp8_pow2.h).

Each function has the name of its C entry point, takes torch tensors that
already live on the GPU, and only marshals arguments: pointers, sizes and the
current CUDA stream.  Every step runs in the library's kernels; there is no
fallback.  A non-zero status raises MoeError.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import load

MOE_EPI_STORE_F32 = 0
MOE_EPI_STORE_BF16 = 1
MOE_EPI_SWIGLU_QUANT = 2
MOE_EPI_SWIGLU_F32 = 3


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib().moe_status_string(status).decode()
        super().__init__(f"{fn}: {msg} ({status})")
        self.status = status


def _lib():
    return load()


def _ptr(t: torch.Tensor | None) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MoeError(fn, status)


def moe_get_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("moe_get_device_error", _lib().moe_get_device_error(ctypes.byref(code), _stream(stream)))
    return code.value


def moe_selftest_wait_timeout(timeout_ns: int, stream=None):
    _check("moe_selftest_wait_timeout", _lib().moe_selftest_wait_timeout(int(timeout_ns), _stream(stream)))


def moe_quantize_act_fp8(x, xq, sx, stream=None):
    rows, cols = x.shape
    _check("moe_quantize_act_fp8",
           _lib().moe_quantize_act_fp8(_ptr(x), rows, cols, _ptr(xq), _ptr(sx), _stream(stream)))


def moe_route_topk(logits, k, idx, w, route_scale=1.5, route_norm=1, stream=None):
    T, E = logits.shape
    _check("moe_route_topk", _lib().moe_route_topk(_ptr(logits), T, E, k, ctypes.c_float(route_scale),
                                                   int(route_norm), _ptr(idx), _ptr(w), _stream(stream)))


def moe_route_hash(token_ids, tid2eid, logits, idx, w, route_scale=1.5, route_norm=1, stream=None):
    T, E = logits.shape
    vocab, k = tid2eid.shape
    if token_ids.shape != (T,):
        raise ValueError("token_ids must be [T]")
    _check("moe_route_hash", _lib().moe_route_hash(_ptr(token_ids), T, _ptr(tid2eid), vocab, _ptr(logits), E, k,
                                                   ctypes.c_float(route_scale), int(route_norm), _ptr(idx),
                                                   _ptr(w), _stream(stream)))


def moe_permute_workspace_size(T: int, E: int, k: int) -> int:
    return int(_lib().moe_permute_workspace_size(T, E, k))


def moe_permute(idx, E, has_shared, xq, sx, counts, offsets, perm, inv, xq_perm, sx_perm, workspace,
                stream=None):
    T, k = idx.shape
    H = xq.shape[1]
    _check("moe_permute", _lib().moe_permute(
        _ptr(idx), T, E, k, int(has_shared), _ptr(xq), _ptr(sx), H, _ptr(counts), _ptr(offsets),
        _ptr(perm), _ptr(inv), _ptr(xq_perm), _ptr(sx_perm), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_permute_noalloc(idx, E, has_shared, xq, sx, counts, offsets, perm, inv, xq_perm, sx_perm, stream=None):
    """moe_permute for callers that cannot allocate device scratch: the library
    keeps the counters in its own fixed device array (see the C header for the
    size limit and the rule that overlapping calls race)."""
    T, k = idx.shape
    H = xq.shape[1]
    _check("moe_permute_noalloc", _lib().moe_permute_noalloc(
        _ptr(idx), T, E, k, int(has_shared), _ptr(xq), _ptr(sx), H, _ptr(counts), _ptr(offsets),
        _ptr(perm), _ptr(inv), _ptr(xq_perm), _ptr(sx_perm), _stream(stream)))


def moe_permute_noalloc_max_counters() -> int:
    return int(_lib().moe_permute_noalloc_max_counters())


def moe_prepared_weights_size(n_mats: int, N: int, K: int) -> int:
    return int(_lib().moe_prepared_weights_size(n_mats, N, K))


def moe_prepare_weights(fp4, e8m0, prepared, paired=False, stream=None):
    """MXFP4 nibbles [n_mats, N, K/2] + E8M0 [n_mats, N, K/32] -> prepared
    blocks (moe_prepared_weights_size bytes); paired=True for w1/w3 used with
    MOE_EPI_SWIGLU_QUANT (gate and up blocks side by side)."""
    n_mats, N, k2 = fp4.shape
    _check("moe_prepare_weights", _lib().moe_prepare_weights(
        _ptr(fp4), _ptr(e8m0), n_mats, N, k2 * 2, int(bool(paired)), _ptr(prepared), _stream(stream)))


MOE_PATH_MXFP4, MOE_PATH_W4AFP8, MOE_PATH_PTPC = 0, 1, 2


def moe_workspace_size(T: int, H: int, I: int, E: int, topk: int, has_shared: int = 1, path: int = 0,
                       route_scale: float = 1.5, swiglu_limit: float = 10.0, route_norm: int = 1) -> int:
    """Scratch bytes for moe_permute and every grouped GEMM of one layer step."""
    from ._lib import MoeConfig
    cfg = MoeConfig(T, H, I, E, topk, route_scale, swiglu_limit, int(has_shared), int(route_norm))
    return int(_lib().moe_workspace_size(ctypes.byref(cfg), int(path)))


def moe_gemm_workspace_size(a_rows: int, n_groups: int, K: int, block_n: int = 0) -> int:
    return int(_lib().moe_gemm_workspace_size(a_rows, n_groups, K, block_n))


def moe_w4afp8_workspace_size(a_rows: int, n_groups: int, N: int, K: int, block_n: int = 0) -> int:
    return int(_lib().moe_w4afp8_workspace_size(a_rows, n_groups, N, K, block_n))


def moe_grouped_gemm_mxfp4(a, a_scale, offsets, w_prepared, G, N, epilogue, out, out_scale=None,
                           workspace=None, swiglu_limit=10.0, block_n=0, stream=None):
    """w_prepared: moe_prepare_weights output for G matrices [N, K] (K = a.shape[1])."""
    a_rows, K = a.shape
    _check("moe_grouped_gemm_mxfp4", _lib().moe_grouped_gemm_mxfp4(
        _ptr(a), _ptr(a_scale), a_rows, _ptr(offsets), G, _ptr(w_prepared), N, K,
        int(epilogue), ctypes.c_float(swiglu_limit), int(block_n), _ptr(out), _ptr(out_scale),
        _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def moe_grouped_gemm_w4afp8(a, a_scale, offsets, w_int4, w_scale_inv, epilogue, out, out_scale=None,
                            workspace=None, swiglu_limit=10.0, block_n=0, stream=None):
    a_rows, K = a.shape
    G, N = w_int4.shape[0], w_int4.shape[1]
    _check("moe_grouped_gemm_w4afp8", _lib().moe_grouped_gemm_w4afp8(
        _ptr(a), _ptr(a_scale), a_rows, _ptr(offsets), G, _ptr(w_int4), _ptr(w_scale_inv), N, K,
        int(epilogue), ctypes.c_float(swiglu_limit), int(block_n), _ptr(out), _ptr(out_scale),
        _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def moe_grouped_gemm_fp8_block128(a, a_scale, offsets, w_e4m3, w_scale_inv, epilogue, out, out_scale=None,
                                  workspace=None, swiglu_limit=10.0, block_n=0, stream=None):
    """FP8 rows x FP8 weights [G, N, K] with float32 scale_inv [G, N/128, K/128];
    offsets [G+1] may start above 0 (a view into a larger grouping)."""
    a_rows, K = a.shape
    G, N = w_e4m3.shape[0], w_e4m3.shape[1]
    _check("moe_grouped_gemm_fp8_block128", _lib().moe_grouped_gemm_fp8_block128(
        _ptr(a), _ptr(a_scale), a_rows, _ptr(offsets), G, _ptr(w_e4m3), _ptr(w_scale_inv), N, K,
        int(epilogue), ctypes.c_float(swiglu_limit), int(block_n), _ptr(out), _ptr(out_scale),
        _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def moe_grouped_gemm_fp8_ptpc(a, a_scale, offsets, w_e4m3, w_scale, epilogue, out, workspace=None,
                              swiglu_limit=10.0, block_n=0, stream=None):
    """PTPC-FP8: E4M3 rows [R, K] with float32 per-row scales [R] x E4M3 weights
    [G, N, K] with float32 per-channel scales [G, N]."""
    a_rows, K = a.shape
    G, N = w_e4m3.shape[0], w_e4m3.shape[1]
    _check("moe_grouped_gemm_fp8_ptpc", _lib().moe_grouped_gemm_fp8_ptpc(
        _ptr(a), _ptr(a_scale), a_rows, _ptr(offsets), G, _ptr(w_e4m3), _ptr(w_scale), N, K,
        int(epilogue), ctypes.c_float(swiglu_limit), int(block_n), _ptr(out),
        _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def moe_quantize_fp8_per_token(x, q, scale, stream=None):
    """bfloat16 or float32 [rows, cols] -> E4M3 [rows, cols] + float32 scale [rows]."""
    rows, cols = x.shape
    is_f32 = 1 if x.element_size() == 4 else 0
    _check("moe_quantize_fp8_per_token", _lib().moe_quantize_fp8_per_token(
        _ptr(x), is_f32, rows, cols, _ptr(q), _ptr(scale), _stream(stream)))


def moe_gather_row_scales(perm, T, k, offsets, E, src, dst, stream=None):
    _check("moe_gather_row_scales", _lib().moe_gather_row_scales(
        _ptr(perm), T, k, _ptr(offsets), E, _ptr(src), _ptr(dst), _stream(stream)))


def moe_swiglu_clamp(gu, hq, sh, limit=10.0, stream=None):
    rows, two_i = gu.shape
    _check("moe_swiglu_clamp", _lib().moe_swiglu_clamp(_ptr(gu), rows, two_i // 2, ctypes.c_float(limit),
                                                       _ptr(hq), _ptr(sh), _stream(stream)))


def moe_combine(o, inv, w, has_shared, offsets, E, y, stream=None):
    T, k = w.shape
    H = o.shape[1]
    _check("moe_combine", _lib().moe_combine(_ptr(o), _ptr(inv), _ptr(w), T, k, H, int(has_shared),
                                             _ptr(offsets), E, _ptr(y), _stream(stream)))


def repack_mxfp4_to_nvfp4(fp4, e8m0, out_fp4, out_e4m3, out_global, stream=None):
    n_mats, N, k2 = fp4.shape
    _check("repack_mxfp4_to_nvfp4", _lib().repack_mxfp4_to_nvfp4(
        _ptr(fp4), _ptr(e8m0), n_mats, N, k2 * 2, _ptr(out_fp4), _ptr(out_e4m3), _ptr(out_global),
        _stream(stream)))


def repack_mxfp4_to_int4g128(fp4, e8m0, out_int4, out_scale_inv, stream=None):
    n_mats, N, k2 = fp4.shape
    _check("repack_mxfp4_to_int4g128", _lib().repack_mxfp4_to_int4g128(
        _ptr(fp4), _ptr(e8m0), n_mats, N, k2 * 2, _ptr(out_int4), _ptr(out_scale_inv), _stream(stream)))


def repack_mxfp4_to_fp8_block128(fp4, e8m0, out_e4m3, out_scale_inv, stream=None):
    """MXFP4 [n_mats, N, K/2] + E8M0 [n_mats, N, K/32] -> E4M3 [n_mats, N, K] and
    float32 scale_inv [n_mats, N/128, K/128] (power-of-two block scales)."""
    n_mats, N, k2 = fp4.shape
    _check("repack_mxfp4_to_fp8_block128", _lib().repack_mxfp4_to_fp8_block128(
        _ptr(fp4), _ptr(e8m0), n_mats, N, k2 * 2, _ptr(out_e4m3), _ptr(out_scale_inv), _stream(stream)))


def repack_mxfp4_to_fp8_per_channel(fp4, e8m0, out_e4m3, out_scale, stream=None):
    """MXFP4 [n_mats, N, K/2] + E8M0 [n_mats, N, K/32] -> E4M3 [n_mats, N, K] and
    float32 per-channel scales [n_mats, N]."""
    n_mats, N, k2 = fp4.shape
    _check("repack_mxfp4_to_fp8_per_channel", _lib().repack_mxfp4_to_fp8_per_channel(
        _ptr(fp4), _ptr(e8m0), n_mats, N, k2 * 2, _ptr(out_e4m3), _ptr(out_scale), _stream(stream)))
