"""A routed-expert MoE FFN layer on top of the C ABI.

MoeLayer owns the device copies of the expert weights (MXFP4, w13 = w1 (gate)
rows followed by w3 (up) rows, then w2), prepared once into the blocks the
tensor-core GEMM streams (moe_prepare_weights), and runs one forward pass as a
fixed sequence of library calls on one stream, with no host synchronisation:

    moe_quantize_act_fp8 -> moe_route_topk -> moe_permute
    -> moe_grouped_gemm_mxfp4(w13, SwiGLU + FP8 requant)
    -> moe_grouped_gemm_mxfp4(w2, float32) -> moe_combine

The shared expert is group E, fed every token with weight 1 ("DeepSeek-V4-
Flash-SI" model card, 架构特性: one shared expert per layer, always active).

tid2eid (int [vocab, topk]) makes it a hash-routed layer (the same card's
first three layers: experts chosen from the token ID): moe_route_hash looks
the experts up by token id in place of moe_route_topk, and forward() /
segments() then take the token ids.

A step whose inputs make a kernel record a device error (an expert id or
token id out of range, see moe_get_device_error) leaves y unspecified: with
the FP8 shared expert, for instance, a rejected pair shifts the shared group
below row T*k, where the side-stream shared GEMMs wrote.  Check the device
error word before using y from untrusted inputs.

weights="ptpc" runs the PTPC-FP8 form of the same layer ("DeepSeek-V4.1-Flash-
Quark-PTPC-FP8" walkthrough, 核心参数): per-channel FP8 weights cast once on
the GPU, per-token dynamic FP8 activations:

    moe_quantize_fp8_per_token -> moe_route_topk -> moe_permute
    -> moe_gather_row_scales -> moe_grouped_gemm_fp8_ptpc(w13, SwiGLU float32)
    -> moe_quantize_fp8_per_token(h) -> moe_grouped_gemm_fp8_ptpc(w2, float32)
    -> moe_combine
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import moe


def _dev(a, device) -> torch.Tensor:
    if isinstance(a, torch.Tensor):
        return a.to(device).contiguous()
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


@dataclasses.dataclass
class Buffers:
    T: int
    xq: torch.Tensor
    sx: torch.Tensor
    idx: torch.Tensor
    w: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    perm: torch.Tensor
    inv: torch.Tensor
    xq_perm: torch.Tensor
    sx_perm: torch.Tensor
    hq: torch.Tensor
    sh: torch.Tensor
    o: torch.Tensor
    y: torch.Tensor
    ws_permute: torch.Tensor
    ws_gemm: torch.Tensor
    block_n: int
    # FP8 shared expert only: offsets [0, T] of its one group and its own GEMM workspace
    shared_off: torch.Tensor | None = None
    ws_shared: torch.Tensor | None = None
    # PTPC-FP8 only: float32 per-row scales and the float32 SwiGLU output
    sxf: torch.Tensor | None = None
    sxf_perm: torch.Tensor | None = None
    hf: torch.Tensor | None = None
    shf: torch.Tensor | None = None


class MoeLayer:
    def __init__(self, w13, w13_e8m0, w2, w2_e8m0, topk: int, route_scale: float = 1.5,
                 swiglu_limit: float = 10.0, has_shared: int = 1, route_norm: int = 1, device="cuda",
                 weights: str = "mxfp4", shared: str = "mxfp4", tid2eid=None):
        """weights="mxfp4" runs the block-scaled MXFP4 GEMMs; weights="w4afp8"
        repacks the experts once on the GPU to symmetric INT4 group-128
        (repack_mxfp4_to_int4g128) and runs the W4AFP8 GEMMs.  shared="fp8"
        casts the shared expert (group E of the arrays) once on the GPU to FP8
        E4M3 with [128, 128] block scales (repack_mxfp4_to_fp8_block128) and
        runs it through moe_grouped_gemm_fp8_block128.  weights="ptpc" casts
        every expert (the shared one included) once on the GPU to PTPC-FP8
        (repack_mxfp4_to_fp8_per_channel) and quantises the activations per
        token."""
        self.device = torch.device(device)
        self.tid2eid = None if tid2eid is None else _dev(np.asarray(tid2eid, np.int32), self.device)
        if self.tid2eid is not None and self.tid2eid.shape[1] != topk:
            raise ValueError("tid2eid must be [vocab, topk]")
        self.G = w13.shape[0]                      # routed experts + shared expert
        self.E = self.G - (1 if has_shared else 0)
        if shared not in ("mxfp4", "fp8") or (shared == "fp8" and (not has_shared or weights == "ptpc")):
            raise ValueError(shared)
        self.shared = shared
        if shared == "fp8":
            d = self.device
            E = self.E
            I2, H = w13.shape[1], w13.shape[2] * 2
            self.ws13_q = torch.empty((1, I2, H), dtype=torch.uint8, device=d)
            self.ws13_s = torch.empty((1, I2 // 128, H // 128), dtype=torch.float32, device=d)
            self.ws2_q = torch.empty((1, H, I2 // 2), dtype=torch.uint8, device=d)
            self.ws2_s = torch.empty((1, H // 128, I2 // 256), dtype=torch.float32, device=d)
            moe.repack_mxfp4_to_fp8_block128(_dev(w13[E:E + 1], d), _dev(w13_e8m0[E:E + 1], d), self.ws13_q,
                                             self.ws13_s)
            moe.repack_mxfp4_to_fp8_block128(_dev(w2[E:E + 1], d), _dev(w2_e8m0[E:E + 1], d), self.ws2_q, self.ws2_s)
            err = moe.moe_get_device_error()
            if err != 0:
                raise moe.MoeError("repack_mxfp4_to_fp8_block128", err)
            # the routed GEMMs cover groups 0 .. E-1 only
            w13, w13_e8m0, w2, w2_e8m0 = w13[:E], w13_e8m0[:E], w2[:E], w2_e8m0[:E]
        self.GR = w13.shape[0]                     # groups of the routed-weight GEMMs
        self.I = w13.shape[1] // 2
        self.H = w13.shape[2] * 2
        assert w2.shape[1] == self.H and w2.shape[2] * 2 == self.I
        self.topk, self.route_scale, self.swiglu_limit = topk, route_scale, swiglu_limit
        self.has_shared, self.route_norm = has_shared, route_norm
        d = self.device
        self.weights = weights
        if weights == "mxfp4":
            # prepared blocks (nibbles + tensor-memory-order scales); the raw
            # MXFP4 arrays are not kept
            w13_d, s13_d = _dev(w13, d), _dev(w13_e8m0, d)
            self.w13_p = torch.empty(moe.moe_prepared_weights_size(self.GR, 2 * self.I, self.H), dtype=torch.uint8,
                                     device=d)
            moe.moe_prepare_weights(w13_d, s13_d, self.w13_p, paired=True)
            del w13_d, s13_d
            w2_d, s2_d = _dev(w2, d), _dev(w2_e8m0, d)
            self.w2_p = torch.empty(moe.moe_prepared_weights_size(self.GR, self.H, self.I), dtype=torch.uint8, device=d)
            moe.moe_prepare_weights(w2_d, s2_d, self.w2_p)
            del w2_d, s2_d
        elif weights == "w4afp8":
            self.w13_q = torch.empty((self.GR, 2 * self.I, self.H // 2), dtype=torch.int8, device=d)
            self.w13_sinv = torch.empty((self.GR, 2 * self.I, self.H // 128), dtype=torch.float32, device=d)
            self.w2_q = torch.empty((self.GR, self.H, self.I // 2), dtype=torch.int8, device=d)
            self.w2_sinv = torch.empty((self.GR, self.H, self.I // 128), dtype=torch.float32, device=d)
            moe.repack_mxfp4_to_int4g128(_dev(w13, d), _dev(w13_e8m0, d), self.w13_q, self.w13_sinv)
            moe.repack_mxfp4_to_int4g128(_dev(w2, d), _dev(w2_e8m0, d), self.w2_q, self.w2_sinv)
            if moe.moe_get_device_error() != 0:
                raise moe.MoeError("repack_mxfp4_to_int4g128", -4)
        elif weights == "ptpc":
            self.w13_q = torch.empty((self.GR, 2 * self.I, self.H), dtype=torch.uint8, device=d)
            self.w13_s = torch.empty((self.GR, 2 * self.I), dtype=torch.float32, device=d)
            self.w2_q = torch.empty((self.GR, self.H, self.I), dtype=torch.uint8, device=d)
            self.w2_s = torch.empty((self.GR, self.H), dtype=torch.float32, device=d)
            moe.repack_mxfp4_to_fp8_per_channel(_dev(w13, d), _dev(w13_e8m0, d), self.w13_q, self.w13_s)
            moe.repack_mxfp4_to_fp8_per_channel(_dev(w2, d), _dev(w2_e8m0, d), self.w2_q, self.w2_s)
            err = moe.moe_get_device_error()
            if err != 0:
                raise moe.MoeError("repack_mxfp4_to_fp8_per_channel", err)
        else:
            raise ValueError(weights)

    def weight_bytes_per_expert(self) -> int:
        """MXFP4 bytes of one expert (nibbles + E8M0 scales of w1, w3, w2)."""
        return 3 * self.I * self.H // 2 + 3 * self.I * self.H // 32

    def alloc(self, T: int, block_n: int = 0) -> Buffers:
        d, H, I, k = self.device, self.H, self.I, self.topk
        R = T * k + (T if self.has_shared else 0)
        u8, i32, f32 = torch.uint8, torch.int32, torch.float32
        # the W4AFP8 w1/w3 GEMM may use narrower token tiles than block_n
        bns = (block_n, 16) if (self.weights in ("w4afp8", "ptpc") or self.shared == "fp8") else (block_n,)
        ws_g = max([moe.moe_gemm_workspace_size(R, self.G, K, bn) for bn in bns for K in (H, I)] + [256])
        if self.weights == "w4afp8":
            # room for the E4M3 copy of the INT4 weights that wide token tiles stream
            ws_g = max([ws_g] + [moe.moe_w4afp8_workspace_size(R, self.GR, N, K, bn) for bn in bns
                                 for N, K in ((2 * I, H), (H, I))])
        return Buffers(
            T=T,
            xq=torch.empty((T, H), dtype=u8, device=d), sx=torch.empty((T, H // 128), dtype=u8, device=d),
            idx=torch.empty((T, k), dtype=i32, device=d), w=torch.empty((T, k), dtype=f32, device=d),
            counts=torch.empty(self.E + 1, dtype=i32, device=d),
            offsets=torch.empty(self.E + 2, dtype=i32, device=d),
            perm=torch.empty(max(R, 1), dtype=i32, device=d), inv=torch.empty(max(T * k, 1), dtype=i32, device=d),
            xq_perm=torch.empty((R, H), dtype=u8, device=d), sx_perm=torch.empty((R, H // 128), dtype=u8, device=d),
            hq=torch.empty((R, I), dtype=u8, device=d), sh=torch.empty((R, I // 128), dtype=u8, device=d),
            o=torch.empty((R, H), dtype=f32, device=d), y=torch.empty((T, H), dtype=torch.bfloat16, device=d),
            ws_permute=torch.empty(moe.moe_permute_workspace_size(T, self.E, k), dtype=u8, device=d),
            ws_gemm=torch.empty(ws_g, dtype=u8, device=d), block_n=block_n,
            **(dict(shared_off=torch.tensor([0, T], dtype=i32, device=d),
                    ws_shared=torch.empty(max([moe.moe_gemm_workspace_size(max(T, 1), 1, K, bn)
                                               for bn in (0, 16, 96, block_n) for K in (H, I)] + [256]),
                                          dtype=u8, device=d))
               if self.shared == "fp8" else {}),
            **(dict(sxf=torch.empty(max(T, 1), dtype=f32, device=d),
                    sxf_perm=torch.zeros(max(R, 1), dtype=f32, device=d),
                    hf=torch.zeros((R, I), dtype=f32, device=d),
                    shf=torch.empty(max(R, 1), dtype=f32, device=d)) if self.weights == "ptpc" else {}))

    def segments(self, x: torch.Tensor, logits: torch.Tensor, buf: Buffers, stream=None, token_ids=None):
        """The forward pass as four callables run in order on `stream`:
        (quantise + route + group, w1/w3 GEMM with SwiGLU, w2 GEMM, combine).
        Each only enqueues library calls, so each can be captured in a CUDA
        graph; forward() runs them eagerly.  token_ids (int32 [T], device):
        required by a hash-routed layer."""
        b = buf
        if self.tid2eid is not None and (token_ids is None or token_ids.dtype != torch.int32):
            raise ValueError("a hash-routed layer needs int32 token_ids")
        g_off = b.offsets[: self.GR + 1]          # the groups of the routed-weight GEMMs

        ptpc = self.weights == "ptpc"

        shared_fp8 = self.shared == "fp8"
        if shared_fp8:
            # The shared expert sees every token in token order, so its GEMMs read
            # xq / sx directly (one group [0, T)) and write rows T*k .. T*k+T of
            # hq / sh / o, where the grouping places the shared group (all T*k
            # routed pairs carry valid expert ids: the routing produces them).
            # They run on a side stream while routing and grouping run.
            Tk = b.T * self.topk
            bn_sh = b.block_n or (16 if b.T <= 256 else 0)
            bn_sh_dual = min(bn_sh, 64) if bn_sh else 0
            if getattr(self, "_side", None) is None:
                self._side = torch.cuda.Stream(self.device)
            side = self._side

            def shared_gemms():
                moe.moe_grouped_gemm_fp8_block128(b.xq, b.sx, b.shared_off, self.ws13_q, self.ws13_s,
                                                  moe.MOE_EPI_SWIGLU_QUANT, b.hq[Tk:], b.sh[Tk:], b.ws_shared,
                                                  self.swiglu_limit, bn_sh_dual)
                moe.moe_grouped_gemm_fp8_block128(b.hq[Tk:], b.sh[Tk:], b.shared_off, self.ws2_q, self.ws2_s,
                                                  moe.MOE_EPI_STORE_F32, b.o[Tk:], None, b.ws_shared,
                                                  self.swiglu_limit, bn_sh)

        def pre():
            main = stream if stream is not None else torch.cuda.current_stream(self.device)
            if ptpc:
                moe.moe_quantize_fp8_per_token(x, b.xq, b.sxf, stream=stream)
            else:
                moe.moe_quantize_act_fp8(x, b.xq, b.sx, stream=stream)
            if shared_fp8 and b.T > 0:
                side.wait_stream(main)                   # xq, sx are ready
                with torch.cuda.stream(side):
                    shared_gemms()
            if self.tid2eid is not None:
                moe.moe_route_hash(token_ids, self.tid2eid, logits, b.idx, b.w, self.route_scale, self.route_norm,
                                   stream=stream)
            else:
                moe.moe_route_topk(logits, self.topk, b.idx, b.w, self.route_scale, self.route_norm, stream=stream)
            # (PTPC: the E8M0 rows moved alongside are unused; the float32
            # per-token scales follow the rows through moe_gather_row_scales)
            moe.moe_permute(b.idx, self.E, self.has_shared, b.xq, b.sx, b.counts, b.offsets, b.perm, b.inv,
                            b.xq_perm, b.sx_perm, b.ws_permute, stream=stream)
            if ptpc:
                moe.moe_gather_row_scales(b.perm, b.T, self.topk, b.offsets, self.E, b.sxf, b.sxf_perm,
                                          stream=stream)
            if shared_fp8 and b.T > 0:
                main.wait_stream(side)                   # the shared rows of hq, sh and o are written

        bn_dual = min(b.block_n, 64) if b.block_n else 0
        if self.weights == "mxfp4":
            def routed13():
                moe.moe_grouped_gemm_mxfp4(b.xq_perm, b.sx_perm, g_off, self.w13_p, self.GR, 2 * self.I,
                                           moe.MOE_EPI_SWIGLU_QUANT, b.hq, b.sh, b.ws_gemm, self.swiglu_limit,
                                           b.block_n, stream=stream)

            def routed2():
                moe.moe_grouped_gemm_mxfp4(b.hq, b.sh, g_off, self.w2_p, self.GR, self.H, moe.MOE_EPI_STORE_F32,
                                           b.o, None, b.ws_gemm, self.swiglu_limit, b.block_n, stream=stream)
        elif ptpc:
            def routed13():
                moe.moe_grouped_gemm_fp8_ptpc(b.xq_perm, b.sxf_perm, g_off, self.w13_q, self.w13_s,
                                              moe.MOE_EPI_SWIGLU_F32, b.hf, b.ws_gemm, self.swiglu_limit, bn_dual,
                                              stream=stream)
                moe.moe_quantize_fp8_per_token(b.hf, b.hq, b.shf, stream=stream)

            def routed2():
                moe.moe_grouped_gemm_fp8_ptpc(b.hq, b.shf, g_off, self.w2_q, self.w2_s, moe.MOE_EPI_STORE_F32,
                                              b.o, b.ws_gemm, self.swiglu_limit, b.block_n, stream=stream)
        else:
            def routed13():
                moe.moe_grouped_gemm_w4afp8(b.xq_perm, b.sx_perm, g_off, self.w13_q, self.w13_sinv,
                                            moe.MOE_EPI_SWIGLU_QUANT, b.hq, b.sh, b.ws_gemm, self.swiglu_limit,
                                            bn_dual, stream=stream)

            def routed2():
                moe.moe_grouped_gemm_w4afp8(b.hq, b.sh, g_off, self.w2_q, self.w2_sinv, moe.MOE_EPI_STORE_F32,
                                            b.o, None, b.ws_gemm, self.swiglu_limit, b.block_n, stream=stream)
        gemm13, gemm2 = routed13, routed2

        def post():
            moe.moe_combine(b.o, b.inv, b.w, self.has_shared, b.offsets, self.E, b.y, stream=stream)

        return pre, gemm13, gemm2, post

    def forward(self, x: torch.Tensor, logits: torch.Tensor, buf: Buffers | None = None,
                stream=None, marks=None, token_ids=None) -> torch.Tensor:
        """x bfloat16 [T, H] (or its uint16 bits), logits float32 [T, E] -> y bfloat16 [T, H].
        token_ids int32 [T] (device): the token ids of a hash-routed layer.

        marks: optional three torch.cuda.Event recorded on the stream before the
        w1/w3 GEMM, between the GEMMs and after the w2 GEMM (for timing)."""
        T = x.shape[0]
        if buf is None or buf.T != T:
            buf = self.alloc(T)
        ev_stream = stream if stream is not None else torch.cuda.current_stream()
        for i, seg in enumerate(self.segments(x, logits, buf, stream, token_ids=token_ids)):
            if marks and i > 0:
                marks[i - 1].record(ev_stream)
            seg()
        return buf.y
