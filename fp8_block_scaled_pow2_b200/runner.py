"""Layer steps from pinned host buffers, with the host copies overlapped.

StepRunner owns the device inputs (x, logits) and the Buffers of one
MoeLayer, captures the four step segments (quantise + route + group, w1/w3
GEMM, w2 GEMM, combine) as CUDA graphs, and runs each step as

    h2d stream:      wait(previous step's grouping done) -> x, logits H2D
    compute stream:  wait(H2D) -> pre -> w1/w3 -> w2
                     -> wait(previous step's y D2H done) -> combine
    d2h stream:      wait(combine) -> y D2H

so the input copy of step i+1 runs while step i's GEMMs run, and the output
copy of step i while step i+1 computes (the two directions on their own
streams, so neither waits behind the other).  The device input buffers are free
once the grouping segment has read them, and y once its copy has left.
Every step still moves its own inputs to the device and its result back.
"""
from __future__ import annotations

import numpy as np
import torch

from .layer import MoeLayer


class StepRunner:
    def __init__(self, layer: MoeLayer, T: int, block_n: int = 0, graphs: bool = True):
        self.layer = layer
        self.T = T
        d = layer.device
        self.buf = layer.alloc(T, block_n)
        self.x = torch.zeros((T, layer.H), dtype=torch.int16, device=d)
        self.logits = torch.zeros((T, layer.E), dtype=torch.float32, device=d)
        self.compute = torch.cuda.current_stream(d)
        self.h2d = torch.cuda.Stream(d)
        self.d2h = torch.cuda.Stream(d)
        segs = layer.segments(self.x, self.logits, self.buf)
        if graphs:
            for f in segs:              # load code and tensor maps before capture
                f()
            torch.cuda.synchronize(d)
            self.graphs = []
            for f in segs:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    f()
                self.graphs.append(g)
            self.run = [g.replay for g in self.graphs]
        else:
            self.graphs = []
            self.run = list(segs)
        self.pre_done = torch.cuda.Event()
        self.in_ready = torch.cuda.Event()
        self.post_done = torch.cuda.Event()
        self.y_copied = torch.cuda.Event()
        torch.cuda.synchronize(d)
        self.pre_done.record(self.compute)
        self.y_copied.record(self.d2h)

    def submit(self, x_host: torch.Tensor, logits_host: torch.Tensor, y_host: torch.Tensor) -> None:
        """Enqueue one step: x_host bf16 bits [T, H] and logits_host float32
        [T, E] in pinned host memory; y_host bf16 [T, H] pinned receives y.
        Asynchronous: y_host holds the result once the d2h stream has passed
        this step's copy (synchronize())."""
        pre, gemm13, gemm2, post = self.run
        with torch.cuda.stream(self.h2d):
            self.h2d.wait_event(self.pre_done)           # the previous step has read x and logits
            self.x.copy_(x_host, non_blocking=True)
            self.logits.copy_(logits_host, non_blocking=True)
            self.in_ready.record(self.h2d)
        with torch.cuda.stream(self.compute):          # the segments run on the compute stream
            self.compute.wait_event(self.in_ready)
            pre()
            self.pre_done.record(self.compute)
            gemm13()
            gemm2()
            self.compute.wait_event(self.y_copied)       # the previous y has left
            post()
            self.post_done.record(self.compute)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.post_done)
            y_host.copy_(self.buf.y, non_blocking=True)
            self.y_copied.record(self.d2h)

    def synchronize(self) -> None:
        self.h2d.synchronize()
        self.compute.synchronize()
        self.d2h.synchronize()

    def close(self) -> None:
        self.synchronize()
        self.graphs = []
        self.run = []


def pinned_inputs(x_bf16_bits: np.ndarray, logits: np.ndarray):
    """Pinned host copies of one step's inputs and a pinned y buffer."""
    xh = torch.from_numpy(np.ascontiguousarray(x_bf16_bits).view(np.int16)).pin_memory()
    lh = torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)).pin_memory()
    yh = torch.empty((xh.shape[0], xh.shape[1]), dtype=torch.bfloat16).pin_memory()
    return xh, lh, yh
