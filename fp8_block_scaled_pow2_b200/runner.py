"""Layer steps from pinned host buffers, with the host copies overlapped.

StepRunner owns two sets of device inputs (x, logits) and the Buffers of one
MoeLayer, captures the four step segments (quantise + route + group, w1/w3
GEMM, w2 GEMM, combine) as CUDA graphs (the first once per input set), and
runs step i as

    h2d stream:      wait(step i-2's grouping done) -> x, logits H2D into set i % 2
    compute stream:  wait(H2D) -> pre(set i % 2) -> w1/w3 -> w2
                     -> wait(step i-1's y D2H done) -> combine
    d2h stream:      wait(combine) -> y D2H

so input copies run back to back, each overlapping the previous steps'
compute, and the output copy of step i runs while step i+1 computes (the two
directions on their own streams, so neither waits behind the other).  With
one input set the copy of step i+1 could only start once step i's grouping
had read the inputs, which left it the time of step i's GEMMs alone.  An
input set is free once the grouping segment has read it, and y once its copy
has left.  Every step still moves its own inputs to the device and its result
back.
"""
from __future__ import annotations

import numpy as np
import torch

from .layer import MoeLayer


class StepRunner:
    def __init__(self, layer: MoeLayer, T: int, block_n: int = 0, graphs: bool = True, input_sets: int = 2):
        """input_sets: device copies of the inputs (2: a step's input copy can
        start before the previous step's grouping has read its inputs; 1: half
        the input memory, the copy waits for that grouping)."""
        if input_sets not in (1, 2):
            raise ValueError("input_sets must be 1 or 2")
        self.layer = layer
        self.T = T
        self.n_sets = input_sets
        d = layer.device
        self.buf = layer.alloc(T, block_n)
        self.x = [torch.zeros((T, layer.H), dtype=torch.int16, device=d) for _ in range(input_sets)]
        self.logits = [torch.zeros((T, layer.E), dtype=torch.float32, device=d) for _ in range(input_sets)]
        self.compute = torch.cuda.current_stream(d)
        self.h2d = torch.cuda.Stream(d)
        self.d2h = torch.cuda.Stream(d)
        # the grouping segment once per input set; the other segments read
        # only the step's intermediate buffers
        s0 = layer.segments(self.x[0], self.logits[0], self.buf)
        s1 = layer.segments(self.x[-1], self.logits[-1], self.buf) if input_sets == 2 else s0
        segs = [s0[0], s1[0], s0[1], s0[2], s0[3]] if input_sets == 2 else list(s0)
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
        self.pre_done = [torch.cuda.Event() for _ in range(input_sets)]   # per input set
        self.in_ready = [torch.cuda.Event() for _ in range(input_sets)]
        self.post_done = torch.cuda.Event()
        self.y_copied = torch.cuda.Event()
        self.step = 0
        torch.cuda.synchronize(d)
        for e in self.pre_done:
            e.record(self.compute)
        self.y_copied.record(self.d2h)

    def submit(self, x_host: torch.Tensor, logits_host: torch.Tensor, y_host: torch.Tensor) -> None:
        """Enqueue one step: x_host bf16 bits [T, H] and logits_host float32
        [T, E] in pinned host memory; y_host bf16 [T, H] pinned receives y.
        Asynchronous: y_host holds the result once the d2h stream has passed
        this step's copy (synchronize())."""
        if self.n_sets == 2:
            pre0, pre1, gemm13, gemm2, post = self.run
        else:
            pre0, gemm13, gemm2, post = self.run
            pre1 = pre0
        i = self.step % self.n_sets
        self.step += 1
        with torch.cuda.stream(self.h2d):
            self.h2d.wait_event(self.pre_done[i])        # step - 2 has read this input set
            self.x[i].copy_(x_host, non_blocking=True)
            self.logits[i].copy_(logits_host, non_blocking=True)
            self.in_ready[i].record(self.h2d)
        with torch.cuda.stream(self.compute):          # the segments run on the compute stream
            self.compute.wait_event(self.in_ready[i])
            (pre1 if i else pre0)()
            self.pre_done[i].record(self.compute)
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
