"""Benchmark of the routed-expert MoE layer (MXFP4 experts, FP8 activations).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|long_prefill|repack|decode_small|prefill_small|repack_small]

A step is one pass of the whole expert path (quantise, route, group, w1/w3
GEMM + SwiGLU + requantise, w2 GEMM, combine) over one batch of synthetic
tokens.  The default workload is the decode layer of a DeepSeek-V4-Flash-
class model: hidden 4096, expert intermediate 2048, 256 routed + 1 shared
experts, top-6, 64 tokens of N(0,1) activations with 0.1% outliers x20,
uniform router logits, MXFP4 experts from N(0, 0.02).  Each rank runs its own
replica on its own tokens (data parallel, no collective on the data path);
`value` is the tokens of all ranks divided by the slowest rank's device time.

One JSON line is printed by rank 0.  `--impl reference` times the CPU oracle
(rank 0 only) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and expert-GEMM TFLOP/s or HBM GB/s vs B200 roofline"
def kernels_per_step(wl: dict, shared: str = "mxfp4", weights: str = "mxfp4") -> int:
    """Library kernels one layer step launches: quant 1, route 1, grouping 2
    (one block for <= 2048 routed pairs, then the gather) or 4 (chunked), two
    GEMM calls of 2 (prep + GEMM; two more with the FP8 shared expert),
    combine 1.  PTPC-FP8 adds the row-scale gather and the per-token
    quantisation of h."""
    grouping = 2 if wl["T"] * wl["k"] <= 2048 else 4
    gemm_calls = 4 if shared == "fp8" else 2
    extra = 2 if weights == "ptpc" else 0
    return 1 + 1 + grouping + gemm_calls * 2 + 1 + extra

WORKLOADS = {
    "repack": dict(T=0, H=4096, I=2048, E=256, k=6, logits="uniform"),
    "decode": dict(T=64, H=4096, I=2048, E=256, k=6, logits="uniform"),
    "prefill": dict(T=4096, H=4096, I=2048, E=256, k=6, logits="zipf"),
    "long_prefill": dict(T=16384, H=4096, I=2048, E=384, k=6, logits="zipf"),
    # small cases of the same shapes, for kernel profiles (a few hundred MB on the device)
    "decode_small": dict(T=64, H=4096, I=2048, E=32, k=6, logits="uniform"),
    "prefill_small": dict(T=1024, H=4096, I=2048, E=32, k=6, logits="zipf"),
    "repack_small": dict(T=0, H=4096, I=2048, E=16, k=6, logits="uniform"),
}


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


GEMM_ENTRY = {"mxfp4": "moe_grouped_gemm_mxfp4", "w4afp8": "moe_grouped_gemm_w4afp8",
              "ptpc": "moe_grouped_gemm_fp8_ptpc"}
GEMM_SOURCES = {"mxfp4": ("common.cuh", "gemm_mxfp4.cuh", "sm100.cuh"),
                "w4afp8": ("common.cuh", "gemm_mxfp4.cuh", "gemm_w4afp8.cuh", "sm100.cuh"),
                "ptpc": ("common.cuh", "gemm_mxfp4.cuh", "gemm_w4afp8.cuh", "sm100.cuh")}


def source_digest(weights: str = "mxfp4") -> str:
    """Digest of the grouped-GEMM kernel sources: recorded DRAM traffic is only
    reported while these are unchanged since the ncu capture."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_block_scaled_pow2_b200", "csrc")
    for f in GEMM_SOURCES[weights]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, weights: str = "mxfp4"):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, or None when the kernels changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(workload)
    if not d or d.get("source_digest") != source_digest(weights) or d.get("weights", "mxfp4") != weights:
        return None
    return d.get("traffic_bytes_per_launch")


def make_inputs(wl: dict, seed: int, rank: int):
    import synth
    T, H, I, E = wl["T"], wl["H"], wl["I"], wl["E"]
    w13, s13, w2, s2 = synth.expert_weights(seed, E + 1, H, I, n_proto=4)
    x = synth.decode_activations(seed + 1000 * rank, T, H)
    logits = (synth.uniform_logits if wl["logits"] == "uniform" else synth.zipf_logits)(seed + 1000 * rank, T, E)
    return x, logits, (w13, s13, w2, s2)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms from before
    the warm-up to after the timed region; summary() keeps the samples whose
    nvidia-smi timestamp falls inside the timed window (widened to the two
    nearest samples when the window is shorter than the sampling period)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = str(gpu_index)
        try:                                    # address the GPU by UUID: robust to device remapping
            import torch
            self.gpu = "GPU-" + str(torch.cuda.get_device_properties(gpu_index).uuid)
        except Exception:
            pass
        self.proc = None
        self.window = None
        # MOE_CLOCKS_DIR: where the sampled clock log is kept (default: a temp dir)
        self.path = os.path.join(os.environ.get("MOE_CLOCKS_DIR") or tempfile.gettempdir(),
                                 f"moe_clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "20", "-i", self.gpu], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return self
        t0 = time.time()
        while time.time() - t0 < 5.0 and os.path.getsize(self.path) == 0 and self.proc.poll() is None:
            time.sleep(0.02)
        return self

    def mark(self, t_begin: float, t_end: float):
        self.window = (t_begin, t_end)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.06)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or self.window is None or not os.path.exists(self.path):
            return None
        import datetime
        rows = []
        with open(self.path) as f:
            for ln in f:
                p = [c.strip() for c in ln.split(",")]
                if len(p) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(p[2]), float(p[3]), p[6:10]))
                except ValueError:
                    continue
        if not rows:
            return None
        b, e = self.window
        inside = [r for r in rows if b <= r[0] <= e]
        if len(inside) < 2:
            inside = sorted(rows, key=lambda r: min(abs(r[0] - b), abs(r[0] - e)))[:2]
        reasons = sorted({n for r in inside for n, v in zip(self.REASONS, r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "window_ms": round(1e3 * (e - b), 1)}


def dist_setup(n_gpus: int):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    else:
        torch.cuda.set_device(0)
    return rank, world, local, pg


def max_over_ranks(value: float, pg) -> float:
    """The slowest rank's time (every rank gets it); plumbing only."""
    if pg is None:
        return value
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


def algorithmic_bytes(layer, buf, wl) -> dict:
    """Bytes each GEMM must move at least once: weights of every expert that
    received rows (nibbles + E8M0 scales), FP8 inputs with their scales, outputs."""
    counts = buf.counts.cpu().numpy()
    active = int((counts > 0).sum())
    R = int(counts.sum())
    H, I = wl["H"], wl["I"]
    w13 = 2 * I * H // 2 + 2 * I * H // 32
    w2 = H * I // 2 + H * I // 32
    w13_bytes = active * w13
    w2_bytes = active * w2
    shared_fp8 = 0
    Rg = R                                       # rows of the grouped (segment-timed) GEMMs
    if getattr(layer, "shared", "mxfp4") == "fp8" and counts[-1] > 0:
        # the FP8 shared expert runs beside the grouping (pre-GEMM segment): its
        # E4M3 weights with float32 [128, 128] block scales, its rows in and out
        w13_bytes -= w13
        w2_bytes -= w2
        Ts = int(counts[-1])
        Rg = R - Ts
        active -= 1
        shared_fp8 = (2 * I * H + 4 * (2 * I // 128) * (H // 128) + H * I + 4 * (H // 128) * (I // 128)
                      + Ts * (H + H // 128) + 2 * Ts * (I + I // 128) + 4 * Ts * H)
    T, E, k = wl["T"], wl["E"], wl["k"]
    ptpc = getattr(layer, "weights", "mxfp4") == "ptpc"
    # quantise (bf16 in, E4M3 + scales out), route (logits in, ids + weights
    # out), group (ids in, perm + inv out, rows and scales gathered), plus the
    # row-scale gather of PTPC; combine (k routed rows + the shared row in,
    # bf16 out, ids + weights in)
    quant = T * H * 2 + T * H + (4 * T if ptpc else T * H // 128)
    route = T * E * 4 + T * k * 8
    group = T * k * 4 + R * 4 + T * k * 4 + 2 * R * (H + H // 128)
    pre = quant + route + group + (3 * 4 * R if ptpc else 0) + shared_fp8
    post = R * H * 4 + T * k * 8 + T * H * 2
    if ptpc:
        # E4M3 weights with one float32 scale per channel; activations E4M3
        # with one float32 scale per row (the float32 h round trip between
        # the GEMM and its per-token requantisation is not counted)
        return dict(active_experts=active, rows=R, pre=pre, post=post,
                    w13=active * (2 * I * H + 4 * 2 * I) + R * (H + 4) + R * (I + 4),
                    w2=active * (H * I + 4 * H) + R * (I + 4) + R * H * 4,
                    flops13=2.0 * R * 2 * I * H, flops2=2.0 * R * H * I)
    return dict(active_experts=active, rows=Rg, pre=pre, post=post,
                w13=w13_bytes + Rg * (H + H // 128) + Rg * (I + I // 128),
                w2=w2_bytes + Rg * (I + I // 128) + Rg * H * 4,
                flops13=2.0 * Rg * 2 * I * H, flops2=2.0 * Rg * H * I)


def run_repack(args, wl):
    """Weight repack sweep: one layer of E experts x (w1, w3 [I, H], w2 [H, I])
    MXFP4 -> NVFP4 (E4M3 scale per 16, per-matrix global scale), -> symmetric
    INT4 group 128 (fp32 scale_inv [N, K/128]) and -> FP8 E4M3 with a
    [128, 128] block scale.  One step = the three repacks of the whole layer.  Metric: GB/s of algorithmic bytes (each repack reads its
    source once and writes its outputs once)."""
    import torch

    import synth
    from fp8_block_scaled_pow2_b200 import moe

    rank, world, local, pg = dist_setup(args.gpus)
    E, H, I = wl["E"], wl["H"], wl["I"]
    w13, s13, w2, s2 = synth.expert_weights(args.seed, E, H, I, n_proto=4)
    # w1 and w3 are separate [I, H] matrices: view w13 [E, 2I, H/2] as [2E, I, H/2]
    mats = [(torch.from_numpy(w13.reshape(2 * E, I, H // 2)).cuda(), torch.from_numpy(s13.reshape(2 * E, I, H // 32)).cuda()),
            (torch.from_numpy(w2).cuda(), torch.from_numpy(s2).cuda())]
    outs = []
    nv_bytes = int4_bytes = fp8_bytes = 0
    for fp4, e8 in mats:
        M, N, k2 = fp4.shape
        K = 2 * k2
        o = dict(nv_fp4=torch.empty_like(fp4), nv_s=torch.empty((M, N, K // 16), dtype=torch.uint8, device="cuda"),
                 nv_g=torch.empty(M, dtype=torch.float32, device="cuda"),
                 q=torch.empty((M, N, k2), dtype=torch.int8, device="cuda"),
                 sinv=torch.empty((M, N, K // 128), dtype=torch.float32, device="cuda"),
                 f8=torch.empty((M, N, K), dtype=torch.uint8, device="cuda"),
                 f8_s=torch.empty((M, N // 128, K // 128), dtype=torch.float32, device="cuda"))
        outs.append(o)
        nv_bytes += 2 * fp4.numel() + e8.numel() + o["nv_s"].numel() + 4 * M
        int4_bytes += fp4.numel() + e8.numel() + o["q"].numel() + 4 * o["sinv"].numel()
        fp8_bytes += fp4.numel() + e8.numel() + o["f8"].numel() + 4 * o["f8_s"].numel()
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev: ev[0].record(stream)
        for (fp4, e8), o in zip(mats, outs):
            moe.repack_mxfp4_to_nvfp4(fp4, e8, o["nv_fp4"], o["nv_s"], o["nv_g"])
        if ev: ev[1].record(stream)
        for (fp4, e8), o in zip(mats, outs):
            moe.repack_mxfp4_to_int4g128(fp4, e8, o["q"], o["sinv"])
        if ev: ev[2].record(stream)
        for (fp4, e8), o in zip(mats, outs):
            moe.repack_mxfp4_to_fp8_block128(fp4, e8, o["f8"], o["f8_s"])
        if ev: ev[3].record(stream)

    clk = ClockSampler(local).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(pg)
    torch.cuda.synchronize()
    w_begin = time.time()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk.mark(w_begin, time.time())
    clk.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), pg)
    nv_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    i4_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    f8_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    peaks = read_peaks()
    total = (nv_bytes + int4_bytes + fp8_bytes) * world * args.steps
    gbs = total / (ms / 1e3) / 1e9
    nv_gbs = nv_bytes / (nv_ms / 1e3) / 1e9
    line = {
        "metric": "weight repack GB/s vs B200 HBM roofline", "value": round(gbs, 1), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": f"repack sweep: {E} experts x (w1, w3 [{I}, {H}], w2 [{H}, {I}]) MXFP4 -> NVFP4, "
                               f"-> INT4 group 128 and -> FP8 E4M3 [128, 128] blocks", "l2": "inputs larger than L2 (3.4 GB per repack)"},
        "roofline": {"bound": "hbm", "achieved": round(nv_gbs, 1), "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": round(nv_gbs / peaks["hbm"], 4), "traffic": None, "kernel": "repack_mxfp4_to_nvfp4",
                     "peak_source": f"{peaks['src']} HBM copy"},
        "repack": {"nvfp4_ms": round(nv_ms, 4), "nvfp4_GBps": round(nv_gbs, 1),
                   "int4_ms": round(i4_ms, 4), "int4_GBps": round(int4_bytes / (i4_ms / 1e3) / 1e9, 1),
                   "fp8_ms": round(f8_ms, 4), "fp8_GBps": round(fp8_bytes / (f8_ms / 1e3) / 1e9, 1),
                   "nvfp4_bytes": nv_bytes, "int4_bytes": int4_bytes, "fp8_bytes": fp8_bytes},
        "gpu_launches": 8 * args.steps,     # per step: 2 x (2 NVFP4 kernels + 1 INT4 + 1 FP8 kernel)
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_ours(args, wl):
    import torch

    from fp8_block_scaled_pow2_b200 import moe
    from fp8_block_scaled_pow2_b200.layer import MoeLayer

    rank, world, local, pg = dist_setup(args.gpus)
    x, logits, (w13, s13, w2, s2) = make_inputs(wl, args.seed, rank)
    layer = MoeLayer(w13, s13, w2, s2, wl["k"], weights=args.weights, shared=args.shared)
    T = wl["T"]
    buf = layer.alloc(T)
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    ld = torch.from_numpy(logits).cuda()
    stream = torch.cuda.current_stream()
    use_graph = args.graph == "on"
    segs = layer.segments(xd, ld, buf)
    if use_graph:
        # each of the four segments (pre, w1/w3, w2, combine) becomes a CUDA
        # graph, so the GEMM events still fall between replays
        for _ in range(2):
            for f in segs:
                f()
        torch.cuda.synchronize()
        graphs = []
        for f in segs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                f()
            graphs.append(g)
        torch.cuda.synchronize()
        runners = [g.replay for g in graphs]
    else:
        runners = list(segs)

    def step(ev=None, seg=None):
        # ev: events before w1/w3, between the GEMMs and after w2 (timed
        # region); seg: events before every segment and after the last
        for i, run in enumerate(runners):
            if seg:
                seg[i].record(stream)
            if ev and i > 0:
                ev[i - 1].record(stream)
            run()
        if seg:
            seg[len(runners)].record(stream)

    clk = ClockSampler(local).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    ab = algorithmic_bytes(layer, buf, wl)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    torch.cuda.synchronize()
    w_begin = time.time()
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk.mark(w_begin, time.time())
    clk.stop()
    barrier(pg)
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, pg)
    g13 = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    g2 = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    # the pre-GEMM segment and the combine, from a separate untimed pass
    segs_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for i in range(args.steps):
        step(seg=segs_ev[i])
    torch.cuda.synchronize()
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in segs_ev)
    post_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in segs_ev)

    # end to end through the public API with host buffers: every step copies
    # its x and logits from pinned host memory and y back, inside the timed
    # region; StepRunner overlaps those copies with the neighbouring steps'
    # compute on a second stream
    from fp8_block_scaled_pow2_b200.runner import StepRunner, pinned_inputs
    runner = StepRunner(layer, T, graphs=use_graph)
    xh, lh, yh = pinned_inputs(x, logits)
    for _ in range(max(1, args.warmup)):
        runner.submit(xh, lh, yh)
    runner.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(runner.compute)
    runner.h2d.wait_event(e0)
    runner.d2h.wait_event(e0)
    for _ in range(args.steps):
        runner.submit(xh, lh, yh)
    e1.record(runner.d2h)                  # after the last step's y has left
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg)
    assert moe.moe_get_device_error() == 0

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    peaks = read_peaks()
    tokens = T * world * args.steps
    value = tokens / (ms_max / 1e3)
    clocks = clk.summary()
    if args.workload == "decode":
        achieved = ab["w13"] / (g13 / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "traffic": recorded_traffic(args.workload, args.weights),
                "kernel": f"{GEMM_ENTRY[args.weights]} (w1/w3, SwiGLU epilogue)",
                "peak_source": f"{peaks['src']} HBM copy"}
    else:
        fp8_peak = 2.0 * peaks["bf16_sustained"]
        achieved = ab["flops13"] / (g13 / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": round(achieved / fp8_peak, 4), "traffic": recorded_traffic(args.workload, args.weights),
                "kernel": f"{GEMM_ENTRY[args.weights]} (w1/w3, SwiGLU epilogue)",
                "peak_source": f"{peaks['src']} bf16 sustained x 2 (FP8 rate)"}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": {"mxfp4": "e4m3xe2m1->f32", "w4afp8": "e4m3xint4->f32",
                                                                                 "ptpc": "e4m3xe4m3->f32"}[args.weights],
        "data": "synthetic",
        "config": {"workload": f"{args.workload} layer: hidden {wl['H']}, intermediate {wl['I']}, "
                               f"{wl['E']} routed + 1 shared experts, top-{wl['k']}, {T} tokens per GPU",
                   "weights": args.weights, "shared_expert": args.shared,
                   "tokens_per_gpu": T, "parallelism": f"replicas x{world} (data parallel, no collective)",
                   "cuda_graph": use_graph,
                   "l2": f"inputs larger than L2: {ab['active_experts']} active experts stream "
                         f"{(ab['w13'] + ab['w2']) / 1e9:.2f} GB of weights per step"},
        "roofline": roof,
        "gemm": {"w13_ms": round(g13, 4), "w2_ms": round(g2, 4),
                 "w13_GBps": round(ab["w13"] / (g13 / 1e3) / 1e9, 1),
                 "w2_GBps": round(ab["w2"] / (g2 / 1e3) / 1e9, 1),
                 "w13_TFLOPs": round(ab["flops13"] / (g13 / 1e3) / 1e12, 2),
                 "w2_TFLOPs": round(ab["flops2"] / (g2 / 1e3) / 1e12, 2),
                 "active_experts": ab["active_experts"], "rows": ab["rows"]},
        "segments": {"pre_ms": round(pre_ms, 4), "pre_GBps": round(ab["pre"] / (pre_ms / 1e3) / 1e9, 1),
                     "post_ms": round(post_ms, 4), "post_GBps": round(ab["post"] / (post_ms / 1e3) / 1e9, 1),
                     "pre": "quantise + route + group (+ row-scale gather)", "post": "combine",
                     "timing": "CUDA events around each segment, a separate pass of the same steps",
                     "bytes": "algorithmic: each input read once, each output written once"},
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "api": "StepRunner.submit (pinned host x, logits in; y out; copies on their own streams)",
                "h2d_bytes_per_step": int(xh.numel() * 2 + lh.numel() * 4),
                "d2h_bytes_per_step": int(yh.numel() * 2)},
        "gpu_launches": kernels_per_step(wl, args.shared, args.weights) * args.steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline and world == 1:
        # the oracle on the host cores, at N = 1 only (rank 0 is the only rank)
        line["cpu_baseline"] = cpu_baseline(wl, args.seed, budget_s=args.cpu_seconds)
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(wl, seed, budget_s=15.0, tokens_per_step=None):
    """Time the oracle on a bounded sample of tokens (rank 0 only)."""
    import synth
    from oracle import ffn
    x, logits, (w13, s13, w2, s2) = make_inputs(wl, seed, 0)
    n, done, t_used = 0, 0, 0.0
    order = (synth.splitmix64(seed, 99, wl["T"]) % np.uint64(wl["T"])).astype(np.int64)
    t_start = time.perf_counter()
    while t_used < budget_s and done < wl["T"]:
        tok = np.unique(order[done:done + (tokens_per_step or 1)])
        t = time.perf_counter()
        ffn.moe_layer(x, logits, w13, s13, w2, s2, wl["k"], tokens=tok)
        t_used += time.perf_counter() - t
        n += len(tok)
        done += tokens_per_step or 1
    return {"value": round(n / t_used, 4), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} tokens of the {wl['T']}-token batch, one oracle call per token "
                      f"({t_used:.1f} s of CPU work, numpy float64, BLAS threads for the matmuls)",
            "wall_s": round(time.perf_counter() - t_start, 1)}


def run_reference_repack(args, wl):
    """The oracle's repacks on one expert's three matrices per step."""
    import synth
    from oracle import repack as Rp
    E, H, I = wl["E"], wl["H"], wl["I"]
    w13, s13, w2, s2 = synth.expert_weights(args.seed, 1, H, I)
    per = (2 * w13.nbytes + s13.nbytes + 2 * s13.nbytes + 4 * 2) + (2 * w2.nbytes + s2.nbytes + 2 * s2.nbytes + 4) \
        + (2 * w13.nbytes + s13.nbytes + 4 * w13.nbytes * 2 // 128) + (2 * w2.nbytes + s2.nbytes + 4 * w2.nbytes * 2 // 128) \
        + (3 * w13.nbytes + s13.nbytes + 4 * w13.nbytes * 2 // (128 * 128)) \
        + (3 * w2.nbytes + s2.nbytes + 4 * w2.nbytes * 2 // (128 * 128))
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        Rp.repack_mxfp4_to_nvfp4(w13.reshape(2, I, H // 2), s13.reshape(2, I, H // 32))
        Rp.repack_mxfp4_to_nvfp4(w2, s2)
        Rp.repack_mxfp4_to_int4g128(w13.reshape(2, I, H // 2), s13.reshape(2, I, H // 32))
        Rp.repack_mxfp4_to_int4g128(w2, s2)
        Rp.repack_mxfp4_to_fp8_block128(w13.reshape(2, I, H // 2), s13.reshape(2, I, H // 32))
        Rp.repack_mxfp4_to_fp8_block128(w2, s2)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    value = per * len(times) / sum(times) / 1e9
    print(json.dumps({
        "impl": "reference", "metric": "weight repack GB/s vs B200 HBM roofline", "value": round(value, 4),
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": f"repack sweep: {E} experts x (w1, w3 [{I}, {H}], w2 [{H}, {I}]) MXFP4 -> NVFP4, "
                               f"-> INT4 group 128 and -> FP8 E4M3 [128, 128] blocks"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one expert's three matrices per step, {len(times)} steps"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
        flush=True)


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.workload.startswith("repack"):
        return run_reference_repack(args, wl)
    import synth
    from oracle import ffn
    x, logits, (w13, s13, w2, s2) = make_inputs(wl, args.seed, 0)
    order = (synth.splitmix64(args.seed, 99, wl["T"]) % np.uint64(wl["T"])).astype(np.int64)
    times = []
    for i in range(args.warmup + args.steps):
        tok = order[i % wl["T"]:i % wl["T"] + 1]
        t = time.perf_counter()
        ffn.moe_layer(x, logits, w13, s13, w2, s2, wl["k"], tokens=tok)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    total = sum(times)
    value = len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / len(times), 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload} layer: hidden {wl['H']}, intermediate {wl['I']}, "
                               f"{wl['E']} routed + 1 shared experts, top-{wl['k']}, {wl['T']} tokens per GPU",
                   "tokens_per_gpu": wl["T"], "parallelism": "CPU oracle, rank 0 only"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one token of the batch per step, {len(times)} steps"},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--weights", choices=["mxfp4", "w4afp8", "ptpc"], default="mxfp4")
    ap.add_argument("--shared", choices=["mxfp4", "fp8"], default="mxfp4",
                    help="shared expert weights: MXFP4 (group E of the grouped GEMM) or FP8 [128, 128] blocks")
    ap.add_argument("--graph", choices=["on", "off"], default="on",
                    help="replay the layer step as four CUDA graphs (off: eager library calls)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.workload.startswith("repack"):
        run_repack(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
