"""Benchmark of the routed-expert MoE layer (MXFP4 experts, FP8 activations).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long_prefill|decode|prefill|repack|decode_small|prefill_small|repack_small]
                    [--weights mxfp4|w4afp8|ptpc] [--shared mxfp4|fp8] [--extras default|none]

A step is one pass of the whole expert path (quantise, route, group, w1/w3
GEMM + SwiGLU + requantise, w2 GEMM, combine) over one batch of synthetic
tokens.  The default workload is the largest layer that fits one GPU: the
long-prefill layer of a DeepSeek-V4-Flash-class model with 384 routed + 1
shared experts (hidden 4096, expert intermediate 2048, top-6), 16384 tokens
of N(0,1) activations with 0.1% outliers x20, router logits biased so that
expert loads follow Zipf(1.1), MXFP4 experts from N(0, 0.02).  The same run
also times, each under its own key of the JSON line, the decode layer (256 +
1 experts, 64 tokens, uniform logits), the prefill layer (4096 tokens, Zipf)
and the long-prefill layer on the W4AFP8 path.  Each rank runs its own
replica on its own tokens (data parallel, no collective on the data path);
`value` is the tokens of all ranks divided by the slowest rank's device time.

One JSON line is printed by rank 0.  `--impl reference` times the CPU oracle
(rank 0 only, one thread) on a bounded sample of the same workload.
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
GEMM_SOURCES = {"mxfp4": ("common.cuh", "gemm_mxfp4.cuh", "gemm_pair.cuh", "sm100.cuh"),
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


def make_inputs(wl: dict, seed: int, rank: int, rows=None):
    """Activations, router logits and the expert weights of one workload;
    the weights as synth.RepeatedExperts views (expert e holds prototype e % 4).
    rows: only these tokens of the batch (their x and logits rows)."""
    import synth
    T, H, I, E = wl["T"], wl["H"], wl["I"], wl["E"]
    views = synth.expert_views(seed, E + 1, H, I, n_proto=4)
    x = synth.decode_activations(seed + 1000 * rank, T, H, rows=rows)
    logits = (synth.uniform_logits if wl["logits"] == "uniform" else synth.zipf_logits)(seed + 1000 * rank, T, E)
    return x, (logits if rows is None else logits[rows]), views


def on_device(view):
    """A RepeatedExperts view expanded to the full [E1, ...] array on the GPU
    (every expert in its own memory), from one upload of the prototypes."""
    import torch
    protos = torch.from_numpy(np.ascontiguousarray(view.protos)).cuda()
    return protos[torch.arange(view.shape[0], device="cuda") % protos.shape[0]].contiguous()


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

    def summary(self, window=None):
        window = window or self.window
        if self.proc is None or window is None or not os.path.exists(self.path):
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
        b, e = window
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
    w13, s13, w2, s2 = (on_device(v) for v in synth.expert_views(args.seed, E, H, I, n_proto=4))
    # w1 and w3 are separate [I, H] matrices: view w13 [E, 2I, H/2] as [2E, I, H/2]
    mats = [(w13.reshape(2 * E, I, H // 2), s13.reshape(2 * E, I, H // 32)), (w2, s2)]
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
    # end to end from host memory: every step copies the MXFP4 weights in from
    # pinned host memory and every repack's outputs back, inside the timed
    # region, in chunks of matrices pipelined over an upload stream, the
    # compute stream and a download stream (double-buffered on the device)
    e2e_ms, h2d_b, d2h_b = repack_e2e(mats, outs, args.steps, pg)
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
        "e2e": {"value": round((nv_bytes + int4_bytes + fp8_bytes) * world * args.steps / (e2e_ms / 1e3) / 1e9, 1),
                "unit": "GB/s", "api": "the three repack entry points on chunks of matrices, pinned host source "
                                       "in and every output back, copies on their own streams",
                "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b},
        "gpu_launches": 8 * args.steps,     # per step: 2 x (2 NVFP4 kernels + 1 INT4 + 1 FP8 kernel)
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        w13, s13, w2, s2 = synth.expert_weights(args.seed, 1, H, I)
        times, threads = reference_repack_times(w13, s13, w2, s2, H, I, 4)
        v = repack_bytes_per_expert(H, I) * 3 / sum(times[1:]) / 1e9
        line["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": "the oracle's three repacks of one expert's w1, w3, w2, three times "
                                          f"after one untimed pass ({sum(times[1:]):.1f} s, one thread)",
                                "host": host_info()}
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def repack_e2e(mats, outs, steps: int, pg, chunk_bytes: int = 256 << 20):
    """Repack steps from pinned host memory: returns (ms for `steps` steps,
    host-to-device bytes per step, device-to-host bytes per step)."""
    import torch

    from fp8_block_scaled_pow2_b200 import moe
    names = ("nv_fp4", "nv_s", "nv_g", "q", "sinv", "f8", "f8_s")
    host_in = [(fp4.cpu().pin_memory(), e8.cpu().pin_memory()) for fp4, e8 in mats]
    host_out = [{n: torch.empty(o[n].shape, dtype=o[n].dtype, pin_memory=True) for n in names} for o in outs]
    h2d_b = sum(a.numel() + b.numel() for a, b in host_in)
    d2h_b = sum(t.numel() * t.element_size() for o in host_out for t in o.values())
    compute = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    # chunks of whole matrices; each set's device arrays serve as two slots
    # (their first and second halves), or one slot for a set of one matrix
    plan = []
    for si, (fp4, e8) in enumerate(mats):
        per = fp4[0].numel() * 8
        n_slots = 2 if fp4.shape[0] >= 2 else 1
        c = max(1, min(fp4.shape[0] // n_slots, chunk_bytes // per))
        for i, m0 in enumerate(range(0, fp4.shape[0], c)):
            b = i % n_slots
            plan.append((si, b, m0, min(fp4.shape[0], m0 + c), b * (fp4.shape[0] // 2)))
    # per (set, slot): inputs uploaded, repacks done, outputs downloaded
    ev = {(si, b): [torch.cuda.Event() for _ in range(3)] for si in range(len(mats)) for b in range(2)}
    for e in ev.values():
        e[1].record(compute)
        e[2].record(compute)

    def step():
        for si, b, m0, m1, d0 in plan:
            fp4, e8 = mats[si]
            o = outs[si]
            in_ready, done, out_free = ev[(si, b)]
            sl = slice(d0, d0 + (m1 - m0))
            with torch.cuda.stream(up):
                up.wait_event(done)                              # the slot's last repack has read its inputs
                fp4[sl].copy_(host_in[si][0][m0:m1], non_blocking=True)
                e8[sl].copy_(host_in[si][1][m0:m1], non_blocking=True)
                in_ready.record(up)
            compute.wait_event(in_ready)
            compute.wait_event(out_free)                         # the slot's last outputs have left
            moe.repack_mxfp4_to_nvfp4(fp4[sl], e8[sl], o["nv_fp4"][sl], o["nv_s"][sl], o["nv_g"][sl])
            moe.repack_mxfp4_to_int4g128(fp4[sl], e8[sl], o["q"][sl], o["sinv"][sl])
            moe.repack_mxfp4_to_fp8_block128(fp4[sl], e8[sl], o["f8"][sl], o["f8_s"][sl])
            done.record(compute)
            with torch.cuda.stream(down):
                down.wait_event(done)
                for n in names:
                    host_out[si][n][m0:m1].copy_(o[n][sl], non_blocking=True)
                out_free.record(down)

    step()
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    up.wait_event(e0)
    down.wait_event(e0)
    for _ in range(steps):
        step()
    down.wait_stream(compute)
    e1.record(down)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    return max_over_ranks(e0.elapsed_time(e1), pg), h2d_b, d2h_b


def roofline(wl: dict, weights: str, ab: dict, g13_ms: float, peaks: dict, workload: str) -> dict:
    """Roofline of the dominant kernel, the w1/w3 GEMM with its SwiGLU
    epilogue: decode-sized batches stream the weights (HBM bound, measured
    copy bandwidth); larger batches are tensor bound, against the FP8 rate
    of the block-scaled MMA taken as 2 x the measured burst bf16 rate (the
    GEMM runs in short launches, not a seconds-long loop)."""
    kernel = f"{GEMM_ENTRY[weights]} (w1/w3, SwiGLU epilogue)"
    traffic = recorded_traffic(workload, weights)
    if wl["T"] <= 256:
        achieved = ab["w13"] / (g13_ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "traffic": traffic, "kernel": kernel,
                "peak_source": f"{peaks['src']} HBM copy (burst)"}
    fp8_peak = round(2.0 * peaks["bf16"], 1)
    achieved = ab["flops13"] / (g13_ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": fp8_peak, "unit": "TFLOP/s",
            "frac": round(achieved / fp8_peak, 4), "traffic": traffic, "kernel": kernel,
            "peak_source": f"{peaks['src']} bf16 burst x 2 (FP8 rate of the block-scaled MMA, nominal ratio)"}


def workload_name(name: str, wl: dict) -> str:
    return (f"{name} layer: hidden {wl['H']}, intermediate {wl['I']}, {wl['E']} routed + 1 shared experts, "
            f"top-{wl['k']}, {wl['T']} tokens per GPU, "
            + ("uniform router logits" if wl["logits"] == "uniform" else "Zipf(1.1) expert loads"))


def bench_layer(args, name: str, weights: str, shared: str, steps: int, warmup: int, rank: int, pg, clk,
                with_e2e: bool) -> dict:
    """Time `steps` layer steps of one workload (CUDA events on the launching
    stream, between barriers), per-GEMM event times, the pre-GEMM segment and
    the combine in a separate pass, and optionally the end-to-end rate from
    pinned host buffers.  Returns the figures; frees the layer."""
    import torch

    from fp8_block_scaled_pow2_b200 import moe
    from fp8_block_scaled_pow2_b200.layer import MoeLayer

    wl = WORKLOADS[name]
    x, logits, views = make_inputs(wl, args.seed, rank)
    layer = MoeLayer(*(on_device(v) for v in views), wl["k"], weights=weights, shared=shared)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    T = wl["T"]
    buf = layer.alloc(T, args.block_n)
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    ld = torch.from_numpy(logits).cuda()
    stream = torch.cuda.current_stream()
    use_graph = args.graph == "on"
    segs = layer.segments(xd, ld, buf)
    graphs = []
    if use_graph:
        # each of the four segments (pre, w1/w3, w2, combine) becomes a CUDA
        # graph, so the GEMM events still fall between replays
        for _ in range(2):
            for f in segs:
                f()
        torch.cuda.synchronize()
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

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    ab = algorithmic_bytes(layer, buf, wl)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    torch.cuda.synchronize()
    w_begin = time.time()
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    window = (w_begin, time.time())
    barrier(pg)
    ms_max = max_over_ranks(t0.elapsed_time(t1), pg)
    g13 = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    g2 = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    # the pre-GEMM segment and the combine, from a separate untimed pass
    segs_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for i in range(steps):
        step(seg=segs_ev[i])
    torch.cuda.synchronize()
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in segs_ev)
    post_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in segs_ev)

    e2e = None
    if with_e2e:
        # end to end through the public API with host buffers: every step copies
        # its x and logits from pinned host memory and y back, inside the timed
        # region; StepRunner overlaps those copies with the neighbouring steps'
        # compute on a second stream
        from fp8_block_scaled_pow2_b200.runner import StepRunner, pinned_inputs
        runner = StepRunner(layer, T, block_n=args.block_n, graphs=use_graph, input_sets=args.input_sets)
        xh, lh, yh = pinned_inputs(x, logits)
        for _ in range(max(1, warmup)):
            runner.submit(xh, lh, yh)
        runner.synchronize()
        barrier(pg)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(runner.compute)
        runner.h2d.wait_event(e0)
        runner.d2h.wait_event(e0)
        for _ in range(steps):
            runner.submit(xh, lh, yh)
        e1.record(runner.d2h)                  # after the last step's y has left
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg)
        e2e = {"ms": e2e_ms, "h2d_bytes_per_step": int(xh.numel() * 2 + lh.numel() * 4),
               "d2h_bytes_per_step": int(yh.numel() * 2)}
        runner.close()
    assert moe.moe_get_device_error() == 0
    graphs.clear()
    del layer, buf, xd, ld
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return dict(wl=wl, T=T, ms_max=ms_max, g13=g13, g2=g2, pre_ms=pre_ms, post_ms=post_ms, ab=ab, e2e=e2e,
                window=window, graph=use_graph)


def layer_fields(name: str, weights: str, shared: str, r: dict, steps: int, world: int, peaks: dict,
                 clk) -> dict:
    """The figures of one timed workload as JSON fields."""
    ab, wl = r["ab"], r["wl"]
    tokens = r["T"] * world * steps
    return {
        "workload": workload_name(name, wl), "weights": weights, "shared_expert": shared,
        "value": round(tokens / (r["ms_max"] / 1e3), 2), "unit": "tokens/s",
        "ms_per_step": round(r["ms_max"] / steps, 4),
        "roofline": roofline(wl, weights, ab, r["g13"], peaks, name),
        "gemm": {"w13_ms": round(r["g13"], 4), "w2_ms": round(r["g2"], 4),
                 "w13_GBps": round(ab["w13"] / (r["g13"] / 1e3) / 1e9, 1),
                 "w2_GBps": round(ab["w2"] / (r["g2"] / 1e3) / 1e9, 1),
                 "w13_TFLOPs": round(ab["flops13"] / (r["g13"] / 1e3) / 1e12, 2),
                 "w2_TFLOPs": round(ab["flops2"] / (r["g2"] / 1e3) / 1e12, 2),
                 "active_experts": ab["active_experts"], "rows": ab["rows"]},
        "segments": {"pre_ms": round(r["pre_ms"], 4), "pre_GBps": round(ab["pre"] / (r["pre_ms"] / 1e3) / 1e9, 1),
                     "post_ms": round(r["post_ms"], 4),
                     "post_GBps": round(ab["post"] / (r["post_ms"] / 1e3) / 1e9, 1),
                     "pre": "quantise + route + group (+ row-scale gather)", "post": "combine",
                     "timing": "CUDA events around each segment, a separate pass of the same steps",
                     "bytes": "algorithmic: each input read once, each output written once"},
        "l2": f"inputs larger than L2: {ab['active_experts']} active experts stream "
              f"{(ab['w13'] + ab['w2']) / 1e9:.2f} GB of weights per step",
        "clocks": clk.summary(r["window"]),
    }


# extra workloads timed in the same run as the default one, each under its own key
DEFAULT_EXTRAS = (("decode", "mxfp4"), ("prefill", "mxfp4"), ("long_prefill", "w4afp8"))


def run_ours(args, wl):
    import torch

    rank, world, local, pg = dist_setup(args.gpus)
    clk = ClockSampler(local).start()
    r = bench_layer(args, args.workload, args.weights, args.shared, args.steps, args.warmup, rank, pg, clk,
                    with_e2e=True)
    extras = []
    if args.extras == "default" and args.workload == "long_prefill" and args.weights == "mxfp4":
        extras = list(DEFAULT_EXTRAS)
    extra_results = []
    for name, weights in extras:
        extra_results.append((name, weights, bench_layer(args, name, weights, "mxfp4", args.steps, args.warmup,
                                                         rank, pg, clk, with_e2e=False)))
    clk.stop()
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    peaks = read_peaks()
    main = layer_fields(args.workload, args.weights, args.shared, r, args.steps, world, peaks, clk)
    tokens = r["T"] * world * args.steps
    line = {
        "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"mxfp4": "e4m3xe2m1->f32", "w4afp8": "e4m3xint4->f32", "ptpc": "e4m3xe4m3->f32"}[args.weights],
        "data": "synthetic",
        "config": {"workload": main["workload"], "weights": args.weights, "shared_expert": args.shared,
                   "tokens_per_gpu": r["T"], "parallelism": f"replicas x{world} (data parallel, no collective)",
                   "cuda_graph": r["graph"], "l2": main["l2"]},
        "roofline": main["roofline"],
        "gemm": main["gemm"],
        "segments": main["segments"],
        "e2e": {"value": round(tokens / (r["e2e"]["ms"] / 1e3), 2), "unit": "tokens/s",
                "api": "StepRunner.submit (pinned host x, logits in; y out; copies on their own streams; "
                       f"{args.input_sets} device input set(s))",
                "h2d_bytes_per_step": r["e2e"]["h2d_bytes_per_step"],
                "d2h_bytes_per_step": r["e2e"]["d2h_bytes_per_step"]},
        "gpu_launches": kernels_per_step(r["wl"], args.shared, args.weights) * args.steps,
        "clocks": main["clocks"],
    }
    for name, weights, rr in extra_results:
        key = name if weights == "mxfp4" else f"{name}_{weights}"
        line[key] = layer_fields(name, weights, "mxfp4", rr, args.steps, world, peaks, clk)
    if not args.no_cpu_baseline and world == 1:
        # the oracle on the host cores, at N = 1 only (rank 0 is the only rank)
        line["cpu_baseline"] = cpu_baseline(wl, args.seed, budget_s=args.cpu_seconds)
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def host_info() -> dict:
    """Host core count and CPU model (for the CPU-baseline record)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def one_thread():
    """Context that holds BLAS (and OpenMP) pools to one thread: the oracle
    baseline is timed single-threaded."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:                      # threadpoolctl missing: numpy's own default
        import contextlib
        return contextlib.nullcontext()


def sample_order(wl: dict, seed: int, n: int) -> np.ndarray:
    """The seeded order in which the oracle legs visit the batch's tokens."""
    import synth
    return (synth.splitmix64(seed, 99, n) % np.uint64(wl["T"])).astype(np.int64)


def cpu_baseline(wl, seed, budget_s=15.0):
    """Time the oracle on a bounded sample of tokens (rank 0 only), one thread,
    one oracle call per token (tokens are independent given the routing)."""
    from oracle import ffn
    order = sample_order(wl, seed, min(wl["T"], 256))
    x, logits, (w13, s13, w2, s2) = make_inputs(wl, seed, 0, rows=order)
    n, t_used = 0, 0.0
    t_start = time.perf_counter()
    with one_thread():
        threads = blas_threads()
        while t_used < budget_s and n < len(order):
            t = time.perf_counter()
            ffn.moe_layer(x[n:n + 1], logits[n:n + 1], w13, s13, w2, s2, wl["k"])
            t_used += time.perf_counter() - t
            n += 1
    return {"value": round(n / t_used, 4), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} tokens of the {wl['T']}-token batch, one oracle call per token "
                      f"({t_used:.1f} s of CPU work, numpy float64 on one thread)",
            "host": host_info(), "wall_s": round(time.perf_counter() - t_start, 1)}


def repack_bytes_per_expert(H: int, I: int) -> int:
    """Algorithmic bytes of the three repacks of one expert (w1, w3 [I, H] and
    w2 [H, I]): each reads its MXFP4 source once and writes its outputs once."""
    nib = 3 * I * H // 2                   # packed nibbles of the three matrices
    e8 = 3 * I * H // 32                   # E8M0 scales
    nv = 2 * nib + e8 + 2 * e8 + 4 * 3     # nibble copy + scales in, E4M3 /16 scales + globals out
    i4 = 2 * nib + e8 + 4 * (3 * I * H // 128)
    f8 = nib + e8 + 2 * nib + 4 * (3 * I * H // (128 * 128))
    return nv + i4 + f8


def reference_repack_times(w13, s13, w2, s2, H, I, n):
    """The oracle's three repacks of one expert, n times, on one thread."""
    from oracle import repack as Rp
    times = []
    with one_thread():
        threads = blas_threads()
        for _ in range(n):
            t = time.perf_counter()
            Rp.repack_mxfp4_to_nvfp4(w13.reshape(2, I, H // 2), s13.reshape(2, I, H // 32))
            Rp.repack_mxfp4_to_nvfp4(w2, s2)
            Rp.repack_mxfp4_to_int4g128(w13.reshape(2, I, H // 2), s13.reshape(2, I, H // 32))
            Rp.repack_mxfp4_to_int4g128(w2, s2)
            Rp.repack_mxfp4_to_fp8_block128(w13.reshape(2, I, H // 2), s13.reshape(2, I, H // 32))
            Rp.repack_mxfp4_to_fp8_block128(w2, s2)
            times.append(time.perf_counter() - t)
    return times, threads


def run_reference_repack(args, wl):
    """The oracle's repacks on one expert's three matrices per step."""
    import synth
    from oracle import repack as Rp
    E, H, I = wl["E"], wl["H"], wl["I"]
    w13, s13, w2, s2 = synth.expert_weights(args.seed, 1, H, I)
    per = repack_bytes_per_expert(H, I)
    times, threads = reference_repack_times(w13, s13, w2, s2, H, I, args.warmup + args.steps)
    times = times[args.warmup:]
    value = per * len(times) / sum(times) / 1e9
    print(json.dumps({
        "impl": "reference", "metric": "weight repack GB/s vs B200 HBM roofline", "value": round(value, 4),
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": f"repack sweep: {E} experts x (w1, w3 [{I}, {H}], w2 [{H}, {I}]) MXFP4 -> NVFP4, "
                               f"-> INT4 group 128 and -> FP8 E4M3 [128, 128] blocks"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"one expert's three matrices per step, {len(times)} steps, one thread",
                         "host": host_info()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
        flush=True)


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.workload.startswith("repack"):
        return run_reference_repack(args, wl)
    from oracle import ffn
    order = sample_order(wl, args.seed, args.warmup + args.steps)
    x, logits, (w13, s13, w2, s2) = make_inputs(wl, args.seed, 0, rows=order)
    times = []
    with one_thread():
        threads = blas_threads()
        for i in range(args.warmup + args.steps):
            t = time.perf_counter()
            ffn.moe_layer(x[i:i + 1], logits[i:i + 1], w13, s13, w2, s2, wl["k"])
            if i >= args.warmup:
                times.append(time.perf_counter() - t)
    total = sum(times)
    value = len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / len(times), 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(args.workload, wl),
                   "tokens_per_gpu": wl["T"], "parallelism": "CPU oracle, rank 0 only"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"one token of the batch per step, {len(times)} steps, one thread",
                         "host": host_info()},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="long_prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--weights", choices=["mxfp4", "w4afp8", "ptpc"], default="mxfp4")
    ap.add_argument("--shared", choices=["mxfp4", "fp8"], default="mxfp4",
                    help="shared expert weights: MXFP4 (group E of the grouped GEMM) or FP8 [128, 128] blocks")
    ap.add_argument("--graph", choices=["on", "off"], default="on",
                    help="replay the layer step as four CUDA graphs (off: eager library calls)")
    ap.add_argument("--block-n", type=int, default=0,
                    help="token rows per GEMM tile (0: the library's choice)")
    ap.add_argument("--input-sets", type=int, default=2, choices=[1, 2],
                    help="device copies of the step inputs in the host-buffer (e2e) runs")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extras", choices=["default", "none"], default="default",
                    help="with the default workload, also time decode, prefill and the W4AFP8 long prefill "
                         "(each under its own key of the JSON line)")
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
