"""Host-side logic of bench.py without a GPU: argument rules, the
max-over-ranks timing with two gloo ranks, the JSON line of the reference
arm, and the roofline bookkeeping."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    bench.barrier(dist)
    v = bench.max_over_ranks(10.0 + 5.0 * rank, dist)
    q.put((rank, v))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_warmup_rule():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_reference_arm_line_on_cpu():
    """The reference arm is the CPU oracle; rank 0 prints one JSON line."""
    env = dict(os.environ, PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, PYTHONPATH=ROOT, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_peaks_and_traffic_bookkeeping(tmp_path):
    p = bench.read_peaks()
    assert p["hbm"] > 1000 and p["bf16"] > 100
    assert bench.source_digest("mxfp4") != bench.source_digest("w4afp8")


def test_roofline_bookkeeping_decode_and_prefill():
    """Decode-sized batches are reported against the measured HBM copy rate,
    larger ones against 2 x the measured burst bf16 rate (the FP8 MMA rate)."""
    peaks = {"hbm": 6548.2, "bf16": 1642.8, "bf16_sustained": 1402.8, "src": "measured"}
    ab = {"w13": 1.7e9, "flops13": 9.62e11}
    r = bench.roofline(bench.WORKLOADS["decode"], "mxfp4", ab, 0.27, peaks, "decode")
    assert r["bound"] == "hbm" and r["peak"] == 6548.2 and abs(r["achieved"] - 1.7e9 / 0.27e-3 / 1e9) < 0.1
    r = bench.roofline(bench.WORKLOADS["long_prefill"], "mxfp4", ab, 0.5, peaks, "long_prefill")
    assert r["bound"] == "tensor" and r["peak"] == 3285.6 and abs(r["frac"] - 9.62e11 / 0.5e-3 / 1e12 / 3285.6) < 1e-4


def test_default_workload_is_the_largest_layer():
    """With no arguments the benchmark times the long-prefill layer (384 + 1
    experts, 16384 tokens), the largest configuration that fits one GPU."""
    seen = {}

    def fake(args, wl):
        seen["workload"], seen["extras"] = args.workload, args.extras

    orig = bench.run_ours
    bench.run_ours = fake
    try:
        bench.main([])
    finally:
        bench.run_ours = orig
    assert seen == {"workload": "long_prefill", "extras": "default"}
    wl = bench.WORKLOADS["long_prefill"]
    assert (wl["T"], wl["E"], wl["H"], wl["I"], wl["k"]) == (16384, 384, 4096, 2048, 6)


def test_repack_byte_count_matches_the_per_matrix_sum():
    """The reference arm's bytes per expert equal the GPU line's per-matrix
    sums for one expert (w1, w3 [I, H], w2 [H, I])."""
    H, I = 4096, 2048
    total = 0
    for M, N, K in ((2, I, H), (1, H, I)):
        fp4, e8 = M * N * K // 2, M * N * K // 32
        total += 2 * fp4 + e8 + 2 * e8 + 4 * M                     # NVFP4
        total += fp4 + e8 + fp4 + 4 * (M * N * K // 128)             # INT4
        total += fp4 + e8 + 2 * fp4 + 4 * (M * (N // 128) * (K // 128))   # FP8 blocks
    assert bench.repack_bytes_per_expert(H, I) == total
