"""Host-side logic of bench.py, on CPU: the reduction of per-rank times over a
world of 2 gloo processes, the whole-job throughput, the reference arm's
behaviour under a launcher (only rank 0 works and prints), and the computed
FLOP count of a plan against a brute-force count."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank times a different amount; the job takes the slowest rank's
        got = bench.reduce_max_over_ranks([1.0 + rank, 10.0 - rank, 3.5], torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1] == [2.0, 10.0, 3.5]


def test_reduce_max_single_process_is_identity():
    import torch
    assert bench.reduce_max_over_ranks([4.0, 2.5], torch.device("cpu")) == [4.0, 2.5]


def test_job_throughput_is_weak_scaling():
    # two ranks, each 1 TFLOP in the slowest rank's 500 ms -> 4 TFLOP/s for the job
    assert bench.job_throughput(2, 1e12, 500.0) == 4.0
    assert bench.job_throughput(1, 1e12, 500.0) == 2.0


def _run_reference(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                           "tiny", "--steps", "1", "--warmup", "0", "--ref-seconds", "0.2", "--gpus", "2"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_reference(1)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _run_reference(0)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == bench.UNIT
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_plan_flops_matches_brute_force():
    rng = np.random.default_rng(3)
    N, Bk, d = 1000, 64, 128            # 16 key blocks, the last holds 40 rows
    nK = -(-N // Bk)
    offsets = np.array([0, 128, 300, 700, 1000])
    G = len(offsets) - 1
    idx = np.stack([np.stack([rng.choice(nK, 5, replace=False) for _ in range(G)]) for _ in range(2)])[None]
    want = 0.0
    for h in range(2):
        for g in range(G):
            for b in idx[0, h, g]:
                valid = min(Bk, N - b * Bk)
                want += 4.0 * d * valid * (offsets[g + 1] - offsets[g])
    assert bench.plan_flops(idx, offsets, N, Bk, d) == want


def test_oracle_samples_of_the_widening_stages():
    # the CPU baselines of the layout build and the top-p stage: bounded samples of
    # the oracle, reported with the threads they used
    rng = np.random.default_rng(0)
    x = (rng.normal(size=(1, 1, 600, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    c = bench.cpu_cluster_sample(x, 16, 2, target_s=0.2)
    assert c["kind"] == "oracle" and c["cores"] == 1 and c["value"] > 0 and "600 tokens" in c["sample"]
    m = np.exp(rng.normal(size=(1, 2, 30, 100))).astype(np.float32)
    t = bench.cpu_top_p_sample(m, 0.5, 12, 0, target_s=0.2)
    assert t["kind"] == "oracle" and t["unit"] == "plan rows/s" and t["value"] > 0 and "30 of 30" in t["sample"]


def test_roofline_peak_choice():
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    # a short timed region is held against the burst figure
    assert bench.roofline_peak(peaks, 300.0, {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0}) == (1600.0, "burst")
    # a long one at full clock too; a long one below it against the sustained figure
    assert bench.roofline_peak(peaks, 5000.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}) == (1600.0, "burst")
    assert bench.roofline_peak(peaks, 5000.0, {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0}) == (1400.0, "sustained")
    assert bench.roofline_peak(peaks, 5000.0, None) == (1400.0, "sustained")
