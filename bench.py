"""Benchmark of the importance-sampled block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan14_10]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed on host cores

One step = the whole hot path on one attention layer: isa_score -> isa_select
-> isa_attention, inputs resident in HBM.  Prints one JSON line (rank 0).

value        computed TFLOP/s of the step: the attention FLOPs the plan makes
             the kernel compute (4 d per query row per selected valid key row,
             padding excluded) divided by the step time.
ms_per_step  milliseconds per call of the whole path.
roofline     the attention kernel (dominant): computed FLOPs per launch / its
             event-timed duration, against the measured bf16 tensor peak
             (burst for a short timed region at full clock, else sustained).
e2e          the same metric through isa_pipeline_host: pinned host Q/K/V in,
             host O out, copies inside the timed region.
plan_reuse_ms_per_call
             ms per attention call when one plan serves r calls, r = 1, 2, 4,
             8: a timed loop of (score + select once, then r attention calls on
             activations that change from call to call).
Multi-GPU: one process per GPU (torchrun); every rank runs its own layer
(weak scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse IS-attention ms/call + computed TFLOP/s vs B200 BF16 peak, per shape"
UNIT = "TFLOP/s (computed)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch, per head, from an ncu capture of the wan14_10 layer cut to 4 heads.
# Q, K, V and O all scale with the head count.  The figure holds only for the
# kernel source whose code (comments and blank lines removed) has a SHA-256
# starting with the recorded prefix; for any other source (or workload) the
# roofline reports traffic as null.
ATTN_TRAFFIC = {"workload": "wan14_10", "src_sha256_prefix": "8598bc353feff525", "bytes_per_head": 308.4e6 / 4}


def attn_code_digest(text: str) -> str:
    """SHA-256 of a CUDA source with // comments and blank lines removed."""
    import hashlib
    import re
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def attn_traffic(workload, heads):
    import hashlib
    src = os.path.join(ROOT, "block_sparse_importance_b200", "csrc", "attn.cu")
    try:
        with open(src) as f:
            code = attn_code_digest(f.read())
    except OSError:
        return None
    sha = code
    if workload != ATTN_TRAFFIC["workload"] or not sha.startswith(ATTN_TRAFFIC["src_sha256_prefix"]):
        return None
    return ATTN_TRAFFIC["bytes_per_head"] * heads


def reduce_max_over_ranks(values, device):
    """Max of each value over all ranks (identity with one process): the job's
    time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job TFLOP/s: every rank computes its own layer (weak scaling), so
    the job does world x flops_per_rank in the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def roofline_peak(peaks, timed_ms: float, clocks):
    """The bf16 peak a kernel timed in this run is held against: the burst
    figure (a short cuBLAS loop at full clock) when the timed region is short
    (< 2 s) or the sampled SM clock stayed at its maximum; the sustained
    figure (seconds of back-to-back GEMMs under the power cap) otherwise."""
    burst = float(peaks.get("bf16_tflops"))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    sm, mx = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    at_max = sm is not None and mx and sm >= 0.97 * mx
    if timed_ms < 2000.0 or at_max:
        return burst, "burst"
    return sustained, "sustained"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def plan_flops(idx: np.ndarray, offsets: np.ndarray, N: int, Bk: int, d: int) -> float:
    """Computed attention FLOPs of a plan: 4 d per (query row, selected valid key row)."""
    L = np.minimum(Bk, N - np.arange(-(-N // Bk)) * Bk)           # valid rows of each key block
    keys = L[idx].sum(axis=-1).astype(np.float64)                   # [B, H, G]
    rows = np.diff(offsets).astype(np.float64)                      # [G]
    return float(4.0 * d * (keys * rows[None, None, :]).sum())


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_query_id(dev) -> str:
    """nvidia-smi id of the torch device (its UUID when torch exposes it)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    if vis:
        return vis.split(",")[dev.index or 0]
    return str(dev.index or 0)


def cpu_oracle_sample(w, inp, target_s: float = 12.0):
    """Time the oracle (score -> select -> attention) on the first groups of
    head 0, growing the sample until it takes about `target_s` seconds."""
    import oracle
    from block_sparse_importance_b200 import workloads as wl
    q = wl.bf16_bits(inp.q[:, :1])
    k = wl.bf16_bits(inp.k[:, :1])
    v = wl.bf16_bits(inp.v[:, :1])
    off = inp.offsets
    G = len(off) - 1
    N, d = q.shape[2], q.shape[3]

    def run(n_groups):
        sub = off[:n_groups + 1]
        t0 = time.perf_counter()
        mass, _, _, _ = oracle.score(q, k, sub, w.k_block, w.n_clusters, w.n_iters, w.scale)
        idx, lw, _ = oracle.select(mass.astype(np.float32), w.n_exact, w.n_sample, w.seed)
        oracle.attention(q, k, v, sub, w.k_block, idx, lw, w.scale, [(0, 0, g) for g in range(n_groups)])
        dt = time.perf_counter() - t0
        return dt, plan_flops(idx, sub, N, w.k_block, d)

    n = min(G, 2)
    dt, fl = run(n)
    while dt < target_s / 4 and n < G:
        n = min(G, max(n + 1, int(n * min(8.0, target_s / max(dt, 1e-3)))))
        dt, fl = run(n)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "head 0, first %d of %d query groups of %s: oracle score+select+attention (fp64), %.1f s"
                      % (n, G, w.name, dt)}


def cpu_cluster_sample(x_head, n_clusters: int, rounds: int, target_s: float = 6.0):
    """Time the oracle's token clustering (fp64) of the first rows of one head,
    growing the sample until it takes about `target_s` seconds; the rate is in
    the distance products' TFLOP/s (2 n C d per round)."""
    import oracle
    N, d = x_head.shape[-2], x_head.shape[-1]

    def run(n):
        t0 = time.perf_counter()
        oracle.cluster_tokens(x_head[..., :n, :], min(n_clusters, n), rounds)
        return time.perf_counter() - t0

    n = min(N, 2048)
    dt = run(n)
    while dt < target_s / 4 and n < N:
        n = min(N, max(n + 1, int(n * min(8.0, target_s / max(dt, 1e-3)))))
        dt = run(n)
    flops = 2.0 * n * min(n_clusters, n) * d * rounds
    # the oracle parallelises over (batch, head): one head runs on one thread
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s (computed)", "cores": 1,
            "kind": "oracle",
            "sample": "head 0 of Q, first %d of %d tokens, %d clusters, %d rounds: oracle clustering (fp64), %.1f s"
                      % (n, N, min(n_clusters, n), rounds, dt)}


def cpu_top_p_sample(mass_np, p: float, S: int, seed: int, target_s: float = 3.0):
    """Time the oracle's top-p selector on the first plan rows of head 0."""
    import oracle
    G = mass_np.shape[2]

    def run(g):
        t0 = time.perf_counter()
        oracle.select_top_p(mass_np[:, :1, :g], p, S, seed)
        return time.perf_counter() - t0

    g = min(G, 16)
    dt = run(g)
    while dt < target_s / 4 and g < G:
        g = min(G, max(g + 1, int(g * min(8.0, target_s / max(dt, 1e-3)))))
        dt = run(g)
    # a whole head that takes less than the target is repeated until it does
    reps = 1
    while dt * reps < target_s / 4:
        reps *= 2
    if reps > 1:
        t0 = time.perf_counter()
        for _ in range(reps):
            run(g)
        dt = (time.perf_counter() - t0) / reps
    return {"value": g / dt, "unit": "plan rows/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "head 0, first %d of %d plan rows, %d repetitions: oracle top-p selector, %.2f s"
                      % (g, G, reps, dt * reps)}


def time_plan_reuse(isa, ctx, stream, w, lay, q, k, v, mass, idx, lw, out, sws, aws, rs=(1, 2, 4, 8), calls=8):
    """ms per attention call when one plan serves r calls, measured: each cycle
    runs isa_score and isa_select once on the current activations and then r
    isa_attention calls, alternating between the activations and a perturbed
    copy (x + 0.05 N(0, 1), in bf16), as consecutive denoising steps would
    present them.  Every r runs the same number of attention calls (`calls`,
    calls / r cycles) after the same idle pause, so that each loop meets the
    GPU at the same clock and power state; events bracket the loop."""
    import torch
    gen = torch.Generator(device=q.device)
    gen.manual_seed(1234)
    alt = [(q, k, v)]
    alt.append(tuple((t.float() + 0.05 * torch.randn(t.shape, generator=gen, device=t.device)).to(t.dtype)
                     for t in (q, k, v)))
    res = {}
    for r in rs:
        def cycle():
            qa, ka, _ = alt[0]
            isa.score(qa, ka, lay, w.n_clusters, w.n_iters, mass=mass, workspace=sws, ctx=ctx)
            isa.select(mass, lay, w.n_exact, w.n_sample, w.seed, idx=idx, log_w=lw, ctx=ctx)
            for j in range(r):
                qa, ka, va = alt[j % 2]
                isa.attention(qa, ka, va, idx, lw, lay, out=out, workspace=aws, ctx=ctx)
        cycle()
        torch.cuda.synchronize()
        time.sleep(0.5)
        cycles = max(1, calls // r)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(cycles):
            cycle()
        e1.record(stream)
        torch.cuda.synchronize()
        res[str(r)] = e0.elapsed_time(e1) / (cycles * r)
    st = ctx.sync_status()
    if st != isa.ISA_OK:
        raise RuntimeError("device status after the plan-reuse loop: %s" % isa.status_string(st))
    del alt
    return res


def reference_arm(args):
    """--impl reference: the fp64 oracle on the host cores, bounded samples."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from block_sparse_importance_b200 import workloads as wl
    w = wl.preset(args.workload)
    inp = wl.make_inputs(w, "cpu", heads=1)
    vals = []
    for _ in range(args.warmup):
        cpu_oracle_sample(w, inp, target_s=2.0)
    for _ in range(args.steps):
        vals.append(cpu_oracle_sample(w, inp, target_s=args.ref_seconds))
    v = statistics.median(x["value"] for x in vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[-1]["cores"], "kind": "oracle",
                             "sample": vals[-1]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "heads": w.heads, "head_dim": w.head_dim, "seq_len": w.seq_len,
            "grid": list(w.grid), "q_block": w.q_block, "k_block": w.k_block, "n_exact": w.n_exact,
            "n_sample": w.n_sample, "n_clusters": w.n_clusters, "n_iters": w.n_iters,
            "density": round(w.density, 4), "variable_groups": w.variable_groups, "batch": w.batch,
            "l2": "inputs larger than L2 (no flush)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="wan14_10")
    ap.add_argument("--heads", type=int, default=0, help="run only the first H heads (profiling cases)")
    ap.add_argument("--impl", default="isa", choices=["isa", "reference"])
    ap.add_argument("--ref-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--top-p", type=float, default=0.0,
                    help="also time isa_select_top_p (exact set by a share of the mass) on the step's mass")
    ap.add_argument("--tail-merge", action="store_true",
                    help="also time isa_tail_merge and isa_attention_merged on the step's plan (variable groups only)")
    ap.add_argument("--cluster", type=int, default=0,
                    help="also time the permuted layout's build: isa_cluster of Q and of K with this many clusters "
                         "(3 rounds) and the row permutations of Q, K and V")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    import torch.distributed as dist
    from block_sparse_importance_b200 import isa
    from block_sparse_importance_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    w = wl.preset(args.workload, seed=0)
    if args.heads:
        w = wl.preset(args.workload, seed=0, heads=args.heads)
    inp = wl.make_inputs(w, str(dev))
    q, k, v = inp.q, inp.k, inp.v
    off_dev = torch.from_numpy(inp.offsets).to(dev) if w.variable_groups else None
    lay = isa.layout_for(q, w.k_block, w.q_block, q_offsets=off_dev, scale=w.scale)
    ctx = isa.context(local)
    stream = torch.cuda.current_stream()
    B, H, N, d = q.shape
    G, nK, S = lay.num_groups, lay.n_key_blocks, w.n_select
    mass = torch.empty(B, H, G, nK, dtype=torch.float32, device=dev)
    idx = torch.empty(B, H, G, S, dtype=torch.int32, device=dev)
    lw = torch.empty(B, H, G, S, dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    sws = torch.empty(isa.score_workspace_bytes(lay, w.n_clusters) + 256, dtype=torch.uint8, device=dev)
    aws_n = isa.attention_workspace_bytes(lay)
    aws = torch.empty(aws_n + 256, dtype=torch.uint8, device=dev) if aws_n else None

    def step(ev=None):
        if ev is not None:
            ev[2].record(stream)
        isa.score(q, k, lay, w.n_clusters, w.n_iters, mass=mass, workspace=sws, ctx=ctx)
        if ev is not None:
            ev[3].record(stream)
        isa.select(mass, lay, w.n_exact, w.n_sample, w.seed, idx=idx, log_w=lw, ctx=ctx)
        if ev is not None:
            ev[0].record(stream)
        isa.attention(q, k, v, idx, lw, lay, out=out, workspace=aws, ctx=ctx)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    st = ctx.sync_status()
    if st != isa.ISA_OK:
        raise RuntimeError("device status after warm-up: %s" % isa.status_string(st))
    flops = plan_flops(idx.cpu().numpy(), inp.offsets, N, w.k_block, d)   # per step (per rank)

    attn_ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_query_id(dev)) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(attn_ev[i])
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    clocks = clk.summary()
    st = ctx.sync_status()
    if st != isa.ISA_OK:
        raise RuntimeError("device status after timing: %s" % isa.status_string(st))
    elapsed_ms = t0.elapsed_time(t1)
    attn_ms = sum(e[0].elapsed_time(e[1]) for e in attn_ev) / args.steps
    score_ms = sum(e[2].elapsed_time(e[3]) for e in attn_ev) / args.steps
    select_ms = sum(e[3].elapsed_time(e[0]) for e in attn_ev) / args.steps
    elapsed_ms, attn_ms, score_ms, select_ms = reduce_max_over_ranks([elapsed_ms, attn_ms, score_ms, select_ms], dev)
    ms_step = elapsed_ms / args.steps
    value = job_throughput(world, flops, ms_step)

    peaks, peak_src = load_peaks()
    achieved = flops / (attn_ms * 1e-3) / 1e12
    peak, peak_kind = roofline_peak(peaks, elapsed_ms, clocks)
    sustained = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": attn_traffic(args.workload, H * B),
                "traffic_unit": "bytes per launch", "kernel": "attn_kernel<128>",
                "peak_source": "%s bf16_tflops%s" % (peak_src, "" if peak_kind == "burst" else "_sustained"),
                "peak_kind": peak_kind,
                "peak_sustained": sustained, "frac_of_sustained": achieved / sustained}

    # the two HBM-bound stages: algorithmic bytes over their event-timed durations
    hbm = float(peaks.get("hbm_gbs"))
    # Q and K read, mass written, centroids and counts written
    score_bytes = 2 * B * H * N * d * 2 + 4 * B * H * G * nK + B * H * G * w.n_clusters * (4 * d + 4)
    select_bytes = B * H * G * (4 * nK + 8 * S)                   # mass read, plan written
    stages = {
        "score": {"ms": score_ms, "bytes": score_bytes, "gbs": score_bytes / (score_ms * 1e-3) / 1e9},
        "select": {"ms": select_ms, "bytes": select_bytes, "gbs": select_bytes / (select_ms * 1e-3) / 1e9},
    }
    for v_ in stages.values():
        v_["frac_hbm"] = v_["gbs"] / hbm

    # score -> select in one call (isa_plan): the mass stays in L2, in chunks
    # of heads, and never reaches HBM
    if rank == 0:
        pp = isa.params(w.n_clusters, w.n_iters, w.n_exact, w.n_sample, w.seed)
        pn = isa.plan_workspace_bytes(lay, pp)
        pws = torch.empty(pn + 256, dtype=torch.uint8, device=dev)
        isa.plan(q, k, lay, pp, idx=idx, log_w=lw, workspace=pws, ctx=ctx)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            isa.plan(q, k, lay, pp, idx=idx, log_w=lw, workspace=pws, ctx=ctx)
        e1.record(stream)
        torch.cuda.synchronize()
        st = ctx.sync_status()
        if st != isa.ISA_OK:
            raise RuntimeError("device status after isa_plan: %s" % isa.status_string(st))
        stages["plan"] = {"ms": e0.elapsed_time(e1) / 3, "score_plus_select_ms": score_ms + select_ms,
                          "workspace_bytes": pn, "mass_bytes_not_allocated": 4 * B * H * G * nK,
                          "what": "isa_plan: score and select in chunks of heads, mass kept in L2"}
        del pws

    # plan reuse across calls: score + select once, then r attention calls
    # with that plan on activations that change from call to call (two input
    # sets, the second a perturbed copy of the first, taken in turn), timed as
    # one loop; ms per attention call
    plan_reuse = None
    if rank == 0:
        plan_reuse = time_plan_reuse(isa, ctx, stream, w, lay, q, k, v, mass, idx, lw, out, sws, aws)

    # dense limit, same tensors (context for the speedup analogue)
    dense_ms = None
    if rank == 0:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        isa.dense_attention(q, k, v, lay, out=out, ctx=ctx)
        e0.record(stream)
        for _ in range(2):
            isa.dense_attention(q, k, v, lay, out=out, ctx=ctx)
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / 2

    # tail merging of the permuted layout on the step's plan: the schedule, and
    # the attention over it (same outputs as the tile-by-tile pass)
    if rank == 0 and args.tail_merge and w.variable_groups:
        sched = isa.tail_merge(idx, lw, lay, ctx=ctx)
        out_m = torch.empty_like(q)
        isa.attention_merged(q, k, v, idx, lw, lay, sched, out=out_m, ctx=ctx)
        e0, e1, e2, e3 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
        e0.record(stream)
        for _ in range(3):
            isa.tail_merge(idx, lw, lay, schedule=sched, ctx=ctx)
        e1.record(stream)
        for _ in range(3):
            isa.attention_merged(q, k, v, idx, lw, lay, sched, out=out_m, ctx=ctx)
        e2.record(stream)
        # the tile-by-tile pass timed the same way, right after
        for _ in range(3):
            isa.attention(q, k, v, idx, lw, lay, out=out_m, workspace=aws, ctx=ctx)
        e3.record(stream)
        torch.cuda.synchronize()
        st = ctx.sync_status()
        if st != isa.ISA_OK:
            raise RuntimeError("device status after tail merging: %s" % isa.status_string(st))
        tm_ms, am_ms, at_ms = e0.elapsed_time(e1) / 3, e1.elapsed_time(e2) / 3, e2.elapsed_time(e3) / 3
        stages["tail_merge"] = {"merge_ms": tm_ms, "attention_merged_ms": am_ms,
                                "attention_same_loop_ms": at_ms, "attention_step_ms": attn_ms,
                                "tflops_merged": flops / (am_ms * 1e-3) / 1e12,
                                "what": "isa_tail_merge, then isa_attention_merged on the step's plan, then "
                                        "isa_attention timed the same way (3 back-to-back calls each)"}
        del sched, out_m

    # the top-p selector on the same mass (count kernel + selector): mass read
    # twice, plan and per-row exact-set sizes written
    if rank == 0 and args.top_p > 0.0:
        ne_rows = torch.empty(B, H, G, dtype=torch.int32, device=dev)
        isa.select_top_p(mass, lay, args.top_p, S, w.seed, idx=idx, log_w=lw, n_exact=ne_rows, ctx=ctx)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            isa.select_top_p(mass, lay, args.top_p, S, w.seed, idx=idx, log_w=lw, n_exact=ne_rows, ctx=ctx)
        e1.record(stream)
        torch.cuda.synchronize()
        st = ctx.sync_status()
        if st != isa.ISA_OK:
            raise RuntimeError("device status after the top-p selector: %s" % isa.status_string(st))
        tp_ms = e0.elapsed_time(e1) / 3
        tp_bytes = B * H * G * (8 * nK + 8 * S + 4)
        ke = ne_rows.float()
        stages["select_top_p"] = {"ms": tp_ms, "p": args.top_p, "bytes": tp_bytes,
                                  "gbs": tp_bytes / (tp_ms * 1e-3) / 1e9,
                                  "frac_hbm": tp_bytes / (tp_ms * 1e-3) / 1e9 / hbm,
                                  "rows_per_s": B * H * G / (tp_ms * 1e-3),
                                  "n_exact_mean": float(ke.mean()), "n_exact_min": int(ke.min()),
                                  "n_exact_max": int(ke.max())}
        if world == 1 and not args.no_cpu_baseline:
            stages["select_top_p"]["cpu_baseline"] = cpu_top_p_sample(mass.cpu().numpy(), args.top_p, S, w.seed)
        del ne_rows

    # the permuted layout's build (token clustering of Q and K, then the row
    # permutations): algorithmic FLOPs are the distance products, 2 N C d per
    # assignment round per tensor and head
    if rank == 0 and args.cluster:
        C_t, it_t = args.cluster, 3
        cws = torch.empty(isa.cluster_workspace_bytes(q, C_t) + 256, dtype=torch.uint8, device=dev)
        qp, kp, vp = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def layout_build():
            rq = isa.cluster(q, C_t, it_t, workspace=cws, ctx=ctx)
            rk = isa.cluster(k, C_t, it_t, workspace=cws, ctx=ctx)
            isa.permute_rows(q, rq["perm"], out=qp, ctx=ctx)
            isa.permute_rows(k, rk["perm"], out=kp, ctx=ctx)
            isa.permute_rows(v, rk["perm"], out=vp, ctx=ctx)

        layout_build()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(2):
            layout_build()
        e1.record(stream)
        torch.cuda.synchronize()
        st = ctx.sync_status()
        if st != isa.ISA_OK:
            raise RuntimeError("device status after the layout build: %s" % isa.status_string(st))
        c_ms = e0.elapsed_time(e1) / 2
        c_flops = 2.0 * N * C_t * d * 2 * B * H * it_t
        stages["cluster"] = {"ms": c_ms, "n_clusters": C_t, "rounds": it_t, "tflop": c_flops / 1e12,
                             "tflops": c_flops / (c_ms * 1e-3) / 1e12,
                             "what": "isa_cluster of Q and of K, then permute_rows of Q, K and V"}
        if world == 1 and not args.no_cpu_baseline:
            stages["cluster"]["cpu_baseline"] = cpu_cluster_sample(wl.bf16_bits(q[:, :1].cpu()), C_t, it_t)
        del qp, kp, vp, cws

    # end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        p = isa.params(w.n_clusters, w.n_iters, w.n_exact, w.n_sample, w.seed)
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty_like(qh).pin_memory()
        del sws
        arena = torch.empty(isa.pipeline_host_workspace_bytes(lay, p) + 256, dtype=torch.uint8, device=dev)
        for _ in range(2):
            isa.pipeline_host(qh, kh, vh, oh, lay, p, arena, ctx=ctx, device=local)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(2, min(args.steps, 5))
        e0.record(stream)
        for _ in range(n_e2e):
            isa.pipeline_host(qh, kh, vh, oh, lay, p, arena, ctx=ctx, device=local)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max_over_ranks([e0.elapsed_time(e1) / n_e2e], dev)[0]
        nbytes = q.numel() * q.element_size()
        e2e = {"value": job_throughput(world, flops, e_ms), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "api": "isa_pipeline_host (pinned host buffers)"}
        del arena

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = wl.make_inputs(w, "cpu", heads=1)
        cpu = cpu_oracle_sample(w, inp_cpu, target_s=args.ref_seconds)

    # key means, k-means (tensor-core kernel for groups of at most 128 rows at
    # d = 128, C <= 16; the per-warp kernel for the rest), mass, selector,
    # attention (+ its tile list for clusters or groups above 128 rows)
    tc_km = d == 128 and w.n_clusters <= 16
    warp_km = (not tc_km) or w.variable_groups or w.q_block > 128
    launches_per_step = 4 + int(tc_km) + int(warp_km) + (1 if aws_n else 0)
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(w),
                "attention_ms": attn_ms, "attention_tflops": achieved,
                "dense_equiv_tflops": world * 4.0 * d * N * N * H * B / (attn_ms * 1e-3) / 1e12,
                "dense_attention_ms": dense_ms,
                "sparse_vs_dense": (dense_ms / attn_ms) if dense_ms else None,
                "computed_tflop_per_step": flops / 1e12,
                "roofline": roofline, "stages": stages, "plan_reuse_ms_per_call": plan_reuse,
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
