"""Estimator quality of the sparse pass against the dense limit, on the GPU.

    python -m block_sparse_importance_b200.estimator_study [--workload wan13] [--heads 4]

At a fixed budget of S key blocks per query group, the attention output of
several plans is compared with isa_dense_attention on the same tensors
(relative L2 over all rows), while the softmax temperature is swept: the
score scale is t / sqrt(d), so larger t makes every row's attention peakier
(lower entropy).  The plans:

  is            the method: an exact set of n_exact blocks plus a systematic
                PPS sample of n_sample blocks, each drawn block weighted by
                1 / pi in the numerator and the denominator (log-weight added
                to its logits);
  top_s         the n_exact + n_sample highest-mass blocks, unweighted
                (truncation, no sample);
  unweighted    the same blocks as `is` with the log-weights dropped (the
                sample counted once instead of 1 / pi times);
  is_small_blk  the method with key blocks a quarter as tall and four times
                as many of them (same number of key rows).

The IS rows are averaged over several seeds; `is_seed_spread` is the largest
minus the smallest error over the seeds.  Everything runs through the
library's own entry points; the dense kernel is the reference.

V is drawn two ways.  `--values noise`: the workload's own V ~ N(0, 1), with
no structure, so a dense output that averages thousands of keys is close to
zero and every sparse estimate is mostly noise relative to it.  `--values
clustered` (default): v = nu_c(n) + 0.5 eps with a mean nu_c ~ N(0, I) per
token centre (the same centres that place q and k), so the blocks that
attention finds also carry the values it averages.
"""
from __future__ import annotations

import argparse
import json

import torch

from block_sparse_importance_b200 import isa
from block_sparse_importance_b200 import workloads as wl


def rel_l2(a: torch.Tensor, b: torch.Tensor) -> float:
    a = a.float()
    b = b.float()
    return float(torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b).clamp_min(1e-30))


def clustered_values(w, B: int, H: int, N: int, d: int, device: str = "cuda") -> torch.Tensor:
    """v = nu_c(n) + 0.5 eps, nu_c ~ N(0, I) per head and token centre."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 7919)
    nu = torch.randn(B, H, w.n_centres, d, generator=gen, device=device)
    cid = torch.from_numpy(wl.token_centres(w)[:N]).to(device)
    v = torch.gather(nu, 2, cid.view(1, 1, N, 1).expand(B, H, N, d))
    v.add_(torch.randn(B, H, N, d, generator=gen, device=device), alpha=0.5)
    return v.to(torch.bfloat16).contiguous()


def run(workload: str = "wan13", heads: int = 4, temps=(0.5, 1.0, 2.0, 4.0, 8.0), seeds=(0, 1, 2, 3),
        density: float = 0.1, values: str = "clustered", keep_plans: bool = False) -> dict:
    """The study's table.  With keep_plans, every row also carries the plans
    it measured (CPU tensors: "plans" maps a plan name to a list of (idx,
    log_w, k_block), one per seed where the row averages over seeds) and the
    result carries the q, k, v it used, so that the figures can be recomputed
    elsewhere."""
    w = wl.preset(workload)
    inp = wl.make_inputs(w, "cuda", heads=heads)
    q, k, v = inp.q, inp.k, inp.v
    if values == "clustered":
        v = clustered_values(w, q.shape[0], q.shape[1], q.shape[2], q.shape[3])
    N, d = q.shape[2], q.shape[3]
    rows = []
    for t in temps:
        scale = t / d ** 0.5
        lay = isa.layout_for(q, w.k_block, w.q_block, scale=scale)
        dense = isa.dense_attention(q, k, v, lay)
        nK = lay.n_key_blocks
        total = max(2, int(density * nK + 0.5))
        ne = int(total / 3 + 0.5)
        ns = total - ne
        mass = isa.score(q, k, lay, w.n_clusters, w.n_iters)
        row = {"t": t, "S": total, "n_exact": ne, "n_sample": ns}
        plans = {"is": [], "unweighted": [], "top_s": [], "is_small_blk": []}

        def keep(name, idx_, lw_, bk):
            if keep_plans:
                plans[name].append((idx_.cpu(), lw_.cpu(), bk))

        errs = []
        for s in seeds:
            idx, lw = isa.select(mass, lay, ne, ns, s)
            errs.append(rel_l2(isa.attention(q, k, v, idx, lw, lay), dense))
            keep("is", idx, lw, w.k_block)
            if s == seeds[0]:
                row["unweighted"] = rel_l2(isa.attention(q, k, v, idx, torch.zeros_like(lw), lay), dense)
                keep("unweighted", idx, torch.zeros_like(lw), w.k_block)
        row["is"] = sum(errs) / len(errs)
        row["is_seed_spread"] = max(errs) - min(errs)
        idx, lw = isa.select(mass, lay, total, 0, 0)
        row["top_s"] = rel_l2(isa.attention(q, k, v, idx, lw, lay), dense)
        keep("top_s", idx, lw, w.k_block)
        # four times as many blocks a quarter as tall (the same key rows)
        bk4 = w.k_block // 4
        lay4 = isa.layout_for(q, bk4, w.q_block, scale=scale)
        total4 = 4 * total
        total4 = -(-total4 // 8) * 8 if bk4 == 16 else total4  # whole 128-row tiles at 16-row blocks
        ne4 = int(total4 / 3 + 0.5)
        mass4 = isa.score(q, k, lay4, w.n_clusters, w.n_iters)
        errs4 = []
        for s in seeds:
            idx4, lw4 = isa.select(mass4, lay4, ne4, total4 - ne4, s)
            errs4.append(rel_l2(isa.attention(q, k, v, idx4, lw4, lay4), dense))
            keep("is_small_blk", idx4, lw4, bk4)
        row["is_small_blk"] = sum(errs4) / len(errs4)
        row["small_blk_S"] = total4
        if keep_plans:
            row["plans"] = plans
        rows.append(row)
    status = isa.context().sync_status()
    res = {"workload": workload, "heads": heads, "N": N, "k_block": w.k_block, "density": density,
           "values": values, "seeds": list(seeds), "rows": rows, "status": status}
    if keep_plans:
        res["qkv"] = tuple(x.cpu() for x in (q, k, v))
        res["offsets"] = inp.offsets
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="wan13")
    ap.add_argument("--heads", type=int, default=4)
    ap.add_argument("--density", type=float, default=0.1)
    ap.add_argument("--values", choices=["clustered", "noise"], default="clustered")
    args = ap.parse_args()
    res = run(args.workload, args.heads, density=args.density, values=args.values)
    print(json.dumps(res))
    print("%6s %5s %9s %9s %11s %9s %13s" % ("t", "S", "is", "top_s", "unweighted", "spread", "is_small_blk"))
    for r in res["rows"]:
        print("%6.2f %5d %9.4f %9.4f %11.4f %9.4f %13.4f" % (r["t"], r["S"], r["is"], r["top_s"], r["unweighted"],
                                                            r["is_seed_spread"], r["is_small_blk"]))


if __name__ == "__main__":
    main()
