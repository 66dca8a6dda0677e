"""Shared builders for the GPU parity tests.

Inputs come from the seeded generators; plans and expected values come from
the CPU oracle only.  Nothing here reads a CUDA result back into an oracle
input."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_sparse_importance_b200 import workloads as wl

# Acceptance bars (bf16 inputs, fp32 accumulation).
ATTN_REL_L2 = 1e-2
ATTN_MAX_ABS = 2e-2
DENSE_MAX_ABS = 5e-3
MASS_REL_L2 = 1e-3
LOGW_ABS = 1e-6


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def random_offsets(N: int, lo: int, hi: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    sizes = []
    left = N
    while left > 0:
        s = int(rng.integers(lo, hi + 1))
        if left - s < lo:
            s = left
        sizes.append(s)
        left -= s
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)


class Case:
    """A small problem: inputs on the CPU, oracle plan and oracle outputs."""

    def __init__(self, preset: str, H: int, N: int, k_block: int, q_block: int, n_exact: int,
                 n_sample: int, offsets=None, seed: int = 0, n_clusters=None):
        w = wl.preset(preset, k_block=k_block, q_block=q_block, n_exact=n_exact, n_sample=n_sample,
                      seed=seed)
        if n_clusters is not None:
            w = wl.preset(preset, k_block=k_block, q_block=q_block, n_exact=n_exact, n_sample=n_sample,
                          seed=seed, n_clusters=n_clusters)
        inp = wl.make_inputs(w, "cpu", heads=H, seq_len=N)
        self.w = w
        self.q, self.k, self.v = inp.q, inp.k, inp.v
        self.variable = offsets is not None
        self.offsets = np.asarray(offsets, np.int32) if offsets is not None else inp.offsets
        self.N, self.H, self.d = N, H, w.head_dim
        self.G = len(self.offsets) - 1
        self.nK = -(-N // k_block)
        self.bits = [wl.bf16_bits(t) for t in (self.q, self.k, self.v)]
        self.seed = seed
        self._plan = None

    def oracle_mass(self):
        q, k, _ = self.bits
        return oracle.score(q, k, self.offsets, self.w.k_block, self.w.n_clusters, self.w.n_iters, self.w.scale)

    def plan(self):
        if self._plan is None:
            mass, _, _, _ = self.oracle_mass()
            idx, lw, bad = oracle.select(mass.astype(np.float32), self.w.n_exact, self.w.n_sample, self.seed)
            self._plan = (idx, lw)
        return self._plan

    def oracle_attention(self, idx=None, lw=None):
        if idx is None:
            idx, lw = self.plan()
        q, k, v = self.bits
        groups = [(0, h, g) for h in range(self.H) for g in range(self.G)]
        res = oracle.attention(q, k, v, self.offsets, self.w.k_block, idx, lw, self.w.scale, groups)
        out = np.zeros((1, self.H, self.N, self.d))
        lse = np.zeros((1, self.H, self.N))
        i = 0
        for h in range(self.H):
            for g in range(self.G):
                o, l = res[i]
                i += 1
                out[0, h, self.offsets[g]:self.offsets[g + 1]] = o
                lse[0, h, self.offsets[g]:self.offsets[g + 1]] = l
        return out, lse

    def layout(self, device="cuda"):
        from block_sparse_importance_b200 import isa
        off = torch.from_numpy(self.offsets).to(device) if self.variable else None
        return isa.Layout(1, self.H, self.N, self.d, self.w.q_block, self.w.k_block, self.G, self.w.scale, off)

    def cuda(self):
        return [t.cuda() for t in (self.q, self.k, self.v)]


def check_attention(out_gpu, out_ref, lse_gpu=None, lse_ref=None, max_abs=ATTN_MAX_ABS, rel=ATTN_REL_L2):
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(o - out_ref)
    assert np.all(np.isfinite(o)), "non-finite output"
    r = rel_l2(o, out_ref)
    assert r <= rel, "rel-L2 %.3g > %.3g" % (r, rel)
    assert err.max() <= max_abs, "max abs %.3g > %.3g" % (err.max(), max_abs)
    if lse_gpu is not None:
        l = lse_gpu.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(l - lse_ref)) < 2e-2
    return r, float(err.max())
