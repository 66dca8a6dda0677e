"""Seeded synthetic workloads shaped like the video-DiT attention layers the
pages evaluate on (Wan2.1-T2V-1.3B / 14B, HunyuanVideo), plus a tiny case.

This module is shared by the tests, the benchmark and the CPU oracle's
callers.  It holds input generation only: shapes, the per-token Gaussian
centre model and the cluster-size draw for the permuted layout.  None of the
method's arithmetic (scoring, selection, attention) lives here.

Sources for the shapes: "AB-Attention: Accurate Block Attention for
Accelerating Video Diffusion Transformers" (abstract: Wan2.1 and
HunyuanVideo workloads; fine key blocks gathered into full tiles) and
"InstaGen: Group-Shared Importance Sampling for Fast Video Generation"
(abstract: one sample per query cluster in a permuted layout).  Token grids
are (frames x height x width) latent grids of those models.

Generator (identical for every preset):
  * token n <-> (t, y, x) in row-major order, n = (t*Hgrid + y)*Wgrid + x;
  * per head, query centres mu_c ~ N(0, I_d) and key centres mu'_c ~ N(0, I_d);
  * token centre c(n) = splitmix64(seed ^ (t<<40 | (y>>3)<<20 | (x>>3))) mod
    n_centres, i.e. every 8x8 spatial cell of a frame shares one centre;
    splitmix64 is the mixer of Steele, Lea and Flood, "Fast splittable
    pseudorandom number generators" (OOPSLA 2014);
  * q = s_h*mu_{c(n)} + 0.5*eps, k = s_h*mu'_{c(n)} + 0.5*eps', v ~ N(0, 1);
  * s_h ~ U[0.5, 2] per head where the preset asks for varied entropy, else 1;
  * everything is rounded to bf16.

Permuted layout ("varclust"): 600 cluster sizes drawn from Zipf(1.2),
clipped to [16, 1024] and rescaled to sum to N; cluster g occupies the rows
[off[g], off[g+1]) and its tokens use centre splitmix64(seed ^ g) mod
n_centres.  Q, K and V share the permutation.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

_MASK64 = (1 << 64) - 1


def splitmix64(x: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser (Steele, Lea, Flood 2014) on uint64 arrays."""
    z = (x.astype(np.uint64) + np.uint64(0x9E3779B97F4A7C15))
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention layer: sizes, block sizes, budget and generator knobs."""
    name: str
    heads: int
    head_dim: int
    grid: tuple            # (frames, height, width) latent token grid
    q_block: int           # rows per query group (uniform layout)
    k_block: int           # rows per key block
    n_exact: int           # k_e: exact top blocks per group
    n_sample: int          # n_s: PPS-sampled blocks per group
    n_clusters: int        # C: k-means clusters per query group
    n_iters: int           # I: k-means iterations
    n_centres: int         # Gaussian centres of the generator
    vary_scale: bool       # per-head centre scale s_h ~ U[0.5, 2]
    variable_groups: int = 0   # >0: permuted layout with this many clusters
    batch: int = 1
    seed: int = 0

    @property
    def seq_len(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def n_key_blocks(self) -> int:
        return -(-self.seq_len // self.k_block)

    @property
    def n_select(self) -> int:
        return self.n_exact + self.n_sample

    @property
    def density(self) -> float:
        return self.n_select / self.n_key_blocks


def _budget(n_kblocks: int, density: float, k_block: int):
    """Block budget for a target density: total rounded to nearest, exact =
    total/3 rounded (the 1:2 exact:sampled split of the Wan-14B preset), and
    with 16-row key blocks the total is rounded up to whole 128-row tiles."""
    total = int(math.floor(density * n_kblocks + 0.5))
    if k_block == 16:
        total = -(-total // 8) * 8
    exact = int(math.floor(total / 3.0 + 0.5))
    return exact, total - exact


def _wan14(density: float, name: str) -> Workload:
    nk = -(-21 * 45 * 80 // 64)
    e, s = _budget(nk, density, 64)
    return Workload(name, 40, 128, (21, 45, 80), 128, 64, e, s, 8, 3, 128, True)


def _hunyuan() -> Workload:
    nk = -(-33 * 45 * 80 // 16)
    e, s = _budget(nk, 0.10, 16)
    return Workload("hunyuan", 24, 128, (33, 45, 80), 128, 16, e, s, 8, 3, 128, False)


def _varclust() -> Workload:
    nk = -(-21 * 45 * 80 // 64)
    e, s = _budget(nk, 0.10, 64)
    return Workload("varclust", 40, 128, (21, 45, 80), 128, 64, e, s, 8, 3, 128, False,
                    variable_groups=600)


PRESETS = {
    "tiny": Workload("tiny", 1, 64, (4, 32, 32), 64, 64, 4, 4, 4, 3, 16, False),
    "wan13": Workload("wan13", 12, 128, (21, 30, 52), 128, 64, 16, 35, 8, 3, 64, False),
    "wan14_5": _wan14(0.05, "wan14_5"),
    "wan14_10": _wan14(0.10, "wan14_10"),
    "wan14_20": _wan14(0.20, "wan14_20"),
    "hunyuan": _hunyuan(),
    "varclust": _varclust(),
}


def preset(name: str, **overrides) -> Workload:
    return dataclasses.replace(PRESETS[name], **overrides)


def cluster_sizes(n_clusters: int, n_tokens: int, seed: int,
                  lo: int = 16, hi: int = 1024, a: float = 1.2) -> np.ndarray:
    """Zipf(a) sizes clipped to [lo, hi], rescaled so they sum to n_tokens.

    The remainder after rescaling is spread +-1 cyclically by index over the
    clusters that stay inside the bounds."""
    rng = np.random.default_rng(seed)
    s = np.clip(rng.zipf(a, n_clusters), lo, hi).astype(np.int64)
    s = np.clip(np.floor(s * n_tokens / s.sum()).astype(np.int64), lo, hi)
    if not (lo * n_clusters <= n_tokens <= hi * n_clusters):
        raise ValueError("cluster bounds cannot cover n_tokens")
    i = 0
    while s.sum() != n_tokens:
        step = 1 if s.sum() < n_tokens else -1
        if lo <= s[i] + step <= hi:
            s[i] += step
        i = (i + 1) % n_clusters
    return s


def group_offsets(w: Workload) -> np.ndarray:
    """Row offsets [G+1] of the query groups (uniform blocks or clusters)."""
    n = w.seq_len
    if w.variable_groups:
        sizes = cluster_sizes(w.variable_groups, n, w.seed)
        return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    g = -(-n // w.q_block)
    return np.minimum(np.arange(g + 1, dtype=np.int64) * w.q_block, n).astype(np.int32)


def token_centres(w: Workload) -> np.ndarray:
    """Centre id of every token, [N] int64."""
    if w.variable_groups:
        off = group_offsets(w)
        g_of_row = np.repeat(np.arange(len(off) - 1, dtype=np.uint64), np.diff(off))
        h = splitmix64(np.uint64(w.seed) ^ g_of_row)
    else:
        t, hh, ww = w.grid
        tt, yy, xx = np.meshgrid(np.arange(t, dtype=np.uint64), np.arange(hh, dtype=np.uint64),
                                 np.arange(ww, dtype=np.uint64), indexing="ij")
        cell = (tt << np.uint64(40)) | ((yy >> np.uint64(3)) << np.uint64(20)) | (xx >> np.uint64(3))
        h = splitmix64(np.uint64(w.seed) ^ cell.reshape(-1))
    return (h % np.uint64(w.n_centres)).astype(np.int64)


@dataclasses.dataclass
class Inputs:
    q: torch.Tensor          # [B, H, N, d] bf16
    k: torch.Tensor
    v: torch.Tensor
    offsets: np.ndarray      # [G+1] int32 row offsets of the query groups
    workload: Workload


def make_inputs(w: Workload, device: str = "cpu", heads: Optional[int] = None,
                seq_len: Optional[int] = None) -> Inputs:
    """Generate Q/K/V for a workload with a seeded torch generator on `device`.

    `heads` / `seq_len` truncate the layer (first heads / first tokens) for
    small parity cases; the centre model is unchanged."""
    H = heads if heads is not None else w.heads
    n_full = w.seq_len
    N = seq_len if seq_len is not None else n_full
    d = w.head_dim
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    B = w.batch
    mu_q = torch.randn(B, H, w.n_centres, d, generator=gen, device=device, dtype=torch.float32)
    mu_k = torch.randn(B, H, w.n_centres, d, generator=gen, device=device, dtype=torch.float32)
    if w.vary_scale:
        s_h = 0.5 + 1.5 * torch.rand(B, H, 1, 1, generator=gen, device=device, dtype=torch.float32)
    else:
        s_h = torch.ones(B, H, 1, 1, device=device, dtype=torch.float32)
    cid = torch.from_numpy(token_centres(w)[:N]).to(device)
    idx = cid.view(1, 1, N, 1).expand(B, H, N, d)
    out = []
    for mu in (mu_q, mu_k):
        x = torch.gather(mu, 2, idx) * s_h
        x.add_(torch.randn(B, H, N, d, generator=gen, device=device, dtype=torch.float32), alpha=0.5)
        out.append(x.to(torch.bfloat16))
        del x
    v = torch.randn(B, H, N, d, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    off = group_offsets(w)
    if N != n_full:
        off = np.unique(np.minimum(off, N)).astype(np.int32)
    return Inputs(out[0].contiguous(), out[1].contiguous(), v.contiguous(), off, w)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a contiguous uint16 numpy array."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
