"""ctypes front end of the fp64 CPU oracle (oracle/isa_ref.cpp).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  Nothing here is used by,
or uses, the CUDA path; the two share only the seeded input generators.

Every function takes bf16 tensors as raw uint16 bit patterns (numpy), so
the oracle reads exactly the values the GPU reads, and computes in fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "isa_ref.cpp")
_LIB = os.path.join(_HERE, "_isa_ref.so")
_lock = threading.Lock()
_lib = None

# Margin below which a k-means assignment counts as a near tie, relative to
# ||q||^2 + ||mu||^2.  A d-term fp32 sum of squares is within d 2^-24 of its
# magnitude (<= 2 (||q||^2 + ||mu||^2)), i.e. 1.5e-5 of that scale at d = 128;
# the threshold keeps a 2x margin over that bound.
KMEANS_TIE_REL = 3e-5


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (OpenMP) into oracle/_isa_ref.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, u32, u64, f64 = ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double
            lib.ref_philox4x64_10.argtypes = [P, P, P]
            lib.ref_group_uniform.argtypes = [u64, i32, i32, i32]
            lib.ref_group_uniform.restype = u32
            lib.ref_key_means.argtypes = [P, i32, i32, i32, P, P]
            lib.ref_kmeans_group.argtypes = [P, i32, i32, i32, i32, f64, P, P]
            lib.ref_kmeans_group.restype = i32
            lib.ref_mass_group.argtypes = [P, P, i32, P, P, i32, i32, f64, P]
            lib.ref_score.argtypes = [P, P, i32, i32, i32, i32, i32, P, i32, i32, i32, f64, f64,
                                      P, P, P, P, i32]
            lib.ref_select_row.argtypes = [P, i32, i32, i32, u32, P, P, P, P]
            lib.ref_select_row.restype = i32
            lib.ref_select.argtypes = [P, i32, i32, i32, i32, i32, i32, u64, P, P, P, i32]
            lib.ref_select.restype = i32
            lib.ref_top_p_count.argtypes = [P, i32, f64, i32, P]
            lib.ref_top_p_count.restype = i32
            lib.ref_select_top_p.argtypes = [P, i32, i32, i32, i32, f64, i32, u64, P, P, P, P, i32]
            lib.ref_select_top_p.restype = i32
            lib.ref_attention.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, i32, P, P, i32, f64,
                                          P, i32, P, P, i32]
            lib.ref_dense_attention.argtypes = [P, P, P, i32, i32, f64, P, i32, P, P, i32]
            lib.ref_cluster_assign.argtypes = [P, i32, i32, P, i32, f64, P, P]
            lib.ref_cluster_assign.restype = None
            lib.ref_cluster_sort.argtypes = [P, i32, i32, P, P]
            lib.ref_cluster_sort.restype = None
            lib.ref_cluster_update.argtypes = [P, i32, i32, P, i32, P, P]
            lib.ref_cluster_update.restype = None
            lib.ref_cluster_tokens.argtypes = [P, i32, i32, i32, i32, i32, f64, P, P, P, P, P, i32]
            lib.ref_tail_merge.argtypes = [P, i32, P, i32, i32, P, P, P, P]
            lib.ref_tail_merge.restype = i32
            lib.ref_num_threads.restype = i32
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().ref_num_threads())


def philox4x64_10(counter, key) -> np.ndarray:
    ctr = _c(np.array(counter, dtype=np.uint64), np.uint64)
    k = _c(np.array(key, dtype=np.uint64), np.uint64)
    out = np.zeros(4, np.uint64)
    _load().ref_philox4x64_10(_p(ctr), _p(k), _p(out))
    return out


def group_uniform(seed: int, batch: int, head: int, group: int) -> int:
    return int(_load().ref_group_uniform(seed, batch, head, group))


def key_means(k_head: np.ndarray, k_block: int):
    """k_head: [N, d] uint16 bf16 bits -> (kbar [nK, d] f64, L [nK] i32)."""
    k_head = _c(k_head, np.uint16)
    N, d = k_head.shape
    nK = -(-N // k_block)
    kbar = np.zeros((nK, d), np.float64)
    L = np.zeros(nK, np.int32)
    _load().ref_key_means(_p(k_head), N, d, k_block, _p(kbar), _p(L))
    return kbar, L


def kmeans_group(q_rows: np.ndarray, n_clusters: int, n_iters: int, tie_rel: float = KMEANS_TIE_REL):
    """q_rows: [n, d] uint16 bf16 bits -> (mu [C, d], counts [C], ambiguous)."""
    if n_iters < 1:
        raise ValueError("n_iters must be >= 1")
    q_rows = _c(q_rows, np.uint16)
    n, d = q_rows.shape
    mu = np.zeros((n_clusters, d), np.float64)
    cnt = np.zeros(n_clusters, np.int32)
    amb = _load().ref_kmeans_group(_p(q_rows), n, d, n_clusters, n_iters, tie_rel, _p(mu), _p(cnt))
    return mu, cnt, bool(amb)


def cluster_assign(x_rows: np.ndarray, mu: np.ndarray, tie_rel: float = KMEANS_TIE_REL):
    """One assignment round: x_rows [n, d] uint16 bf16 bits, mu [C, d] ->
    (labels [n] i32, ambiguous [n] bool)."""
    x_rows = _c(x_rows, np.uint16)
    mu = _c(mu, np.float64)
    n, d = x_rows.shape
    C = mu.shape[0]
    lab = np.zeros(n, np.int32)
    amb = np.zeros(n, np.int32)
    _load().ref_cluster_assign(_p(x_rows), n, d, _p(mu), C, tie_rel, _p(lab), _p(amb))
    return lab, amb.astype(bool)


def cluster_sort(labels: np.ndarray, n_clusters: int):
    """Stable counting sort: labels [n] -> (perm [n] i32, offsets [C + 1] i32)."""
    labels = _c(labels, np.int32)
    if labels.size and (labels.min() < 0 or labels.max() >= n_clusters):
        raise ValueError("labels out of range")
    perm = np.zeros(labels.size, np.int32)
    off = np.zeros(n_clusters + 1, np.int32)
    _load().ref_cluster_sort(_p(labels), labels.size, n_clusters, _p(perm), _p(off))
    return perm, off


def cluster_update(x_rows: np.ndarray, labels: np.ndarray, mu: np.ndarray):
    """Mean update: returns (new mu [C, d] f64, counts [C] i32); an empty
    cluster keeps its row of `mu`."""
    x_rows = _c(x_rows, np.uint16)
    labels = _c(labels, np.int32)
    mu = np.array(mu, dtype=np.float64, copy=True, order="C")
    n, d = x_rows.shape
    C = mu.shape[0]
    cnt = np.zeros(C, np.int32)
    _load().ref_cluster_update(_p(x_rows), n, d, _p(labels), C, _p(mu), _p(cnt))
    return mu, cnt


def cluster_tokens(x: np.ndarray, n_clusters: int, n_iters: int, tie_rel: float = KMEANS_TIE_REL,
                   threads: int = 0):
    """Clustering of every (batch, head) over the whole sequence.
    x: [B, H, N, d] uint16 bf16 bits -> (labels [B,H,N], perm [B,H,N],
    offsets [B,H,C+1], mu [B,H,C,d] f64, ambiguous [B,H] bool)."""
    x = _c(x, np.uint16)
    B, H, N, d = x.shape
    C = n_clusters
    lab = np.zeros((B, H, N), np.int32)
    perm = np.zeros((B, H, N), np.int32)
    off = np.zeros((B, H, C + 1), np.int32)
    mu = np.zeros((B, H, C, d), np.float64)
    amb = np.zeros((B, H), np.int32)
    st = _load().ref_cluster_tokens(_p(x), B * H, N, d, C, n_iters, tie_rel, _p(lab), _p(perm), _p(off), _p(mu),
                                    _p(amb), threads)
    if st != 0:
        raise ValueError("ref_cluster_tokens: need N >= 1, 1 <= C <= N, n_iters >= 1")
    return lab, perm, off, mu, amb.astype(bool)


def tail_merge(offsets: np.ndarray, idx: np.ndarray, k_block: int):
    """Merged tail tiles of the permuted layout, per (batch, head).

    offsets [G+1] int32 (shared by every head); idx [B, H, G, S] int32 plans.
    Returns a list over b*H + h of (members [n, 4], slots [n, 4], ulen [n],
    units [n, 4 S]): the tiles in the order they were opened, each with its
    member clusters (-1 past the last), the first row of each member's slot,
    and the union of the members' plan blocks, ascending."""
    off = _c(offsets, np.int32)
    idx = _c(idx, np.int32)
    B, H, G, S = idx.shape
    assert len(off) == G + 1
    n_tails = int(np.count_nonzero(np.diff(off) % 128))
    res = []
    for bh in range(B * H):
        mem = np.full((max(n_tails, 1), 4), -1, np.int32)
        slo = np.full((max(n_tails, 1), 4), -1, np.int32)
        ul = np.zeros(max(n_tails, 1), np.int32)
        un = np.zeros((max(n_tails, 1), 4 * S), np.int32)
        rows = idx.reshape(B * H, G, S)[bh]
        n = _load().ref_tail_merge(_p(off), G, _p(np.ascontiguousarray(rows)), S, k_block, _p(mem), _p(slo),
                                   _p(ul), _p(un))
        res.append((mem[:n], slo[:n], ul[:n], un[:n]))
    return res


def mass_group(mu: np.ndarray, counts: np.ndarray, kbar: np.ndarray, L: np.ndarray, scale: float):
    mu = _c(mu, np.float64)
    counts = _c(counts, np.int32)
    kbar = _c(kbar, np.float64)
    L = _c(L, np.int32)
    C, d = mu.shape
    nK = kbar.shape[0]
    out = np.zeros(nK, np.float64)
    _load().ref_mass_group(_p(mu), _p(counts), C, _p(kbar), _p(L), nK, d, scale, _p(out))
    return out


def score(q: np.ndarray, k: np.ndarray, offsets: np.ndarray, k_block: int, n_clusters: int,
          n_iters: int, scale: float, tie_rel: float = KMEANS_TIE_REL, threads: int = 0):
    """q, k: [B, H, N, d] uint16 bf16 bits; offsets [G+1].
    Returns mass [B,H,G,nK] f64, centroids [B,H,G,C,d] f64, counts [B,H,G,C] i32,
    ambiguous [B,H,G] bool."""
    if n_iters < 1:
        raise ValueError("n_iters must be >= 1")
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    off = _c(offsets, np.int32)
    B, H, N, d = q.shape
    G = len(off) - 1
    nK = -(-N // k_block)
    mass = np.zeros((B, H, G, nK), np.float64)
    cen = np.zeros((B, H, G, n_clusters, d), np.float64)
    cnt = np.zeros((B, H, G, n_clusters), np.int32)
    amb = np.zeros((B, H, G), np.int32)
    _load().ref_score(_p(q), _p(k), B, H, N, d, G, _p(off), k_block, n_clusters, n_iters, scale,
                      tie_rel, _p(mass), _p(cen), _p(cnt), _p(amb), threads)
    return mass, cen, cnt, amb.astype(bool)


def select_row(mass_row: np.ndarray, n_exact: int, n_sample: int, U: int):
    """One plan row from fp32 mass with an explicit 32-bit uniform U.
    Returns (idx [S] i32, log_w [S] f32, pi [nK] f64, bad)."""
    m = _c(mass_row, np.float32)
    nK = m.shape[0]
    S = n_exact + n_sample
    idx = np.zeros(S, np.int32)
    lw = np.zeros(S, np.float32)
    pi = np.zeros(nK, np.float64)
    bad = np.zeros(1, np.int32)
    st = _load().ref_select_row(_p(m), nK, n_exact, n_sample, ctypes.c_uint32(U), _p(idx), _p(lw),
                                _p(pi), _p(bad))
    if st != 0:
        raise ValueError("ref_select_row failed with %d" % st)
    return idx, lw, pi, bool(bad[0])


def select(mass: np.ndarray, n_exact: int, n_sample: int, seed: int, threads: int = 0):
    """mass: [B, H, G, nK] fp32 -> (idx [B,H,G,S] i32, log_w [B,H,G,S] f32, bad)."""
    m = _c(mass, np.float32)
    B, H, G, nK = m.shape
    S = n_exact + n_sample
    idx = np.zeros((B, H, G, S), np.int32)
    lw = np.zeros((B, H, G, S), np.float32)
    bad = np.zeros(1, np.int32)
    st = _load().ref_select(_p(m), B, H, G, nK, n_exact, n_sample, ctypes.c_uint64(seed), _p(idx),
                            _p(lw), _p(bad), threads)
    if st != 0:
        raise ValueError("ref_select failed with %d" % st)
    return idx, lw, bool(bad[0])


def top_p_count(mass_row: np.ndarray, p: float, S: int):
    """Exact-set size of one row under the top-p rule (see ref_top_p_count).
    Returns (k_e, bad)."""
    m = _c(mass_row, np.float32)
    bad = np.zeros(1, np.int32)
    k = _load().ref_top_p_count(_p(m), m.shape[0], ctypes.c_double(p), S, _p(bad))
    if k < 0:
        raise ValueError("ref_top_p_count: bad arguments")
    return int(k), bool(bad[0])


def select_top_p(mass: np.ndarray, p: float, S: int, seed: int, threads: int = 0):
    """mass: [B, H, G, nK] fp32 -> (idx [B,H,G,S] i32, log_w [B,H,G,S] f32,
    k_e [B,H,G] i32, bad) under the top-p rule."""
    m = _c(mass, np.float32)
    B, H, G, nK = m.shape
    idx = np.zeros((B, H, G, S), np.int32)
    lw = np.zeros((B, H, G, S), np.float32)
    ke = np.zeros((B, H, G), np.int32)
    bad = np.zeros(1, np.int32)
    st = _load().ref_select_top_p(_p(m), B, H, G, nK, ctypes.c_double(p), S, ctypes.c_uint64(seed), _p(idx),
                                  _p(lw), _p(ke), _p(bad), threads)
    if st != 0:
        raise ValueError("ref_select_top_p failed with %d" % st)
    return idx, lw, ke, bool(bad[0])


def attention(q, k, v, offsets, k_block: int, idx, log_w, scale: float, groups, threads: int = 0):
    """Sparse attention of the listed (batch, head, group) triples.

    q, k, v: [B, H, N, d] uint16 bf16 bits; idx/log_w: [B, H, G, S].
    Returns a list of (out [n_g, d] f64, lse [n_g] f64), one per listed group."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    off = _c(offsets, np.int32)
    idx = _c(idx, np.int32)
    lw = _c(log_w, np.float32)
    B, H, N, d = q.shape
    G = len(off) - 1
    S = idx.shape[-1]
    gl = _c(np.array(groups, dtype=np.int32).reshape(-1, 3), np.int32)
    sizes = [int(off[g + 1] - off[g]) for (_, _, g) in gl]
    total = sum(sizes)
    out = np.zeros((total, d), np.float64)
    lse = np.zeros(total, np.float64)
    _load().ref_attention(_p(q), _p(k), _p(v), B, H, N, d, G, _p(off), k_block, _p(idx), _p(lw), S,
                          scale, _p(gl), len(gl), _p(out), _p(lse), threads)
    res, o = [], 0
    for s in sizes:
        res.append((out[o:o + s], lse[o:o + s]))
        o += s
    return res


def dense_attention(q, k, v, scale: float, rows, threads: int = 0):
    """Dense softmax attention for listed rows: rows = [(batch*H + head, row), ...].
    q, k, v: [B, H, N, d] uint16.  Returns (out [n, d] f64, lse [n] f64)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    B, H, N, d = q.shape
    r = _c(np.array(rows, dtype=np.int64).reshape(-1, 2), np.int64)
    out = np.zeros((len(r), d), np.float64)
    lse = np.zeros(len(r), np.float64)
    _load().ref_dense_attention(_p(q), _p(k), _p(v), N, d, scale, _p(r), len(r), _p(out), _p(lse),
                                threads)
    return out, lse
