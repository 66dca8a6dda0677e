"""Thin ctypes binding of libisa.so (include/isa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing the calls raise; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libisa.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "isa.h")

ISA_OK, ISA_ERR_INVALID_ARG, ISA_ERR_UNSUPPORTED, ISA_ERR_CUDA, ISA_ERR_TIMEOUT, ISA_ERR_DEVICE_CHECK = range(6)
ISA_DEBUG_WAIT_TIMEOUT_NS, ISA_DEBUG_STALL_ATTENTION = 1, 2

_i32, _u64, _f32, _P, _sz = ctypes.c_int32, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class Shape(ctypes.Structure):
    _fields_ = [("batch", _i32), ("heads", _i32), ("seq_len", _i32), ("head_dim", _i32),
                ("q_block", _i32), ("k_block", _i32), ("num_groups", _i32), ("q_offsets", _P),
                ("scale", _f32)]


class Params(ctypes.Structure):
    _fields_ = [("n_clusters", _i32), ("n_iters", _i32), ("n_exact", _i32), ("n_sample", _i32),
                ("seed", _u64)]


class IsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s (status %d)" % (message, status))
        self.status = status


_lib = None
_lock = threading.Lock()


def lib():
    """Load libisa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libisa.so not built: run python -m block_sparse_importance_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            S, Pp = ctypes.POINTER(Shape), ctypes.POINTER(Params)
            L.isa_create.argtypes = [ctypes.c_int, ctypes.POINTER(_P)]
            L.isa_destroy.argtypes = [_P]
            L.isa_destroy.restype = None
            L.isa_status_string.argtypes = [ctypes.c_int]
            L.isa_status_string.restype = ctypes.c_char_p
            L.isa_last_error.argtypes = [_P]
            L.isa_last_error.restype = ctypes.c_char_p
            L.isa_sync_status.argtypes = [_P, _P]
            L.isa_score_workspace_bytes.argtypes = [S, _i32]
            L.isa_score_workspace_bytes.restype = _sz
            L.isa_score.argtypes = [_P, S, _P, _P, _i32, _i32, _P, _P, _P, _P, _sz, _P]
            L.isa_select.argtypes = [_P, S, _P, _i32, _i32, _u64, _P, _P, _P]
            L.isa_select_top_p.argtypes = [_P, S, _P, ctypes.c_double, _i32, _u64, _P, _P, _P, _P]
            L.isa_cluster_workspace_bytes.argtypes = [S, _i32]
            L.isa_cluster_workspace_bytes.restype = _sz
            L.isa_cluster.argtypes = [_P, S, _P, _i32, _i32, _P, _P, _P, _P, _P, _P, _P, _sz, _P]
            L.isa_cluster_assign.argtypes = [_P, S, _P, _P, _i32, _P, _P, _sz, _P]
            L.isa_cluster_sort.argtypes = [_P, S, _P, _i32, _P, _P, _P, _P, _P]
            L.isa_cluster_update.argtypes = [_P, S, _P, _P, _P, _i32, _P, _P, _sz, _P]
            L.isa_permute_rows.argtypes = [_P, S, _P, _P, _i32, _P, _P]
            L.isa_attention_workspace_bytes.argtypes = [S]
            L.isa_attention_workspace_bytes.restype = _sz
            L.isa_attention.argtypes = [_P, S, _P, _P, _P, _P, _P, _i32, _P, _P, _P, _sz, _P]
            L.isa_dense_attention.argtypes = [_P, S, _P, _P, _P, _P, _P, _P]
            L.isa_tail_merge_workspace_bytes.argtypes = [S, _i32]
            L.isa_tail_merge_workspace_bytes.restype = _sz
            L.isa_tail_merge.argtypes = [_P, S, _P, _P, _i32, _P, _sz, _P]
            L.isa_attention_merged.argtypes = [_P, S, _P, _P, _P, _P, _P, _i32, _P, _sz, _P, _P, _P]
            L.isa_plan_workspace_bytes.argtypes = [S, Pp]
            L.isa_plan_workspace_bytes.restype = _sz
            L.isa_plan.argtypes = [_P, S, Pp, _P, _P, _P, _P, _P, _sz, _P]
            L.isa_pipeline_workspace_bytes.argtypes = [S, Pp]
            L.isa_pipeline_workspace_bytes.restype = _sz
            L.isa_pipeline.argtypes = [_P, S, Pp, _P, _P, _P, _P, _P, _P, _P, _P, _sz, _P]
            L.isa_pipeline_host_workspace_bytes.argtypes = [S, Pp]
            L.isa_pipeline_host_workspace_bytes.restype = _sz
            L.isa_pipeline_host.argtypes = [_P, S, Pp, _P, _P, _P, _P, _P, _sz, _P]
            L.isa_debug_set.argtypes = [_P, _i32, _u64]
            L.isa_debug_set.restype = ctypes.c_int
            L.isa_attention_noalloc.argtypes = [_P, S, _P, _P, _P, _P, _P, _i32, _P, _P, _P]
            for name in ("isa_create", "isa_sync_status", "isa_score", "isa_select", "isa_select_top_p", "isa_attention",
                         "isa_dense_attention", "isa_pipeline", "isa_pipeline_host", "isa_attention_noalloc",
                         "isa_cluster", "isa_cluster_assign", "isa_cluster_sort", "isa_cluster_update",
                         "isa_permute_rows"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def declared_symbols():
    """Names of the entry points include/isa.h declares."""
    with open(HEADER) as f:
        return sorted(set(re.findall(r"^ISA_API [^;]*?\b(isa_\w+)\(", f.read(), flags=re.M)))


def status_string(status: int) -> str:
    return lib().isa_status_string(status).decode()


class Context:
    """An isa_context on one CUDA device (owns the device status word)."""

    def __init__(self, device: int = 0):
        h = _P()
        st = lib().isa_create(device, ctypes.byref(h))
        if st != ISA_OK:
            raise IsaError(st, "isa_create(%d): %s" % (device, status_string(st)))
        self.handle = h
        self.device = device

    def close(self):
        if getattr(self, "handle", None):
            lib().isa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def check(self, status: int, what: str):
        if status != ISA_OK:
            msg = lib().isa_last_error(self.handle).decode()
            raise IsaError(status, "%s: %s: %s" % (what, status_string(status), msg))

    def debug_set(self, knob: int, value: int):
        """Failure-detection test hooks (ISA_DEBUG_* in include/isa.h)."""
        self.check(lib().isa_debug_set(self.handle, knob, value), "isa_debug_set")

    def sync_status(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        """Synchronise the stream; return (and clear) the device status word."""
        return lib().isa_sync_status(self.handle, _stream(stream))


_contexts = {}


def context(device: int = 0) -> Context:
    if device not in _contexts:
        _contexts[device] = Context(device)
    return _contexts[device]


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return _P(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return _P(t.data_ptr()) if t is not None else _P(0)


def _dev(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (name, dtype))
    return t


@dataclass
class Layout:
    """Problem shape (isa_shape) for Q/K/V of shape [B, H, N, d]."""
    batch: int
    heads: int
    seq_len: int
    head_dim: int
    q_block: int
    k_block: int
    num_groups: int
    scale: float
    q_offsets: Optional[torch.Tensor] = None   # device int32 [G+1]

    @property
    def n_key_blocks(self) -> int:
        return -(-self.seq_len // self.k_block)

    def c(self) -> Shape:
        return Shape(self.batch, self.heads, self.seq_len, self.head_dim, self.q_block, self.k_block,
                     self.num_groups, _ptr(self.q_offsets), self.scale)


def layout_for(q: torch.Tensor, k_block: int, q_block: int = 128, q_offsets: Optional[torch.Tensor] = None,
               scale: Optional[float] = None) -> Layout:
    B, H, N, d = q.shape
    G = (len(q_offsets) - 1) if q_offsets is not None else -(-N // q_block)
    return Layout(B, H, N, d, q_block, k_block, G, scale if scale is not None else d ** -0.5, q_offsets)


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def score_workspace_bytes(lay: Layout, n_clusters: int) -> int:
    return int(lib().isa_score_workspace_bytes(ctypes.byref(lay.c()), n_clusters))


def attention_workspace_bytes(lay: Layout) -> int:
    return int(lib().isa_attention_workspace_bytes(ctypes.byref(lay.c())))


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]):
    if nbytes == 0:
        return None
    if ws is None or ws.numel() * ws.element_size() < nbytes:
        ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    return ws


def score(q, k, lay: Layout, n_clusters: int, n_iters: int, mass=None, centroids=None, counts=None,
          workspace=None, ctx: Optional[Context] = None, stream=None):
    """isa_score: estimated attention mass [B, H, G, nK] (fp32)."""
    ctx = ctx or context(q.device.index or 0)
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k")
    B, H, G, nK = lay.batch, lay.heads, lay.num_groups, lay.n_key_blocks
    mass = mass if mass is not None else _empty((B, H, G, nK), torch.float32, q.device)
    nb = score_workspace_bytes(lay, n_clusters)
    workspace = _workspace(nb, q.device, workspace)
    sh = lay.c()
    st = lib().isa_score(ctx.handle, ctypes.byref(sh), _ptr(q), _ptr(k), n_clusters, n_iters, _ptr(mass),
                         _ptr(centroids), _ptr(counts), _ptr(workspace), nb, _stream(stream))
    ctx.check(st, "isa_score")
    return mass


def select(mass, lay: Layout, n_exact: int, n_sample: int, seed: int, idx=None, log_w=None,
           ctx: Optional[Context] = None, stream=None):
    """isa_select: plan (idx [B,H,G,S] int32, log_w [B,H,G,S] fp32)."""
    ctx = ctx or context(mass.device.index or 0)
    _dev(mass, torch.float32, "mass")
    S = n_exact + n_sample
    shp = (lay.batch, lay.heads, lay.num_groups, S)
    idx = idx if idx is not None else _empty(shp, torch.int32, mass.device)
    log_w = log_w if log_w is not None else _empty(shp, torch.float32, mass.device)
    sh = lay.c()
    st = lib().isa_select(ctx.handle, ctypes.byref(sh), _ptr(mass), n_exact, n_sample, ctypes.c_uint64(seed),
                          _ptr(idx), _ptr(log_w), _stream(stream))
    ctx.check(st, "isa_select")
    return idx, log_w


def select_top_p(mass, lay: Layout, top_p: float, n_select: int, seed: int, idx=None, log_w=None, n_exact=None,
                 ctx: Optional[Context] = None, stream=None):
    """isa_select_top_p: plan of n_select blocks per row whose exact part
    keeps a share top_p of the row's mass; returns (idx, log_w, n_exact)
    with n_exact [B,H,G] int32 the exact-set size of each row."""
    ctx = ctx or context(mass.device.index or 0)
    _dev(mass, torch.float32, "mass")
    shp = (lay.batch, lay.heads, lay.num_groups, n_select)
    idx = idx if idx is not None else _empty(shp, torch.int32, mass.device)
    log_w = log_w if log_w is not None else _empty(shp, torch.float32, mass.device)
    n_exact = n_exact if n_exact is not None else _empty(shp[:3], torch.int32, mass.device)
    sh = lay.c()
    st = lib().isa_select_top_p(ctx.handle, ctypes.byref(sh), _ptr(mass), float(top_p), n_select,
                                ctypes.c_uint64(seed), _ptr(idx), _ptr(log_w), _ptr(n_exact), _stream(stream))
    ctx.check(st, "isa_select_top_p")
    return idx, log_w, n_exact


def _rows_shape(x: torch.Tensor) -> Shape:
    """isa_shape of the token-clustering calls (batch, heads, seq_len, head_dim)."""
    B, H, N, d = x.shape
    return Shape(B, H, N, d, 1, 64, N, None, 1.0)


def cluster_workspace_bytes(x: torch.Tensor, n_clusters: int) -> int:
    return int(lib().isa_cluster_workspace_bytes(ctypes.byref(_rows_shape(x)), n_clusters))


def cluster(x, n_clusters: int, n_iters: int, workspace=None, ctx: Optional[Context] = None, stream=None):
    """isa_cluster: k-means of every (batch, head) over the whole sequence and
    the stable sort of its labels.  Returns a dict of device tensors:
    centroids [B,H,C,d] f32, labels / perm [B,H,N] i32, offsets / groups
    [B,H,C+1] i32 and n_groups [B,H] i32."""
    ctx = ctx or context(x.device.index or 0)
    _dev(x, torch.bfloat16, "x")
    B, H, N, d = x.shape
    C = n_clusters
    r = {"centroids": _empty((B, H, C, d), torch.float32, x.device),
         "labels": _empty((B, H, N), torch.int32, x.device),
         "perm": _empty((B, H, N), torch.int32, x.device),
         "offsets": _empty((B, H, C + 1), torch.int32, x.device),
         "groups": _empty((B, H, C + 1), torch.int32, x.device),
         "n_groups": _empty((B, H), torch.int32, x.device)}
    sh = _rows_shape(x)
    nb = int(lib().isa_cluster_workspace_bytes(ctypes.byref(sh), C))
    ws = _workspace(nb, x.device, workspace)
    st = lib().isa_cluster(ctx.handle, ctypes.byref(sh), _ptr(x), C, n_iters, _ptr(r["centroids"]), _ptr(r["labels"]),
                           _ptr(r["perm"]), _ptr(r["offsets"]), _ptr(r["groups"]), _ptr(r["n_groups"]), _ptr(ws), nb,
                           _stream(stream))
    ctx.check(st, "isa_cluster")
    return r


def cluster_assign(x, centroids, workspace=None, ctx: Optional[Context] = None, stream=None):
    """isa_cluster_assign: nearest of the given centroids [B,H,C,d] f32 -> labels [B,H,N] i32."""
    ctx = ctx or context(x.device.index or 0)
    _dev(x, torch.bfloat16, "x")
    _dev(centroids, torch.float32, "centroids")
    C = centroids.shape[2]
    labels = _empty(x.shape[:3], torch.int32, x.device)
    sh = _rows_shape(x)
    nb = int(lib().isa_cluster_workspace_bytes(ctypes.byref(sh), C))
    ws = _workspace(nb, x.device, workspace)
    st = lib().isa_cluster_assign(ctx.handle, ctypes.byref(sh), _ptr(x), _ptr(centroids), C, _ptr(labels), _ptr(ws),
                                  nb, _stream(stream))
    ctx.check(st, "isa_cluster_assign")
    return labels


def cluster_sort(labels, n_clusters: int, head_dim: int = 128, ctx: Optional[Context] = None, stream=None):
    """isa_cluster_sort: labels [B,H,N] i32 -> (perm, offsets, groups, n_groups)."""
    ctx = ctx or context(labels.device.index or 0)
    _dev(labels, torch.int32, "labels")
    B, H, N = labels.shape
    C = n_clusters
    perm = _empty((B, H, N), torch.int32, labels.device)
    off = _empty((B, H, C + 1), torch.int32, labels.device)
    grp = _empty((B, H, C + 1), torch.int32, labels.device)
    ng = _empty((B, H), torch.int32, labels.device)
    sh = Shape(B, H, N, head_dim, 1, 64, N, None, 1.0)
    st = lib().isa_cluster_sort(ctx.handle, ctypes.byref(sh), _ptr(labels), C, _ptr(perm), _ptr(off), _ptr(grp),
                                _ptr(ng), _stream(stream))
    ctx.check(st, "isa_cluster_sort")
    return perm, off, grp, ng


def cluster_update(x, perm, offsets, centroids, workspace=None, ctx: Optional[Context] = None, stream=None):
    """isa_cluster_update: centroids [B,H,C,d] f32 updated in place to the
    means of the sorted clusters (empty clusters keep theirs)."""
    ctx = ctx or context(x.device.index or 0)
    _dev(x, torch.bfloat16, "x")
    _dev(centroids, torch.float32, "centroids")
    C = centroids.shape[2]
    sh = _rows_shape(x)
    nb = int(lib().isa_cluster_workspace_bytes(ctypes.byref(sh), C))
    ws = _workspace(nb, x.device, workspace)
    st = lib().isa_cluster_update(ctx.handle, ctypes.byref(sh), _ptr(x), _ptr(perm), _ptr(offsets), C,
                                  _ptr(centroids), _ptr(ws), nb, _stream(stream))
    ctx.check(st, "isa_cluster_update")
    return centroids


def permute_rows(x, perm, inverse: bool = False, out=None, ctx: Optional[Context] = None, stream=None):
    """isa_permute_rows: out[i] = x[perm[i]], or out[perm[i]] = x[i] with inverse."""
    ctx = ctx or context(x.device.index or 0)
    _dev(x, torch.bfloat16, "x")
    _dev(perm, torch.int32, "perm")
    out = out if out is not None else _empty(x.shape, torch.bfloat16, x.device)
    st = lib().isa_permute_rows(ctx.handle, ctypes.byref(_rows_shape(x)), _ptr(x), _ptr(perm), 1 if inverse else 0,
                                _ptr(out), _stream(stream))
    ctx.check(st, "isa_permute_rows")
    return out


def attention(q, k, v, idx, log_w, lay: Layout, out=None, lse=None, workspace=None,
              ctx: Optional[Context] = None, stream=None, want_lse: bool = False):
    """isa_attention: sparse pass over the plan; returns out (and lse)."""
    ctx = ctx or context(q.device.index or 0)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, torch.bfloat16, n)
    _dev(idx, torch.int32, "idx")
    _dev(log_w, torch.float32, "log_w")
    out = out if out is not None else torch.empty_like(q)
    if want_lse and lse is None:
        lse = _empty(q.shape[:3], torch.float32, q.device)
    nb = attention_workspace_bytes(lay)
    workspace = _workspace(nb, q.device, workspace)
    sh = lay.c()
    st = lib().isa_attention(ctx.handle, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(log_w),
                             int(idx.shape[-1]), _ptr(out), _ptr(lse), _ptr(workspace), nb, _stream(stream))
    ctx.check(st, "isa_attention")
    return (out, lse) if want_lse else out


def tail_merge_workspace_bytes(lay: Layout, n_sel: int) -> int:
    return int(lib().isa_tail_merge_workspace_bytes(ctypes.byref(lay.c()), int(n_sel)))


def tail_merge(idx, log_w, lay: Layout, schedule=None, ctx: Optional[Context] = None, stream=None):
    """isa_tail_merge: the merged-tail schedule of a plan (permuted layout);
    returns the schedule buffer (uint8) for attention_merged."""
    ctx = ctx or context(idx.device.index or 0)
    _dev(idx, torch.int32, "idx")
    _dev(log_w, torch.float32, "log_w")
    n_sel = int(idx.shape[-1])
    nb = tail_merge_workspace_bytes(lay, n_sel)
    schedule = _workspace(nb, idx.device, schedule)
    st = lib().isa_tail_merge(ctx.handle, ctypes.byref(lay.c()), _ptr(idx), _ptr(log_w), n_sel, _ptr(schedule), nb,
                              _stream(stream))
    ctx.check(st, "isa_tail_merge")
    return schedule


def attention_merged(q, k, v, idx, log_w, lay: Layout, schedule, out=None, lse=None, ctx: Optional[Context] = None,
                     stream=None, want_lse: bool = False):
    """isa_attention_merged: the sparse pass over the schedule of tail_merge."""
    ctx = ctx or context(q.device.index or 0)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, torch.bfloat16, n)
    _dev(idx, torch.int32, "idx")
    _dev(log_w, torch.float32, "log_w")
    out = out if out is not None else torch.empty_like(q)
    if want_lse and lse is None:
        lse = _empty(q.shape[:3], torch.float32, q.device)
    n_sel = int(idx.shape[-1])
    nb = schedule.numel() * schedule.element_size()
    st = lib().isa_attention_merged(ctx.handle, ctypes.byref(lay.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                    _ptr(log_w), n_sel, _ptr(schedule), nb, _ptr(out), _ptr(lse), _stream(stream))
    ctx.check(st, "isa_attention_merged")
    return (out, lse) if want_lse else out


def dense_attention(q, k, v, lay: Layout, out=None, lse=None, ctx: Optional[Context] = None, stream=None,
                    want_lse: bool = False):
    """isa_dense_attention: softmax(scale Q K^T) V over all keys."""
    ctx = ctx or context(q.device.index or 0)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, torch.bfloat16, n)
    out = out if out is not None else torch.empty_like(q)
    if want_lse and lse is None:
        lse = _empty(q.shape[:3], torch.float32, q.device)
    sh = lay.c()
    st = lib().isa_dense_attention(ctx.handle, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                   _stream(stream))
    ctx.check(st, "isa_dense_attention")
    return (out, lse) if want_lse else out


def params(n_clusters: int, n_iters: int, n_exact: int, n_sample: int, seed: int) -> Params:
    return Params(n_clusters, n_iters, n_exact, n_sample, seed)


def pipeline_workspace_bytes(lay: Layout, p: Params) -> int:
    return int(lib().isa_pipeline_workspace_bytes(ctypes.byref(lay.c()), ctypes.byref(p)))


def pipeline_host_workspace_bytes(lay: Layout, p: Params) -> int:
    return int(lib().isa_pipeline_host_workspace_bytes(ctypes.byref(lay.c()), ctypes.byref(p)))


def plan_workspace_bytes(lay: Layout, p: Params) -> int:
    sh = lay.c()
    return int(lib().isa_plan_workspace_bytes(ctypes.byref(sh), ctypes.byref(p)))


def plan(q, k, lay: Layout, p: Params, idx=None, log_w=None, workspace=None, ctx: Optional[Context] = None,
         stream=None):
    """isa_plan: score -> select in one call; returns (idx, log_w) [B,H,G,S]."""
    ctx = ctx or context(q.device.index or 0)
    for t, n in ((q, "q"), (k, "k")):
        _dev(t, torch.bfloat16, n)
    S = p.n_exact + p.n_sample
    shp = (lay.batch, lay.heads, lay.num_groups, S)
    idx = idx if idx is not None else _empty(shp, torch.int32, q.device)
    log_w = log_w if log_w is not None else _empty(shp, torch.float32, q.device)
    nb = plan_workspace_bytes(lay, p)
    workspace = _workspace(nb, q.device, workspace)
    sh = lay.c()
    st = lib().isa_plan(ctx.handle, ctypes.byref(sh), ctypes.byref(p), _ptr(q), _ptr(k), _ptr(idx), _ptr(log_w),
                        _ptr(workspace), nb, _stream(stream))
    ctx.check(st, "isa_plan")
    return idx, log_w


def pipeline(q, k, v, lay: Layout, p: Params, out=None, lse=None, plan_idx=None, plan_log_w=None,
             workspace=None, ctx: Optional[Context] = None, stream=None):
    """isa_pipeline: score -> select -> attention on device buffers."""
    ctx = ctx or context(q.device.index or 0)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, torch.bfloat16, n)
    out = out if out is not None else torch.empty_like(q)
    nb = pipeline_workspace_bytes(lay, p)
    workspace = _workspace(nb, q.device, workspace)
    sh = lay.c()
    st = lib().isa_pipeline(ctx.handle, ctypes.byref(sh), ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                            _ptr(lse), _ptr(plan_idx), _ptr(plan_log_w), _ptr(workspace), nb, _stream(stream))
    ctx.check(st, "isa_pipeline")
    return out


def pipeline_host(q_host, k_host, v_host, out_host, lay: Layout, p: Params, workspace,
                  ctx: Optional[Context] = None, stream=None, device: int = 0):
    """isa_pipeline_host: host (pinned) Q/K/V in, host O out, device arena."""
    ctx = ctx or context(device)
    for t, n in ((q_host, "q"), (k_host, "k"), (v_host, "v"), (out_host, "out")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous host bf16 tensor" % n)
    nb = pipeline_host_workspace_bytes(lay, p)
    if workspace.numel() * workspace.element_size() < nb:
        raise ValueError("arena too small: need %d bytes" % nb)
    sh = lay.c()
    st = lib().isa_pipeline_host(ctx.handle, ctypes.byref(sh), ctypes.byref(p), _ptr(q_host), _ptr(k_host),
                                 _ptr(v_host), _ptr(out_host), _ptr(workspace), nb, _stream(stream))
    ctx.check(st, "isa_pipeline_host")
    return out_host


def attention_noalloc(q, k, v, idx, log_w, lay: Layout, out=None, lse=None, ctx: Optional[Context] = None,
                      stream=None, want_lse: bool = False):
    """isa_attention_noalloc: the same pass as attention(), for callers that
    cannot allocate device memory (no workspace argument: the library's own
    1 MiB scratch array holds the tile list).  Calls that overlap on the GPU
    share that array, so keep them ordered."""
    ctx = ctx or context(q.device.index or 0)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, torch.bfloat16, n)
    _dev(idx, torch.int32, "idx")
    _dev(log_w, torch.float32, "log_w")
    out = out if out is not None else torch.empty_like(q)
    if want_lse and lse is None:
        lse = _empty(q.shape[:3], torch.float32, q.device)
    sh = lay.c()
    st = lib().isa_attention_noalloc(ctx.handle, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                     _ptr(log_w), int(idx.shape[-1]), _ptr(out), _ptr(lse), _stream(stream))
    ctx.check(st, "isa_attention_noalloc")
    return (out, lse) if want_lse else out
