"""Thin ctypes binding of librtp.so (C ABI in include/rtp.h).

The functions below carry the C names and only marshal arguments: torch
tensors become device pointers, the current torch stream becomes the
cudaStream_t, the config becomes an ``rtp_attn_cfg`` struct.  Every step of
the attention path runs in the library's CUDA kernels; there is no fallback.
If librtp.so is missing or fails to load, importing this module raises.

``hybrid_prefill_layer`` and ``sparse_decode_step`` chain the calls of one
layer / one decode step and allocate their intermediate buffers with torch
(device memory is the only thing torch is used for here).
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# RTP_LIB may name another build of the library (for example one compiled
# with different tuning macros); by default the in-tree build is loaded.
LIB_PATH = os.environ.get("RTP_LIB") or os.path.join(_HERE, "librtp.so")

RTP_OK, RTP_ERR_INVALID_ARG, RTP_ERR_UNSUPPORTED, RTP_ERR_CUDA, RTP_ERR_TIMEOUT, RTP_ERR_NO_MEMORY = range(6)
RTP_HEAD_SWA, RTP_HEAD_FULL, RTP_HEAD_SPARSE = 0, 1, 2


class RtpError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")
        self.status = status


class rtp_attn_cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "seq", "n_q_heads", "n_kv_heads", "head_dim", "window",
                                            "block", "rank", "topk", "n_sink", "n_local")] + [("scale", ctypes.c_float)]


class rtp_clusters(ctypes.Structure):
    _fields_ = [("clu_end", ctypes.c_int), ("n_clusters", ctypes.c_int), ("centroids", ctypes.c_void_p),
                ("members", ctypes.c_void_p), ("offsets", ctypes.c_void_p), ("k_sorted", ctypes.c_void_p),
                ("v_sorted", ctypes.c_void_p), ("chunk_centroids", ctypes.c_void_p), ("chunk_start", ctypes.c_void_p),
                ("chunk_len", ctypes.c_void_p), ("n_chunks", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m swa_hybrid_attention_b200.build` "
                          "(the CUDA extension is required; there is no CPU path)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, L, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_size_t
    cfgp = ctypes.POINTER(rtp_attn_cfg)
    sig = {
        "rtp_route_heads": (I, [cfgp, P, P, ctypes.POINTER(P)]),
        "rtp_route_heads_range": (I, [cfgp, P, I, I, P, ctypes.POINTER(P)]),
        "rtp_route_heads_split": (I, [cfgp, P, I, I, I, P, ctypes.POINTER(P)]),
        "rtp_plan_num_local_items": (L, [P]),
        "rtp_plan_destroy": (None, [P]),
        "rtp_plan_num_sparse": (I, [P]),
        "rtp_plan_num_items": (L, [P]),
        "rtp_plan_sparse_heads": (I, [P, P]),
        "rtp_plan_work_items": (I, [P, P]),
        "rtp_indexer_project": (I, [P, P, P, P, P, P, P]),
        "rtp_block_select": (I, [P, P, P, P, P, P]),
        "rtp_block_select_dynamic": (I, [P, P, P, ctypes.c_float, I, ctypes.c_float, P, P, P]),
        "rtp_block_select_rowmax": (I, [P, P, P, P, P, P, P]),
        "rtp_indexer_project_heads": (I, [P, P, P, P, P]),
        "rtp_block_select_heads": (I, [P, P, P, P, P, P]),
        "rtp_hybrid_prefill_heads": (I, [P, P, P, P, P, P, P, P]),
        "rtp_hybrid_prefill": (I, [P, P, P, P, P, P, P, P]),
        "rtp_hybrid_prefill_items": (I, [P, P, P, P, P, P, P, L, L, I, P]),
        "rtp_pipeline_create": (I, [cfgp, P, I, P, ctypes.POINTER(P)]),
        "rtp_pipeline_destroy": (None, [P]),
        "rtp_hybrid_prefill_host": (I, [P] * 15),
        "rtp_decode_workspace_bytes": (S, [cfgp, P, I]),
        "rtp_sparse_decode": (I, [cfgp, P, I, P, P, P, P, P, P, P, S, P, P, P]),
        "rtp_sparse_decode_noalloc": (I, [cfgp, P, I, P, P, P, P, P, P, P, P, P]),
        "rtp_cache_centroids": (I, [cfgp, P, I, P, P, P, P]),
        "rtp_cache_append": (I, [cfgp, P, I, P, P, P, P, P, P, P]),
        "rtp_cache_cluster_workspace_bytes": (S, [cfgp, I]),
        "rtp_cache_cluster": (I, [cfgp, P, I, P, P, P, ctypes.POINTER(rtp_clusters), P, S, P]),
        "rtp_decode_clustered_workspace_bytes": (S, [cfgp, P, I, I]),
        "rtp_sparse_decode_clustered": (I, [cfgp, P, I, P, P, P, P, ctypes.POINTER(rtp_clusters), P, P, S, P, P, P]),
        "rtp_last_device_status": (I, [P]),
        "rtp_selftest_bounded_wait": (I, [ctypes.c_uint, P]),
        "rtp_status_str": (ctypes.c_char_p, [I]),
        "rtp_version": (I, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("rtp_route_heads", "rtp_route_heads_range", "rtp_route_heads_split", "rtp_plan_num_local_items",
            "rtp_hybrid_prefill_items", "rtp_plan_destroy", "rtp_plan_num_sparse", "rtp_plan_num_items",
            "rtp_plan_sparse_heads", "rtp_plan_work_items", "rtp_indexer_project", "rtp_block_select",
            "rtp_block_select_dynamic", "rtp_block_select_rowmax", "rtp_indexer_project_heads",
            "rtp_block_select_heads", "rtp_hybrid_prefill_heads", "rtp_pipeline_create", "rtp_pipeline_destroy", "rtp_hybrid_prefill_host",
            "rtp_hybrid_prefill", "rtp_decode_workspace_bytes", "rtp_sparse_decode", "rtp_sparse_decode_noalloc",
            "rtp_cache_centroids", "rtp_cache_append", "rtp_cache_cluster_workspace_bytes", "rtp_cache_cluster",
            "rtp_decode_clustered_workspace_bytes", "rtp_sparse_decode_clustered",
            "rtp_last_device_status", "rtp_selftest_bounded_wait",
            "rtp_status_str", "rtp_version")


def status_str(s: int) -> str:
    return _lib.rtp_status_str(int(s)).decode()


def _check(name: str, s: int):
    if s != RTP_OK:
        raise RtpError(name, s)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return t.data_ptr()
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _kinds(kinds) -> ctypes.Array:
    return (ctypes.c_uint8 * len(kinds))(*[int(x) for x in kinds])


@dataclass
class AttnConfig:
    batch: int
    seq: int
    n_q_heads: int
    n_kv_heads: int
    window: int
    block: int = 128
    topk: int = 0
    n_local: int = 1
    scale: float = 0.0
    head_dim: int = 128
    rank: int = 16
    n_sink: int = 1

    def c(self) -> rtp_attn_cfg:
        return rtp_attn_cfg(self.batch, self.seq, self.n_q_heads, self.n_kv_heads, self.head_dim, self.window,
                            self.block, self.rank, self.topk, self.n_sink, self.n_local, self.scale)

    @property
    def kmax(self) -> int:
        return self.topk + 1 + self.n_local


# ------------------------------------------------------------- C-named calls


def rtp_route_heads(cfg: AttnConfig, kinds, stream=None) -> int:
    """Returns an opaque plan handle (int); free with rtp_plan_destroy."""
    out = ctypes.c_void_p()
    c = cfg.c()
    _check("rtp_route_heads", _lib.rtp_route_heads(ctypes.byref(c), _kinds(kinds), _stream(stream),
                                                     ctypes.byref(out)))
    return out.value


def rtp_route_heads_range(cfg: AttnConfig, kinds, q_begin: int, q_end: int, stream=None) -> int:
    """A plan for query rows [q_begin, q_end) only (one context-parallel rank's share)."""
    out = ctypes.c_void_p()
    c = cfg.c()
    _check("rtp_route_heads_range", _lib.rtp_route_heads_range(ctypes.byref(c), _kinds(kinds), int(q_begin),
                                                                 int(q_end), _stream(stream), ctypes.byref(out)))
    return out.value


def rtp_route_heads_split(cfg: AttnConfig, kinds, q_begin: int, q_end: int, key_begin: int, stream=None) -> int:
    """A ranged plan whose work list puts the tiles that see only keys >= key_begin first."""
    out = ctypes.c_void_p()
    c = cfg.c()
    _check("rtp_route_heads_split", _lib.rtp_route_heads_split(ctypes.byref(c), _kinds(kinds), int(q_begin),
                                                                 int(q_end), int(key_begin), _stream(stream),
                                                                 ctypes.byref(out)))
    return out.value


def rtp_plan_num_local_items(plan: int) -> int:
    return _lib.rtp_plan_num_local_items(plan)


def rtp_plan_destroy(plan: int) -> None:
    _lib.rtp_plan_destroy(plan)


def rtp_plan_num_sparse(plan: int) -> int:
    return _lib.rtp_plan_num_sparse(plan)


def rtp_plan_num_items(plan: int) -> int:
    return _lib.rtp_plan_num_items(plan)


def rtp_plan_sparse_heads(plan: int) -> list:
    n = rtp_plan_num_sparse(plan)
    buf = (ctypes.c_int32 * max(1, n))()
    _check("rtp_plan_sparse_heads", _lib.rtp_plan_sparse_heads(plan, buf))
    return list(buf)[:n]


def rtp_plan_work_items(plan: int):
    import numpy as np

    n = rtp_plan_num_items(plan)
    arr = np.empty((n, 4), dtype=np.int32)
    _check("rtp_plan_work_items", _lib.rtp_plan_work_items(plan, arr.ctypes.data_as(ctypes.c_void_p)))
    return arr


def rtp_indexer_project(plan: int, q, k, proj, centroids, qbar, stream=None) -> None:
    _check("rtp_indexer_project", _lib.rtp_indexer_project(plan, _ptr(q), _ptr(k), _ptr(proj), _ptr(centroids),
                                                           _ptr(qbar), _stream(stream)))


def rtp_block_select(plan: int, qbar, centroids, sel, sel_cnt, stream=None) -> None:
    _check("rtp_block_select", _lib.rtp_block_select(plan, _ptr(qbar), _ptr(centroids), _ptr(sel), _ptr(sel_cnt),
                                                     _stream(stream)))


def rtp_block_select_dynamic(plan: int, qbar, centroids, mass: float, min_k: int, beta: float, sel, sel_cnt,
                             stream=None) -> None:
    _check("rtp_block_select_dynamic",
           _lib.rtp_block_select_dynamic(plan, _ptr(qbar), _ptr(centroids), float(mass), int(min_k), float(beta),
                                         _ptr(sel), _ptr(sel_cnt), _stream(stream)))


def rtp_block_select_rowmax(plan: int, q, proj, centroids, sel, sel_cnt, stream=None) -> None:
    _check("rtp_block_select_rowmax",
           _lib.rtp_block_select_rowmax(plan, _ptr(q), _ptr(proj), _ptr(centroids), _ptr(sel), _ptr(sel_cnt),
                                        _stream(stream)))


def rtp_indexer_project_heads(plan: int, q, proj, qbar_heads, stream=None) -> None:
    _check("rtp_indexer_project_heads",
           _lib.rtp_indexer_project_heads(plan, _ptr(q), _ptr(proj), _ptr(qbar_heads), _stream(stream)))


def rtp_block_select_heads(plan: int, qbar_heads, centroids, sel, sel_cnt, stream=None) -> None:
    _check("rtp_block_select_heads",
           _lib.rtp_block_select_heads(plan, _ptr(qbar_heads), _ptr(centroids), _ptr(sel), _ptr(sel_cnt),
                                       _stream(stream)))


def rtp_hybrid_prefill_heads(plan: int, q, k, v, sel, sel_cnt, o, stream=None) -> None:
    _check("rtp_hybrid_prefill_heads",
           _lib.rtp_hybrid_prefill_heads(plan, _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(sel_cnt), _ptr(o),
                                         _stream(stream)))


def default_selection_beta(cfg: AttnConfig) -> float:
    """Softmax scale / group: weighs a block like the group-mean of its attention logits."""
    scale = cfg.scale if cfg.scale > 0 else 1.0 / math.sqrt(cfg.head_dim)
    return scale / (cfg.n_q_heads // cfg.n_kv_heads)


def rtp_hybrid_prefill(plan: int, q, k, v, sel, sel_cnt, o, stream=None) -> None:
    _check("rtp_hybrid_prefill", _lib.rtp_hybrid_prefill(plan, _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(sel_cnt),
                                                         _ptr(o), _stream(stream)))


def rtp_hybrid_prefill_items(plan: int, q, k, v, sel, sel_cnt, o, item_begin: int, item_end: int,
                             max_ctas: int = 0, stream=None) -> None:
    _check("rtp_hybrid_prefill_items",
           _lib.rtp_hybrid_prefill_items(plan, _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(sel_cnt), _ptr(o),
                                         int(item_begin), int(item_end), int(max_ctas), _stream(stream)))


def rtp_pipeline_create(cfg: AttnConfig, kinds, n_chunks: int, stream=None) -> int:
    out = ctypes.c_void_p()
    c = cfg.c()
    _check("rtp_pipeline_create", _lib.rtp_pipeline_create(ctypes.byref(c), _kinds(kinds), int(n_chunks),
                                                             _stream(stream), ctypes.byref(out)))
    return out.value


def rtp_pipeline_destroy(pipeline: int) -> None:
    _lib.rtp_pipeline_destroy(pipeline)


def rtp_hybrid_prefill_host(pipeline: int, q_host, k_host, v_host, proj, o_host, q_dev, k_dev, v_dev, o_dev,
                            centroids=None, qbar=None, sel=None, sel_cnt=None, stream=None) -> None:
    _check("rtp_hybrid_prefill_host",
           _lib.rtp_hybrid_prefill_host(pipeline, _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(proj),
                                        _ptr(o_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev), _ptr(o_dev),
                                        _ptr(centroids), _ptr(qbar), _ptr(sel), _ptr(sel_cnt), _stream(stream)))


def rtp_decode_workspace_bytes(cfg: AttnConfig, kinds, cache_len: int) -> int:
    c = cfg.c()
    return int(_lib.rtp_decode_workspace_bytes(ctypes.byref(c), _kinds(kinds), int(cache_len)))


def rtp_sparse_decode(cfg: AttnConfig, kinds, cache_len: int, q, kcache, vcache, centroids, proj, o, workspace,
                      ws_bytes: int, sel_out=None, cnt_out=None, stream=None) -> None:
    c = cfg.c()
    _check("rtp_sparse_decode", _lib.rtp_sparse_decode(ctypes.byref(c), _kinds(kinds), int(cache_len), _ptr(q),
                                                       _ptr(kcache), _ptr(vcache), _ptr(centroids), _ptr(proj),
                                                       _ptr(o), _ptr(workspace), int(ws_bytes), _ptr(sel_out),
                                                       _ptr(cnt_out), _stream(stream)))


def rtp_sparse_decode_noalloc(cfg: AttnConfig, kinds, cache_len: int, q, kcache, vcache, centroids, proj, o,
                              sel_out=None, cnt_out=None, stream=None) -> None:
    """Decode step whose scratch is the library's fixed device array (no allocation)."""
    c = cfg.c()
    _check("rtp_sparse_decode_noalloc",
           _lib.rtp_sparse_decode_noalloc(ctypes.byref(c), _kinds(kinds), int(cache_len), _ptr(q), _ptr(kcache),
                                          _ptr(vcache), _ptr(centroids), _ptr(proj), _ptr(o), _ptr(sel_out),
                                          _ptr(cnt_out), _stream(stream)))


def rtp_cache_centroids(cfg: AttnConfig, kinds, cache_len: int, kcache, proj, centroids, stream=None) -> None:
    """Centroids of every complete cache block of the retrieval heads (cfg.seq = cache capacity)."""
    c = cfg.c()
    _check("rtp_cache_centroids", _lib.rtp_cache_centroids(ctypes.byref(c), _kinds(kinds), int(cache_len),
                                                           _ptr(kcache), _ptr(proj), _ptr(centroids),
                                                           _stream(stream)))


def rtp_cache_append(cfg: AttnConfig, kinds, pos: int, k_new, v_new, kcache, vcache, proj, centroids,
                     stream=None) -> None:
    """Writes cache row `pos`; completes the centroid of the block that row fills (cfg.seq = capacity)."""
    c = cfg.c()
    _check("rtp_cache_append", _lib.rtp_cache_append(ctypes.byref(c), _kinds(kinds), int(pos), _ptr(k_new),
                                                     _ptr(v_new), _ptr(kcache), _ptr(vcache), _ptr(proj),
                                                     _ptr(centroids), _stream(stream)))


class Clusters:
    """Device arrays of a clustered KV cache (rtp_clusters), allocated with torch."""

    def __init__(self, batch: int, n_kv_heads: int, clu_end: int, n_clusters: int, block: int, device,
                 in_place: bool = False):
        """in_place: no cluster-ordered copy of K/V (k_sorted / v_sorted NULL):
        the clustered decode gathers each chunk's member rows from the cache."""
        n = clu_end - block
        self.clu_end, self.n_clusters, self.n = clu_end, n_clusters, n
        self.max_chunks = n // 128 + n_clusters
        i32 = dict(dtype=torch.int32, device=device)
        self.centroids = torch.zeros(batch, n_kv_heads, n_clusters, 16, dtype=torch.float32, device=device)
        self.members = torch.zeros(batch, n_kv_heads, n, **i32)
        self.offsets = torch.zeros(batch, n_kv_heads, n_clusters + 1, **i32)
        if in_place:
            self.k_sorted = self.v_sorted = None
        else:
            self.k_sorted = torch.zeros(batch, n_kv_heads, n, 128, dtype=torch.bfloat16, device=device)
            self.v_sorted = torch.zeros_like(self.k_sorted)
        self.chunk_centroids = torch.zeros(batch, n_kv_heads, self.max_chunks, 16, dtype=torch.float32,
                                           device=device)
        self.chunk_start = torch.zeros(batch, n_kv_heads, self.max_chunks, **i32)
        self.chunk_len = torch.zeros(batch, n_kv_heads, self.max_chunks, **i32)
        self.n_chunks = torch.zeros(batch, n_kv_heads, **i32)

    def c(self) -> rtp_clusters:
        return rtp_clusters(self.clu_end, self.n_clusters, _ptr(self.centroids), _ptr(self.members),
                            _ptr(self.offsets), _ptr(self.k_sorted), _ptr(self.v_sorted), _ptr(self.chunk_centroids),
                            _ptr(self.chunk_start), _ptr(self.chunk_len), _ptr(self.n_chunks))


def rtp_cache_cluster_workspace_bytes(cfg: AttnConfig, clu_end: int) -> int:
    c = cfg.c()
    return int(_lib.rtp_cache_cluster_workspace_bytes(ctypes.byref(c), int(clu_end)))


def rtp_cache_cluster(cfg: AttnConfig, kinds, iters: int, kcache, vcache, proj, clusters: Clusters, workspace,
                      ws_bytes: int, stream=None) -> None:
    c, cl = cfg.c(), clusters.c()
    _check("rtp_cache_cluster", _lib.rtp_cache_cluster(ctypes.byref(c), _kinds(kinds), int(iters), _ptr(kcache),
                                                       _ptr(vcache), _ptr(proj), ctypes.byref(cl), _ptr(workspace),
                                                       int(ws_bytes), _stream(stream)))


def rtp_decode_clustered_workspace_bytes(cfg: AttnConfig, kinds, cache_len: int, clu_end: int) -> int:
    c = cfg.c()
    return int(_lib.rtp_decode_clustered_workspace_bytes(ctypes.byref(c), _kinds(kinds), int(cache_len),
                                                         int(clu_end)))


def rtp_sparse_decode_clustered(cfg: AttnConfig, kinds, cache_len: int, q, kcache, vcache, proj, clusters: Clusters,
                                o, workspace, ws_bytes: int, sel_out=None, cnt_out=None, stream=None) -> None:
    c, cl = cfg.c(), clusters.c()
    _check("rtp_sparse_decode_clustered",
           _lib.rtp_sparse_decode_clustered(ctypes.byref(c), _kinds(kinds), int(cache_len), _ptr(q), _ptr(kcache),
                                            _ptr(vcache), _ptr(proj), ctypes.byref(cl), _ptr(o), _ptr(workspace),
                                            int(ws_bytes), _ptr(sel_out), _ptr(cnt_out), _stream(stream)))


def cluster_cache(kcache, vcache, proj, kinds, *, clu_end: int, n_clusters: int, iters: int = 8, block: int = 128,
                  stream=None, in_place: bool = False) -> Clusters:
    """k-means clustering of rows [block, clu_end) of the retrieval heads of a
    cache [batch][n_kv_heads][capacity][128]; returns the Clusters arrays
    (in_place: without the cluster-ordered copy of K/V)."""
    B, H, cap = kcache.shape[0], kcache.shape[1], kcache.shape[2]
    cfg = AttnConfig(B, cap, H, H, 1, block, 0, 1)
    cl = Clusters(B, H, clu_end, n_clusters, block, kcache.device, in_place=in_place)
    ws_bytes = rtp_cache_cluster_workspace_bytes(cfg, clu_end)
    if ws_bytes == 0:
        raise RtpError("rtp_cache_cluster_workspace_bytes", RTP_ERR_INVALID_ARG)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=kcache.device)
    rtp_cache_cluster(cfg, kinds, iters, kcache, vcache, proj, cl, ws, ws_bytes, stream)
    return cl


def sparse_decode_clustered_step(q, kcache, vcache, proj, kinds, clusters: Clusters, *, window: int,
                                 block: int = 128, topk: int = 32, scale: float = 0.0, cache_len: int | None = None,
                                 stream=None, return_selection: bool = False):
    """One decode step with clustered retrieval heads; returns o (and (sel, cnt))."""
    B, Hq = q.shape[0], q.shape[1]
    Hkv, cap = kcache.shape[1], kcache.shape[2]
    Lc = cap if cache_len is None else int(cache_len)
    cfg = AttnConfig(B, cap, Hq, Hkv, window, block, topk, 1, scale)
    ws_bytes = rtp_decode_clustered_workspace_bytes(cfg, kinds, Lc, clusters.clu_end)
    if ws_bytes == 0:
        raise RtpError("rtp_decode_clustered_workspace_bytes", RTP_ERR_INVALID_ARG)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    sel = cnt = None
    if return_selection:
        kmax = 1 + (Lc - clusters.clu_end + 127) // 128 + topk
        sel = torch.full((B, Hkv, kmax), -1, dtype=torch.int32, device=q.device)
        cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=q.device)
    rtp_sparse_decode_clustered(cfg, kinds, Lc, q, kcache, vcache, proj, clusters, o, ws, ws_bytes, sel, cnt, stream)
    return (o, sel, cnt) if return_selection else o


def rtp_last_device_status(stream=None) -> int:
    return int(_lib.rtp_last_device_status(_stream(stream)))


def rtp_selftest_bounded_wait(limit_ms: int, stream=None) -> int:
    """Runs the bounded-wait self-test; returns the status (RTP_ERR_TIMEOUT expected)."""
    return int(_lib.rtp_selftest_bounded_wait(int(limit_ms), _stream(stream)))


def rtp_version() -> int:
    return int(_lib.rtp_version())


# ------------------------------------------------------------ conveniences


class Plan:
    """Owns a routing plan (rtp_route_heads / rtp_plan_destroy)."""

    def __init__(self, cfg: AttnConfig, kinds, stream=None, q_range: tuple | None = None,
                 key_begin: int | None = None):
        """q_range: a ranged plan (rtp_route_heads_range); with key_begin as
        well, a split plan (rtp_route_heads_split) whose first n_local items
        see only keys >= key_begin."""
        self.cfg = cfg
        self.kinds = list(kinds)
        self.q_range = (0, cfg.seq) if q_range is None else (int(q_range[0]), int(q_range[1]))
        if key_begin is not None:
            self.handle = rtp_route_heads_split(cfg, kinds, self.q_range[0], self.q_range[1], key_begin, stream)
        elif q_range is None:
            self.handle = rtp_route_heads(cfg, kinds, stream)
        else:
            self.handle = rtp_route_heads_range(cfg, kinds, self.q_range[0], self.q_range[1], stream)
        self.n_items = rtp_plan_num_items(self.handle)
        self.n_local = rtp_plan_num_local_items(self.handle)
        self.n_sparse = rtp_plan_num_sparse(self.handle)
        self.slot_heads = rtp_plan_sparse_heads(self.handle)

    def close(self):
        if self.handle:
            rtp_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def buffers(self, device, per_head: bool = False) -> dict:
        """Indexer / selection buffers for this plan (allocated with torch);
        per_head adds those of the per-head selection."""
        c = self.cfg
        nb = c.seq // c.block
        ns = max(self.n_sparse, 0)
        bufs = dict(
            centroids=torch.empty(c.batch, ns, nb, 16, dtype=torch.float32, device=device),
            qbar=torch.empty(c.batch, ns, nb, 16, dtype=torch.float32, device=device),
            sel=torch.empty(c.batch, ns, nb, c.kmax, dtype=torch.int32, device=device),
            sel_cnt=torch.empty(c.batch, ns, nb, dtype=torch.int32, device=device),
        )
        if per_head:
            G = c.n_q_heads // c.n_kv_heads
            bufs["qbar_heads"] = torch.empty(c.batch, ns, G, nb, 16, dtype=torch.float32, device=device)
            bufs["sel_heads"] = torch.empty(c.batch, ns, G, nb, c.kmax, dtype=torch.int32, device=device)
            bufs["cnt_heads"] = torch.empty(c.batch, ns, G, nb, dtype=torch.int32, device=device)
        return bufs

    def run(self, q, k, v, proj, o, bufs: dict, stream=None, dynamic: dict | None = None,
            score: str = "mean") -> None:
        """One layer: indexer + selection (if any retrieval slot) + prefill.

        dynamic: None for the fixed top-k selection, else a dict with `mass`
        and optionally `min_k` (default 0) and `beta` (default: softmax scale
        / group) for rtp_block_select_dynamic (topk is then the cap).
        score: "mean" (the query-block summary) or "rowmax" (the largest
        low-rank logit over the block's rows, rtp_block_select_rowmax) for the
        fixed top-k selection, or "heads" (one selection per query head:
        rtp_indexer_project_heads, rtp_block_select_heads and
        rtp_hybrid_prefill_heads; bufs from buffers(device, per_head=True)).
        """
        if score not in ("mean", "rowmax", "heads") or (score != "mean" and dynamic is not None):
            raise RtpError("Plan.run", RTP_ERR_INVALID_ARG)
        if self.n_sparse > 0 and score == "heads":
            rtp_indexer_project(self.handle, q, k, proj, bufs["centroids"], bufs["qbar"], stream)
            rtp_indexer_project_heads(self.handle, q, proj, bufs["qbar_heads"], stream)
            rtp_block_select_heads(self.handle, bufs["qbar_heads"], bufs["centroids"], bufs["sel_heads"],
                                   bufs["cnt_heads"], stream)
            rtp_hybrid_prefill_heads(self.handle, q, k, v, bufs["sel_heads"], bufs["cnt_heads"], o, stream)
            return
        if self.n_sparse > 0:
            rtp_indexer_project(self.handle, q, k, proj, bufs["centroids"], bufs["qbar"], stream)
            if score == "rowmax":
                rtp_block_select_rowmax(self.handle, q, proj, bufs["centroids"], bufs["sel"], bufs["sel_cnt"],
                                        stream)
            elif dynamic is None:
                rtp_block_select(self.handle, bufs["qbar"], bufs["centroids"], bufs["sel"], bufs["sel_cnt"], stream)
            else:
                beta = dynamic.get("beta")
                rtp_block_select_dynamic(self.handle, bufs["qbar"], bufs["centroids"], dynamic["mass"],
                                         dynamic.get("min_k", 0),
                                         default_selection_beta(self.cfg) if beta is None else beta, bufs["sel"],
                                         bufs["sel_cnt"], stream)
            rtp_hybrid_prefill(self.handle, q, k, v, bufs["sel"], bufs["sel_cnt"], o, stream)
        else:
            rtp_hybrid_prefill(self.handle, q, k, v, None, None, o, stream)


class HostPipeline:
    """Prefill of layers whose Q/K/V/O live in host memory, chunked so that
    uploads, kernels and downloads overlap (rtp_pipeline_create /
    rtp_hybrid_prefill_host).  Owns the device staging buffers."""

    def __init__(self, cfg: AttnConfig, kinds, n_chunks: int = 8, device="cuda", stream=None):
        self.cfg = cfg
        self.handle = rtp_pipeline_create(cfg, kinds, n_chunks, stream)
        c = cfg
        qs = (c.batch, c.n_q_heads, c.seq, 128)
        ks = (c.batch, c.n_kv_heads, c.seq, 128)
        bf = dict(dtype=torch.bfloat16, device=device)
        self.q, self.k, self.v, self.o = (torch.empty(qs, **bf), torch.empty(ks, **bf), torch.empty(ks, **bf),
                                          torch.empty(qs, **bf))
        self.plan = Plan(cfg, kinds, stream)  # for the shapes of the selection buffers
        self.bufs = self.plan.buffers(device)
        self.plan.close()

    def run(self, q_host, k_host, v_host, proj, o_host, stream=None) -> None:
        b = self.bufs
        rtp_hybrid_prefill_host(self.handle, q_host, k_host, v_host, proj, o_host, self.q, self.k, self.v, self.o,
                                b["centroids"], b["qbar"], b["sel"], b["sel_cnt"], stream)

    def close(self):
        if self.handle:
            rtp_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def hybrid_prefill_layer(q, k, v, kinds, proj=None, *, window: int, block: int = 128, topk: int = 0,
                         n_local: int = 1, scale: float = 0.0, stream=None):
    """Prefill attention of one layer; returns (o, buffers)."""
    cfg = AttnConfig(q.shape[0], q.shape[2], q.shape[1], k.shape[1], window, block, topk, n_local, scale)
    plan = Plan(cfg, kinds, stream)
    bufs = plan.buffers(q.device)
    o = torch.empty_like(q)
    if proj is None:
        proj = torch.zeros(128, 16, dtype=torch.float32, device=q.device)
    plan.run(q, k, v, proj, o, bufs, stream)
    plan.close()
    return o, bufs


def sparse_decode_step(q, kcache, vcache, centroids, proj, kinds, *, window: int, block: int = 128, topk: int = 32,
                       n_local: int = 4, scale: float = 0.0, stream=None, return_selection: bool = False,
                       cache_len: int | None = None):
    """One decode step; returns o (and (sel, cnt) when asked).

    The caches are [batch][n_kv_heads][capacity][128]; the first `cache_len`
    rows (default: all) are the cached tokens, the last of them the new one.
    """
    B, Hq = q.shape[0], q.shape[1]
    Hkv, cap = kcache.shape[1], kcache.shape[2]
    Lc = cap if cache_len is None else int(cache_len)
    if not 1 <= Lc <= cap:
        raise RtpError("rtp_sparse_decode", RTP_ERR_INVALID_ARG)
    cfg = AttnConfig(B, cap, Hq, Hkv, window, block, topk, n_local, scale)
    ws_bytes = rtp_decode_workspace_bytes(cfg, kinds, Lc)
    if ws_bytes == 0:
        raise RtpError("rtp_decode_workspace_bytes", RTP_ERR_INVALID_ARG)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    sel = cnt = None
    if return_selection:
        sel = torch.full((B, Hkv, cfg.kmax), -1, dtype=torch.int32, device=q.device)
        cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=q.device)
    rtp_sparse_decode(cfg, kinds, Lc, q, kcache, vcache, centroids, proj, o, ws, ws_bytes, sel, cnt, stream)
    return (o, sel, cnt) if return_selection else o


class DecodeCache:
    """A KV cache of fixed capacity with the block centroids decode scores.

    Tensors are allocated once ([batch][n_kv_heads][capacity][128] bf16 K and
    V, [batch][n_kv_heads][capacity // block][16] fp32 centroids); tokens are
    added with `append` (rtp_cache_append) or in bulk with `load` (a prefill's
    K/V, followed by rtp_cache_centroids), and `decode` runs rtp_sparse_decode
    over the rows held so far.
    """

    def __init__(self, batch: int, n_kv_heads: int, capacity: int, kinds, proj, *, block: int = 128,
                 device="cuda"):
        self.kinds = [int(x) for x in kinds]
        self.block = block
        self.capacity = capacity
        self.length = 0
        self.proj = proj.to(device=device, dtype=torch.float32).contiguous()
        self.k = torch.zeros(batch, n_kv_heads, capacity, 128, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros_like(self.k)
        self.centroids = torch.zeros(batch, n_kv_heads, capacity // block, 16, dtype=torch.float32, device=device)

    def _cfg(self, n_q_heads: int = 0, window: int = 1, topk: int = 0, n_local: int = 1, scale: float = 0.0):
        B, H = self.k.shape[0], self.k.shape[1]
        return AttnConfig(B, self.capacity, n_q_heads or H, H, window, self.block, topk, n_local, scale)

    def load(self, k, v, stream=None) -> None:
        """Replace the contents by k, v [batch][n_kv_heads][n][128] and build their centroids."""
        n = k.shape[2]
        if n > self.capacity:
            raise RtpError("rtp_cache_centroids", RTP_ERR_INVALID_ARG)
        self.k[:, :, :n].copy_(k)
        self.v[:, :, :n].copy_(v)
        self.length = n
        if n > 0:
            rtp_cache_centroids(self._cfg(), self.kinds, n, self.k, self.proj, self.centroids, stream)

    def append(self, k_new, v_new, stream=None) -> None:
        """Append one token per sequence (k_new, v_new [batch][n_kv_heads][128] or [..][1][128])."""
        rtp_cache_append(self._cfg(), self.kinds, self.length, k_new.contiguous(), v_new.contiguous(), self.k, self.v,
                         self.proj, self.centroids, stream)
        self.length += 1

    def decode(self, q, *, window: int, topk: int = 32, n_local: int = 4, scale: float = 0.0, stream=None,
               return_selection: bool = False):
        """One decode step for q [batch][n_q_heads][1][128] over the rows held."""
        return sparse_decode_step(q, self.k, self.v, self.centroids, self.proj, self.kinds, window=window,
                                  block=self.block, topk=topk, n_local=n_local, scale=scale, stream=stream,
                                  return_selection=return_selection, cache_len=self.length)
