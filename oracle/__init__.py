"""CPU oracle for headwise hybrid (SWA + sparse retrieval) attention.

TEST INFRASTRUCTURE ONLY: the plain fp64 statement of what the attention
path computes, used to check the CUDA library.  Only the tests, the package
smoke check and the CPU-baseline leg of the benchmark import this module;
the library never does, and this module never imports the library.

Most of the arithmetic lives in oracle.cpp (C++17, fp64, std::thread); this
file compiles it with g++ on first use and marshals numpy arrays through
ctypes.  Two functions are written here instead: attention_rows_mm, the same
exact attention as attention_rows with the logits and weighted sums of each
query block's rows taken as fp64 matrix products (torch on the CPU, fast
enough for tens of thousands of rows at 1M keys), and round_bf16, the
single rounding of an fp64 result to bf16 for comparison.
Each function states the passage of the RTPurbo / RTPurboV2 pages it
follows (see the header of oracle.cpp for the page titles).

Pinned by the not-gpu tests (tests/test_oracle_pins.py) against brute-force
masked attention (both attention statements), torch's scaled-dot-product
attention in fp64 on CPU, exact nearest-even rounding by rational
arithmetic, full sorts, closed forms and invariants; tests/test_oracle_mutants.py
checks that each of a list of planted mistakes in this package makes those pins
fail.  The pages print no worked example, so no value here is tied to the
authors' own implementation.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

SWA, FULL, SPARSE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (g++ -O2, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-Wall", "-o", _LIB, _SRC]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        D = ctypes.c_double
        _lib.oracle_project_rows.argtypes = [P, L, I, P, I, P]
        _lib.oracle_centroids.argtypes = [P, L, I, I, P, I, P]
        _lib.oracle_qbar.argtypes = [P, I, L, I, I, P, I, P]
        _lib.oracle_scores.argtypes = [P, P, L, I, P]
        _lib.oracle_select.argtypes = [P, P, L, I, P, L, I, I, I, P, P, P]
        _lib.oracle_select_dynamic.argtypes = [P, P, L, I, P, L, I, I, I, D, I, D, P, P, P, P]
        _lib.oracle_rowmax_scores.argtypes = [P, I, L, I, I, P, I, P, L, L, P]
        _lib.oracle_select_rowmax.argtypes = [P, I, L, I, I, P, I, P, L, P, L, I, I, I, P, P, P]
        _lib.oracle_kmeans.argtypes = [P, L, I, I, I, P, P]
        _lib.oracle_attention_keys.argtypes = [P, I, P, P, I, P, L, D, P]
        _lib.oracle_attention_rows.argtypes = [P, P, L, P, P, L, I, I, L, I, P, P, I, D, P]
        _lib.oracle_attention_probs.argtypes = [P, L, P, L, I, I, L, I, P, P, I, D, P]
        _lib.oracle_decode_head.argtypes = [P, I, P, P, L, I, P, L, P, I, I, L, I, I, I, I, I, P, P, P, D, P]
        for f in ("oracle_project_rows", "oracle_centroids", "oracle_qbar", "oracle_scores", "oracle_select",
                  "oracle_select_dynamic", "oracle_rowmax_scores", "oracle_select_rowmax", "oracle_kmeans", "oracle_attention_keys",
                  "oracle_attention_rows", "oracle_attention_probs", "oracle_decode_head"):
            getattr(_lib, f).restype = None
    return _lib


def _bf16_bits(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 array of its bit patterns.

    Accepts a torch bf16 tensor (any device) or a uint16 numpy array.
    """
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16))


def _f32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float32)
    return np.ascontiguousarray(x.detach().cpu().float().numpy())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def project_rows(x, proj) -> np.ndarray:
    """Low-rank projection of bf16 rows [n, 128] -> fp64 [n, 16] (RTPurboV2 page, r = 16)."""
    xb = _bf16_bits(x).reshape(-1, 128)
    p = _f32(proj)
    r = p.shape[1]
    out = np.empty((xb.shape[0], r), dtype=np.float64)
    _load().oracle_project_rows(_ptr(xb), xb.shape[0], 128, _ptr(p), r, _ptr(out))
    return out


def centroids(k_head, block: int, proj) -> np.ndarray:
    """Block centroids of one KV head's keys [N, 128] -> fp64 [N/B, 16] (RTPurboV2 page, clustering)."""
    kb = _bf16_bits(k_head).reshape(-1, 128)
    p = _f32(proj)
    r = p.shape[1]
    n = kb.shape[0]
    out = np.empty((n // block, r), dtype=np.float64)
    _load().oracle_centroids(_ptr(kb), n, 128, block, _ptr(p), r, _ptr(out))
    return out


def qbar(q_group, block: int, proj) -> np.ndarray:
    """Query-block summaries of one group's heads [G, N, 128] -> fp64 [N/B, 16]."""
    qb = _bf16_bits(q_group)
    G = qb.shape[0]
    qb = qb.reshape(G, -1, 128)
    n = qb.shape[1]
    p = _f32(proj)
    r = p.shape[1]
    out = np.empty((n // block, r), dtype=np.float64)
    _load().oracle_qbar(_ptr(qb), G, n, 128, block, _ptr(p), r, _ptr(out))
    return out


def scores(qbar_row: np.ndarray, C: np.ndarray) -> np.ndarray:
    """s_j = qbar . c_j for every block j (fp64)."""
    q = np.ascontiguousarray(qbar_row, dtype=np.float64)
    c = np.ascontiguousarray(C, dtype=np.float64)
    out = np.empty(c.shape[0], dtype=np.float64)
    _load().oracle_scores(_ptr(q), _ptr(c), c.shape[0], c.shape[1], _ptr(out))
    return out


def select(qbar_rows: np.ndarray, C: np.ndarray, t_list, topk: int, n_local: int):
    """Block selection (sink + top-k by (score desc, index asc) + local).

    Returns (sel [nq, kmax] int32 padded with -1, cnt [nq], kth_score [nq]).
    """
    q = np.ascontiguousarray(qbar_rows, dtype=np.float64)
    c = np.ascontiguousarray(C, dtype=np.float64)
    t = np.ascontiguousarray(t_list, dtype=np.int32)
    nq = t.shape[0]
    kmax = topk + 1 + n_local
    sel = np.empty((nq, kmax), dtype=np.int32)
    cnt = np.empty(nq, dtype=np.int32)
    kth = np.empty(nq, dtype=np.float64)
    _load().oracle_select(_ptr(q), _ptr(c), c.shape[0], c.shape[1], _ptr(t), nq, topk, n_local, kmax, _ptr(sel),
                          _ptr(cnt), _ptr(kth))
    return sel, cnt, kth


def rowmax_scores(q_group, proj, C: np.ndarray, t: int, block: int) -> np.ndarray:
    """Row-max scores of query block t (the alternative to the block mean as
    the query-side aggregate of the RTPurboV2 indexer): u_i = sum_h P^T q_{h,i}
    over the block's rows, s_j = max_i u_i . c_j for every block j (fp64).
    q_group: the group's heads [G, N, 128] bf16; C: [nb, 16]."""
    qb = _bf16_bits(q_group)
    G = qb.shape[0]
    qb = qb.reshape(G, -1, 128)
    p = _f32(proj)
    c = np.ascontiguousarray(C, dtype=np.float64)
    out = np.empty(c.shape[0], dtype=np.float64)
    _load().oracle_rowmax_scores(_ptr(qb), G, qb.shape[1], 128, block, _ptr(p), p.shape[1], _ptr(c), c.shape[0],
                                 int(t), _ptr(out))
    return out


def select_rowmax(q_group, proj, C: np.ndarray, t_list, block: int, topk: int, n_local: int):
    """Block selection with row-max scores and the fixed rule (sink + top-k by
    (score desc, index asc) + local).  Returns (sel, cnt, kth_score) as select."""
    qb = _bf16_bits(q_group)
    G = qb.shape[0]
    qb = qb.reshape(G, -1, 128)
    p = _f32(proj)
    c = np.ascontiguousarray(C, dtype=np.float64)
    t = np.ascontiguousarray(t_list, dtype=np.int32)
    nq = t.shape[0]
    kmax = topk + 1 + n_local
    sel = np.empty((nq, kmax), dtype=np.int32)
    cnt = np.empty(nq, dtype=np.int32)
    kth = np.empty(nq, dtype=np.float64)
    _load().oracle_select_rowmax(_ptr(qb), G, qb.shape[1], 128, block, _ptr(p), p.shape[1], _ptr(c), c.shape[0],
                                 _ptr(t), nq, topk, n_local, kmax, _ptr(sel), _ptr(cnt), _ptr(kth))
    return sel, cnt, kth


def select_dynamic(qbar_rows: np.ndarray, C: np.ndarray, t_list, cap: int, n_local: int, mass: float,
                   min_k: int, beta: float):
    """Dynamic block selection (RTPurboV2 page: the budget should vary by head,
    length and query instead of a fixed top-k).

    The shortest prefix of the candidates in (score desc, index asc) order
    whose softmax weights exp(beta * (s - max s)) reach `mass` of their total,
    clamped to [min_k, cap], plus the sink and local blocks.
    Returns (sel [nq, cap+1+n_local] int32 padded with -1, cnt [nq],
    cum_lo [nq], cum_hi [nq]): the selected mass fraction without / with the
    last candidate taken.
    """
    q = np.ascontiguousarray(qbar_rows, dtype=np.float64)
    c = np.ascontiguousarray(C, dtype=np.float64)
    t = np.ascontiguousarray(t_list, dtype=np.int32)
    nq = t.shape[0]
    kmax = cap + 1 + n_local
    sel = np.empty((nq, kmax), dtype=np.int32)
    cnt = np.empty(nq, dtype=np.int32)
    lo = np.empty(nq, dtype=np.float64)
    hi = np.empty(nq, dtype=np.float64)
    _load().oracle_select_dynamic(_ptr(q), _ptr(c), c.shape[0], c.shape[1], _ptr(t), nq, cap, n_local, kmax,
                                  float(mass), int(min_k), float(beta), _ptr(sel), _ptr(cnt), _ptr(lo), _ptr(hi))
    return sel, cnt, lo, hi


def attention_rows(q_rows, pos, k_head, v_head, mode: int, window: int = 0, block: int = 64, sel=None, cnt=None,
                   scale: float | None = None) -> np.ndarray:
    """Exact softmax attention for given rows of one query head -> fp64 [n, 128].

    mode 0 = SWA (i-W < j <= i), 1 = full causal, 2 = sparse over sel[t(i)].
    """
    qb = _bf16_bits(q_rows).reshape(-1, 128)
    pp = np.ascontiguousarray(pos, dtype=np.int64)
    kb = _bf16_bits(k_head).reshape(-1, 128)
    vb = _bf16_bits(v_head).reshape(-1, 128)
    n = kb.shape[0]
    if sel is None:
        sel = np.zeros((1, 1), dtype=np.int32)
        cnt = np.zeros(1, dtype=np.int32)
    s = np.ascontiguousarray(sel, dtype=np.int32)
    c = np.ascontiguousarray(cnt, dtype=np.int32)
    kmax = s.shape[-1]
    sc = 1.0 / np.sqrt(128.0) if scale is None else float(scale)
    out = np.empty((qb.shape[0], 128), dtype=np.float64)
    _load().oracle_attention_rows(_ptr(qb), _ptr(pp), qb.shape[0], _ptr(kb), _ptr(vb), n, 128, mode, window, block,
                                  _ptr(s), _ptr(c), kmax, sc, _ptr(out))
    return out


def attention_probs(q_row, i: int, k_head, mode: int, window: int = 0, block: int = 64, sel=None, cnt=None,
                    scale: float | None = None) -> np.ndarray:
    """Normalised attention weights of one row over all N keys (0 where invisible)."""
    qb = _bf16_bits(q_row).reshape(128)
    kb = _bf16_bits(k_head).reshape(-1, 128)
    n = kb.shape[0]
    if sel is None:
        sel = np.zeros((1, 1), dtype=np.int32)
        cnt = np.zeros(1, dtype=np.int32)
    s = np.ascontiguousarray(sel, dtype=np.int32)
    c = np.ascontiguousarray(cnt, dtype=np.int32)
    sc = 1.0 / np.sqrt(128.0) if scale is None else float(scale)
    out = np.empty(n, dtype=np.float64)
    _load().oracle_attention_probs(_ptr(qb), i, _ptr(kb), n, 128, mode, window, block, _ptr(s), _ptr(c),
                                   s.shape[-1], sc, _ptr(out))
    return out


def decode_head(q_group, kc_head, vc_head, C_head, proj, mode: int, window: int, block: int, topk: int,
                n_local: int, sel=None, cnt=None, scale: float | None = None):
    """Sparse / SWA decode of one sequence and one KV head (query at Lc-1).

    q_group [G, 128] bf16; caches [Lc, 128] bf16; C_head [Lc/B, 16] fp32.
    If sel/cnt are given (one row), that selection is used; otherwise the
    oracle selects.  Returns (out [G,128] fp64, sel [kmax], cnt, kth_score).
    """
    qb = _bf16_bits(q_group).reshape(-1, 128)
    G = qb.shape[0]
    kb = _bf16_bits(kc_head).reshape(-1, 128)
    vb = _bf16_bits(vc_head).reshape(-1, 128)
    Lc = kb.shape[0]
    Cf = _f32(C_head).reshape(-1, 16)
    p = _f32(proj)
    kmax = topk + 1 + n_local
    use_given = sel is not None
    s = np.full(kmax, -1, dtype=np.int32) if sel is None else np.ascontiguousarray(sel, dtype=np.int32).reshape(-1)
    c = np.zeros(1, dtype=np.int32) if cnt is None else np.array([int(np.asarray(cnt).reshape(-1)[0])],
                                                                  dtype=np.int32)
    kth = np.zeros(1, dtype=np.float64)
    sc = 1.0 / np.sqrt(128.0) if scale is None else float(scale)
    out = np.empty((G, 128), dtype=np.float64)
    _load().oracle_decode_head(_ptr(qb), G, _ptr(kb), _ptr(vb), Lc, 128, _ptr(Cf), Cf.shape[0], _ptr(p), 16, mode,
                               window, block, topk, n_local, kmax, int(use_given), _ptr(s), _ptr(c), _ptr(kth), sc,
                               _ptr(out))
    return out, s, int(c[0]), float(kth[0])


def cache_centroids(kcache, cache_len: int, kinds, block: int, proj, C=None) -> np.ndarray:
    """Centroids of the complete blocks of a KV cache (RTPurboV2 page: decode
    scores the centroids of the projected cached keys; clustering the K cache
    after a full-attention prefill).

    kcache: bf16 [batch][H][cap][128] (torch tensor or uint16 bit array).
    Returns fp64 [batch][H][cap // block][16]: for every head of kind SPARSE,
    block b < cache_len // block holds the mean of P^T k_j over the block's
    rows; every other entry is copied from C (NaN when C is None).
    """
    kb = _bf16_bits(kcache)
    nb_, H, cap = kb.shape[0], kb.shape[1], kb.shape[2]
    nbc = cap // block
    out = np.full((nb_, H, nbc, 16), np.nan) if C is None else np.array(C, dtype=np.float64, copy=True)
    n = (cache_len // block) * block
    for b in range(nb_):
        for h in range(H):
            if int(kinds[h]) == SPARSE and n > 0:
                out[b, h, : n // block] = centroids(kb[b, h, :n], block, proj)
    return out


def cache_append(kcache, vcache, C, kinds, pos: int, k_new, v_new, block: int, proj):
    """One token appended to a KV cache of fixed capacity (RTPurboV2 page: a
    block's centroid stands for its keys once all of them are cached).

    Row `pos` of every (sequence, head) becomes k_new / v_new
    ([batch][H][128]).  If that row is the last of its block, the block's
    centroid is (re)computed for every SPARSE head from the cached rows of the
    block; no other centroid changes.  Returns new arrays (kcache, vcache as
    uint16 bf16 bits, C as fp64); the inputs are not modified.
    """
    kc = _bf16_bits(kcache).copy()
    vc = _bf16_bits(vcache).copy()
    Cn = np.array(C, dtype=np.float64, copy=True)
    kc[:, :, pos] = _bf16_bits(k_new).reshape(kc.shape[0], kc.shape[1], 128)
    vc[:, :, pos] = _bf16_bits(v_new).reshape(vc.shape[0], vc.shape[1], 128)
    if (pos + 1) % block == 0:
        blk = (pos + 1) // block - 1
        for b in range(kc.shape[0]):
            for h in range(kc.shape[1]):
                if int(kinds[h]) == SPARSE:
                    Cn[b, h, blk] = centroids(kc[b, h, blk * block:(blk + 1) * block], block, proj)[0]
    return kc, vc, Cn


def kmeans(X: np.ndarray, n_clusters: int, iters: int):
    """Lloyd's k-means on projected keys X [n, r] (RTPurboV2 page: clustering of
    the projected keys).  Evenly spaced initial centroids, nearest centroid by
    squared distance (ties to the lower index), empty clusters keep their
    centroid.  Returns (centroids [nc, r] fp64, assignment [n] int32)."""
    x = np.ascontiguousarray(X, dtype=np.float64)
    n, r = x.shape
    mu = np.empty((n_clusters, r), dtype=np.float64)
    assign = np.zeros(n, dtype=np.int32)
    _load().oracle_kmeans(_ptr(x), n, r, n_clusters, iters, _ptr(mu), _ptr(assign))
    return mu, assign


def cluster_chunks(assign: np.ndarray, row0: int, n_clusters: int, chunk: int = 128):
    """Members of each cluster (key positions row0 + index, ascending) in
    cluster order, and the cluster's members cut into chunks of at most
    `chunk` keys.  Returns (members [n], offsets [nc+1], chunks: list of
    (cluster, start, length) with start an index into members)."""
    a = np.asarray(assign)
    order = np.lexsort((np.arange(a.size), a))  # by cluster, then position
    members = (order + row0).astype(np.int64)
    counts = np.bincount(a, minlength=n_clusters)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    chunks = []
    for c in range(n_clusters):
        for s0 in range(int(offsets[c]), int(offsets[c + 1]), chunk):
            chunks.append((c, s0, min(chunk, int(offsets[c + 1]) - s0)))
    return members, offsets, chunks


def attention_keys(q_group, kc_head, vc_head, keys, scale: float | None = None) -> np.ndarray:
    """Exact attention of the group's query rows [G, 128] over the listed cached keys -> fp64 [G, 128]."""
    qb = _bf16_bits(q_group).reshape(-1, 128)
    kb = _bf16_bits(kc_head).reshape(-1, 128)
    vb = _bf16_bits(vc_head).reshape(-1, 128)
    kk = np.ascontiguousarray(keys, dtype=np.int64)
    sc = 1.0 / np.sqrt(128.0) if scale is None else float(scale)
    out = np.empty((qb.shape[0], 128), dtype=np.float64)
    _load().oracle_attention_keys(_ptr(qb), qb.shape[0], _ptr(kb), _ptr(vb), 128, _ptr(kk), kk.size, sc, _ptr(out))
    return out


def decode_clustered_keys(members, chunks, chosen, block: int, clu_end: int, cache_len: int) -> np.ndarray:
    """Keys a clustered decode step attends to: the sink block, the keys of the
    chosen chunks (all inside [block, clu_end)) and the unclustered tail
    [clu_end, cache_len), ascending."""
    keys = list(range(0, min(block, cache_len)))
    for x in chosen:
        _, s0, n = chunks[int(x)]
        keys.extend(int(k) for k in members[s0:s0 + n])
    keys.extend(range(clu_end, cache_len))
    return np.array(sorted(keys), dtype=np.int64)


def topk_chunks(qbar_row: np.ndarray, chunk_centroids: np.ndarray, topk: int) -> np.ndarray:
    """The topk chunks by (score desc, index asc), ascending."""
    s = scores(qbar_row, chunk_centroids)
    order = np.lexsort((np.arange(s.size), -s))
    return np.sort(order[:topk])


# Largest finite bf16: fraction 1.1111111b, exponent 127.
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 in one step (ties to even), returned as fp64.

    bf16 has fp32's 8-bit exponent and 7 fraction bits.  A normal value keeps
    the top 7 of fp64's 52 fraction bits, rounded half-to-even on the 45 bits
    dropped; a value below the smallest normal bf16 (2^-126) is rounded to a
    multiple of 2^-133 (the subnormal spacing); a value whose rounding exceeds
    the largest finite bf16 becomes infinite; NaN stays NaN.  (Rounding to
    fp32 first and then to bf16 would round twice, which differs when the
    first rounding lands exactly half-way between two bf16 values.)
    """
    a = np.array(x, dtype=np.float64, copy=True)
    u = a.view(np.uint64)
    keep = np.uint64(45)
    lsb = (u >> keep) & np.uint64(1)
    r = ((u + np.uint64((1 << 44) - 1) + lsb) >> keep) << keep
    out = r.view(np.float64).copy()
    tiny = np.abs(a) < 2.0 ** -126
    out[tiny] = np.round(a[tiny] * 2.0 ** 133) * 2.0 ** -133  # np.round: half to even
    over = np.isfinite(a) & (np.abs(out) > _BF16_MAX)
    out[over] = np.copysign(np.inf, a[over])
    out[np.isnan(a)] = np.nan
    return out


def attention_rows_mm(q_rows, pos, k_head, v_head, mode: int, window: int = 0, block: int = 64, sel=None,
                      cnt=None, scale: float | None = None) -> np.ndarray:
    """Exact softmax attention for given rows of one query head -> fp64 [n, 128].

    The same definition as attention_rows (RTPurbo page, opening section:
    streaming heads keep a window, full heads every earlier token; the "Full
    Attention Strikes Back" summary: exact softmax over the selected set),
    computed with fp64 matrix products: the rows are taken in groups that
    share a query block t = i // block, and for each group
      J      = a key range (or the selected blocks of t) holding every key
               visible to any row of the group,
      s_ij   = scale * q_i . k_j for j in J         (one fp64 matmul),
      s_ij   = -inf where j is not visible to i      (i-W < j <= i for SWA,
               j <= i for full and, inside the selected blocks, sparse),
      O_i    = sum_j p_ij v_j / sum_j p_ij,  p_ij = exp(s_ij - max_j s_ij)
                                                     (one fp64 matmul).
    mode 0 = SWA, 1 = full causal, 2 = sparse over sel[t] (first cnt[t]
    entries).  A row with no visible key gets zeros.
    """
    import torch

    qb = torch.from_numpy(_bf16_bits(q_rows).reshape(-1, 128).view(np.int16)).view(torch.bfloat16)
    kb = torch.from_numpy(_bf16_bits(k_head).reshape(-1, 128).view(np.int16)).view(torch.bfloat16)
    vb = torch.from_numpy(_bf16_bits(v_head).reshape(-1, 128).view(np.int16)).view(torch.bfloat16)
    pp = np.ascontiguousarray(pos, dtype=np.int64)
    sc = 1.0 / np.sqrt(128.0) if scale is None else float(scale)
    out = np.zeros((qb.shape[0], 128), dtype=np.float64)
    tq = pp // block
    for t in np.unique(tq):
        idx = np.nonzero(tq == t)[0]
        i = torch.from_numpy(pp[idx])
        hi = int(pp[idx].max())
        if mode == SWA:
            keys = torch.arange(max(0, int(pp[idx].min()) - window + 1), hi + 1)
        elif mode == FULL:
            keys = torch.arange(0, hi + 1)
        else:
            blocks = [int(b) for b in np.asarray(sel)[t, :int(np.asarray(cnt)[t])]]
            keys = torch.cat([torch.arange(b * block, (b + 1) * block) for b in blocks]) if blocks else \
                torch.zeros(0, dtype=torch.int64)
            keys = keys[keys <= hi]
        if keys.numel() == 0:
            continue
        visible = keys[None, :] <= i[:, None]
        if mode == SWA:
            visible &= keys[None, :] > i[:, None] - window
        qd = qb[torch.from_numpy(idx)].double()
        s = (qd @ kb[keys].double().T) * sc
        s = s.masked_fill(~visible, float("-inf"))
        m = s.max(dim=1, keepdim=True).values
        ok = torch.isfinite(m[:, 0])
        p = torch.exp(s - torch.where(torch.isfinite(m), m, torch.zeros_like(m)))
        o = (p @ vb[keys].double()) / p.sum(dim=1, keepdim=True)
        o[~ok] = 0.0
        out[idx] = o.numpy()
    return out
