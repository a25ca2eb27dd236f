"""The benchmark's FLOP accounting against brute-force counts.

bench.py reports algorithmic TFLOP/s = 4 * 128 * G * (visible query-key
pairs) / time, the pairs coming from closed forms per head kind
(bench.algorithmic_pairs).  Here the closed forms are compared with a
brute-force count over an explicit visibility mask built from the rules
(i - W < j <= i for streaming heads, j <= i for full heads, j <= i inside
the selected blocks for sparse heads, the selection being the oracle's:
block 0, the k best candidates by score and the L local blocks), and the
full-size totals are compared with figures worked out separately, before
the bench existed, from the configurations' shapes (1.796e14 for the
1M-token layer, 2.206e14 and 8.264e14 for the 48-layer 32K and 128K
models).
"""

import numpy as np
import pytest

import bench
import oracle
from swa_hybrid_attention_b200 import inputs


def brute_pairs(kind, n, window, block, topk, n_local, rng):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    m = j <= i
    if kind == inputs.SWA:
        m &= j > i - window
    elif kind == inputs.SPARSE:
        nb = n // block
        C = rng.standard_normal((nb, 16))
        Q = rng.standard_normal((nb, 16))
        sel, cnt, _ = oracle.select(Q, C, np.arange(nb), topk, n_local)
        allowed = np.zeros((nb, nb), dtype=bool)
        for t in range(nb):
            allowed[t, sel[t, :cnt[t]]] = True
        m &= allowed[i // block, j // block]
    return int(m.sum())


@pytest.mark.parametrize("n,window,block,topk,n_local", [
    (512, 100, 64, 2, 1), (1024, 256, 64, 3, 2), (1024, 1, 128, 0, 1), (1024, 5000, 128, 64, 1),
    (1984, 300, 64, 5, 2), (2048, 512, 128, 4, 4)])
def test_pairs_closed_forms_equal_brute_force(n, window, block, topk, n_local):
    rng = np.random.default_rng(n + topk)
    for kind in (inputs.SWA, inputs.FULL, inputs.SPARSE):
        got = bench.algorithmic_pairs(kind, n, window, block, topk, n_local)
        assert got == brute_pairs(kind, n, window, block, topk, n_local, rng), kind


@pytest.mark.parametrize("wid,layers,expected", [(3, [0], 1.796e14), (1, range(48), 2.206e14),
                                                 (2, range(48), 8.264e14)])
def test_full_size_flops_match_the_published_figures(wid, layers, expected):
    w = inputs.workload(wid)
    total = sum(bench.layer_flops(w, w.kinds[layer])[0] for layer in layers)
    assert abs(total - expected) <= 1e-3 * expected, total


def test_decode_and_indexer_bytes_match_the_published_figures():
    """The byte counts behind the decode and indexer roofline fractions: 95.0 MB
    and 7.3e8 FLOPs per 8 x 256K decode step (37 blocks of 128 keys for each of
    three retrieval heads, the 8192-key window, centroids, q and o, per
    sequence), and 2.42 GB per indexer launch on the 1M-token layer (K of the
    retrieval head and Q of its group of eight, plus the centroids and
    summaries)."""
    w = inputs.workload(4)
    bytes_, flops = bench.decode_work(w, w.kinds[0], w.cache_len)
    assert abs(bytes_ - 95.0e6) <= 1e-3 * 95.0e6, bytes_
    assert abs(flops - 7.3e8) <= 1e-2 * 7.3e8, flops
    w3 = inputs.workload(3)
    ib = bench.indexer_bytes(w3, w3.kinds[0])
    assert abs(ib - 2.42e9) <= 5e-3 * 2.42e9, ib
