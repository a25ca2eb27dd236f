"""Pins of the CPU oracle against things other than itself.

The pages print no worked example, so the oracle is pinned by construction:
  * brute-force dense attention over an explicit boolean mask built here from
    the visibility rules (window, causal, selected blocks);
  * torch's scaled_dot_product_attention on CPU in fp64 with the same mask;
  * invariants: SWA with W >= N equals full causal, sparse attention whose
    selection covers every block equals full causal, each row of weights is
    a distribution, V = 1 gives O = 1, a single visible key returns its V row;
  * projection/centroids: coordinate selection is exact, centroids are linear
    (mean of projections = projection of the mean), random projector equals a
    plain matrix product;
  * selection: brute-force scoring + full sort with the (score desc, index asc)
    rule, a planted dominant block, degenerate sizes;
  * decode: equals the last prefill row when both use the same selection;
  * KV-cache maintenance: filling a cache one append at a time gives the
    centroids of a plain numpy mean-then-project of each complete block, only
    the appended row and (on a block's last row) that block's centroid change,
    and non-retrieval heads' centroids are never written.
"""

import numpy as np
import pytest
import torch

import oracle
from swa_hybrid_attention_b200 import inputs

SCALE = 1.0 / np.sqrt(128.0)


def widen(x):
    return x.float().double().cpu().numpy()


def mask_matrix(n, mode, window=0, block=64, sel=None, cnt=None):
    """Explicit [n, n] visibility mask, built from the rules directly."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    m = j <= i
    if mode == oracle.SWA:
        m = m & (j > i - window)
    elif mode == oracle.SPARSE:
        allowed = np.zeros((n // block + 1, n // block + 1), dtype=bool)
        for t in range(n // block):
            for e in range(cnt[t]):
                allowed[t, sel[t, e]] = True
        m = m & allowed[i // block, j // block]
    return m


def dense_reference(q, k, v, m):
    s = (q @ k.T) * SCALE
    s = np.where(m, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v


def random_selection(n, block, kmax, rng):
    """A random valid selection per query block: diagonal always, sink, random earlier blocks."""
    nb = n // block
    sel = np.full((nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros(nb, dtype=np.int32)
    for t in range(nb):
        pool = list(range(1, t))
        rng.shuffle(pool)
        chosen = sorted(set([0, t] + pool[: kmax - 2]))
        sel[t, : len(chosen)] = chosen
        cnt[t] = len(chosen)
    return sel, cnt


@pytest.fixture(scope="module")
def small():
    return inputs.small_prefill(384, 2, 1, [oracle.FULL], seed=7)


# The two statements of exact attention: per row (C++) and per query-block
# group with fp64 matrix products (torch).  Every brute-force pin runs on both.
ATTENTION = {"rows": oracle.attention_rows, "mm": oracle.attention_rows_mm}


@pytest.mark.parametrize("impl", sorted(ATTENTION))
@pytest.mark.parametrize("n", [128, 384, 1024])
@pytest.mark.parametrize("mode,window", [(oracle.FULL, 0), (oracle.SWA, 100), (oracle.SWA, 1), (oracle.SWA, 256)])
def test_attention_matches_bruteforce(n, mode, window, impl):
    d = inputs.small_prefill(n, 1, 1, [mode], seed=11 + n)
    q, k, v = d["q"][0, 0], d["k"][0, 0], d["v"][0, 0]
    rows = np.arange(n)
    got = ATTENTION[impl](q, rows, k, v, mode, window)
    ref = dense_reference(widen(q), widen(k), widen(v), mask_matrix(n, mode, window))
    assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("impl", sorted(ATTENTION))
@pytest.mark.parametrize("n,block", [(384, 64), (1024, 128), (1024, 64)])
def test_sparse_attention_matches_bruteforce(n, block, impl):
    rng = np.random.default_rng(n + block)
    d = inputs.small_prefill(n, 1, 1, [oracle.SPARSE], seed=3)
    q, k, v = d["q"][0, 0], d["k"][0, 0], d["v"][0, 0]
    sel, cnt = random_selection(n, block, 5, rng)
    got = ATTENTION[impl](q, np.arange(n), k, v, oracle.SPARSE, 0, block, sel, cnt)
    ref = dense_reference(widen(q), widen(k), widen(v), mask_matrix(n, oracle.SPARSE, 0, block, sel, cnt))
    assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("impl", sorted(ATTENTION))
def test_attention_matches_torch_sdpa_fp64(impl):
    n, block = 512, 64
    rng = np.random.default_rng(5)
    d = inputs.small_prefill(n, 1, 1, [oracle.SPARSE], seed=21)
    q, k, v = d["q"][0, 0], d["k"][0, 0], d["v"][0, 0]
    sel, cnt = random_selection(n, block, 4, rng)
    for mode, window in [(oracle.FULL, 0), (oracle.SWA, 77), (oracle.SPARSE, 0)]:
        m = mask_matrix(n, mode, window, block, sel, cnt)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.double()[None, None], k.double()[None, None], v.double()[None, None],
            attn_mask=torch.from_numpy(m)[None, None], scale=SCALE)[0, 0].numpy()
        got = ATTENTION[impl](q, np.arange(n), k, v, mode, window, block, sel, cnt)
        assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("mode,window,block", [(oracle.FULL, 0, 64), (oracle.SWA, 300, 64), (oracle.SWA, 1, 128),
                                               (oracle.SPARSE, 0, 64), (oracle.SPARSE, 0, 128)])
def test_grouped_attention_equals_row_attention_on_scattered_rows(mode, window, block):
    """Rows in random order from scattered query blocks (several per block,
    one alone, the last ragged block), with a scale: both statements agree."""
    n = 1000
    rng = np.random.default_rng(block + window)
    d = inputs.small_prefill(n, 1, 1, [mode], seed=61)
    q, k, v = d["q"][0, 0], d["k"][0, 0], d["v"][0, 0]
    sel, cnt = random_selection(n + block, block, 6, rng)
    rows = rng.permutation(np.concatenate([rng.choice(n, 40, replace=False), [0, n - 1, 130]]))
    a = oracle.attention_rows(q[rows], rows, k, v, mode, window, block, sel, cnt, 0.07)
    b = oracle.attention_rows_mm(q[rows], rows, k, v, mode, window, block, sel, cnt, 0.07)
    assert np.max(np.abs(a - b)) <= 1e-12


def test_swa_with_window_ge_seq_is_full_bitwise(small):
    q, k, v = small["q"][0, 0], small["k"][0, 0], small["v"][0, 0]
    n = q.shape[0]
    rows = np.arange(n)
    full = oracle.attention_rows(q, rows, k, v, oracle.FULL)
    for w in (n, n + 1, 10 * n):
        swa = oracle.attention_rows(q, rows, k, v, oracle.SWA, w)
        assert np.array_equal(full, swa)


def test_sparse_covering_all_blocks_is_full_bitwise(small):
    q, k, v = small["q"][0, 0], small["k"][0, 0], small["v"][0, 0]
    n, block = q.shape[0], 64
    nb = n // block
    sel = np.tile(np.arange(nb, dtype=np.int32), (nb, 1))
    cnt = np.full(nb, nb, dtype=np.int32)
    rows = np.arange(n)
    full = oracle.attention_rows(q, rows, k, v, oracle.FULL)
    sp = oracle.attention_rows(q, rows, k, v, oracle.SPARSE, 0, block, sel, cnt)
    assert np.array_equal(full, sp)


@pytest.mark.parametrize("mode,window", [(oracle.FULL, 0), (oracle.SWA, 50)])
def test_rows_are_distributions(small, mode, window):
    q, k, v = small["q"][0, 0], small["k"][0, 0], small["v"][0, 0]
    n = q.shape[0]
    for i in (0, 1, 49, 50, 51, 200, n - 1):
        p = oracle.attention_probs(q[i], i, k, mode, window)
        assert abs(p.sum() - 1.0) <= 1e-12
        vis = np.arange(n) <= i
        if mode == oracle.SWA:
            vis &= np.arange(n) > i - window
        assert np.all(p[~vis] == 0.0) and np.all(p[vis] > 0.0)
        # the same weights as the output row (same logits, same scale)
        row = oracle.attention_rows(q[i:i + 1], np.array([i]), k, v, mode, window)[0]
        assert np.max(np.abs(p @ widen(v) - row)) <= 1e-12


def test_ones_value_gives_ones(small):
    q, k = small["q"][0, 0], small["k"][0, 0]
    ones = torch.ones_like(k)
    n = q.shape[0]
    for mode, w in [(oracle.FULL, 0), (oracle.SWA, 7)]:
        o = oracle.attention_rows(q, np.arange(n), k, ones, mode, w)
        assert np.max(np.abs(o - 1.0)) <= 1e-14


def test_single_visible_key_returns_its_value(small):
    q, k, v = small["q"][0, 0], small["k"][0, 0], small["v"][0, 0]
    # row 0 sees only key 0; with W = 1 every row sees only itself
    o0 = oracle.attention_rows(q[:1], np.array([0]), k, v, oracle.FULL)
    assert np.array_equal(o0[0], widen(v[0]))
    n = q.shape[0]
    o = oracle.attention_rows(q, np.arange(n), k, v, oracle.SWA, 1)
    assert np.array_equal(o, widen(v))


def test_scale_enters_the_logits():
    d = inputs.small_prefill(128, 1, 1, [oracle.FULL], seed=2)
    q, k, v = d["q"][0, 0], d["k"][0, 0], d["v"][0, 0]
    m = mask_matrix(128, oracle.FULL)
    s = (widen(q) @ widen(k).T) * 0.3
    s = np.where(m, s, -np.inf)
    p = np.exp(s - s.max(1, keepdims=True))
    ref = (p / p.sum(1, keepdims=True)) @ widen(v)
    got = oracle.attention_rows(q, np.arange(128), k, v, oracle.FULL, scale=0.3)
    assert np.max(np.abs(got - ref)) <= 1e-12


# ----------------------------------------------------------------- projection


def test_lowfreq_projection_selects_coordinates_exactly():
    d = inputs.small_prefill(256, 1, 1, [oracle.SPARSE], seed=9)
    k = d["k"][0, 0]
    got = oracle.project_rows(k, inputs.lowfreq_projector())
    dims = list(range(56, 64)) + list(range(120, 128))
    assert np.array_equal(got, widen(k)[:, dims])


def test_random_projection_is_matrix_product():
    d = inputs.small_prefill(256, 1, 1, [oracle.SPARSE], seed=4)
    k = d["k"][0, 0]
    p = inputs.random_projector(123)
    got = oracle.project_rows(k, p)
    ref = widen(k) @ p.double().numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("block", [64, 128])
def test_centroids_are_linear(block):
    d = inputs.small_prefill(1024, 1, 1, [oracle.SPARSE], seed=6)
    k = d["k"][0, 0]
    p = inputs.random_projector(5)
    got = oracle.centroids(k, block, p)
    mean_k = widen(k).reshape(-1, block, 128).mean(axis=1)
    ref = mean_k @ p.double().numpy()
    assert got.shape == (1024 // block, 16)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_qbar_is_sum_over_heads_of_block_means():
    d = inputs.small_prefill(512, 4, 1, [oracle.SPARSE], seed=8)
    q = d["q"][0]
    p = inputs.random_projector(6)
    got = oracle.qbar(q, 64, p)
    qn = widen(q)  # [G, N, 128]
    ref = sum(qn[h].reshape(-1, 64, 128).mean(axis=1) for h in range(4)) @ p.double().numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


# ------------------------------------------------------------------ selection


def brute_select(qb, C, t, topk, n_local):
    s = C @ qb
    cands = list(range(1, t - n_local + 1))
    if len(cands) > topk:
        cands = sorted(cands, key=lambda j: (-s[j], j))[:topk]
    chosen = set(cands) | {0} | set(range(max(0, t - n_local + 1), t + 1))
    return sorted(chosen)


@pytest.mark.parametrize("nb,topk,n_local", [(32, 16, 2), (40, 5, 3), (9, 4, 1), (64, 1, 0), (12, 20, 2)])
def test_selection_matches_bruteforce(nb, topk, n_local):
    rng = np.random.default_rng(nb * 100 + topk)
    C = rng.standard_normal((nb, 16))
    qb = rng.standard_normal((nb, 16))
    # plant exact ties to exercise the index tie-break
    C[5] = C[7]
    C[nb - 2] = C[3]
    sel, cnt, kth = oracle.select(qb, C, np.arange(nb), topk, n_local)
    for t in range(nb):
        ref = brute_select(qb[t], C, t, topk, n_local)
        assert cnt[t] == len(ref)
        assert list(sel[t, : cnt[t]]) == ref
        assert np.all(sel[t, cnt[t]:] == -1)
        ncand = max(0, t - n_local)
        if ncand > topk:
            s = C @ qb[t]
            kept = [j for j in ref if 1 <= j <= t - n_local]
            assert abs(kth[t] - min(s[j] for j in kept)) <= 1e-12 * (1 + abs(kth[t]))
        else:
            assert np.isnan(kth[t])


def test_selection_picks_planted_block():
    rng = np.random.default_rng(1)
    nb = 64
    C = rng.standard_normal((nb, 16)) * 0.01
    qb = rng.standard_normal((nb, 16))
    C[17] = qb[50] * 10.0  # dominates for query block 50
    sel, cnt, _ = oracle.select(qb, C, np.arange(nb), 1, 2)
    assert list(sel[50, : cnt[50]]) == [0, 17, 49, 50]


def test_selection_small_t_is_full_causal():
    rng = np.random.default_rng(2)
    nb = 16
    C = rng.standard_normal((nb, 16))
    qb = rng.standard_normal((nb, 16))
    sel, cnt, _ = oracle.select(qb, C, np.arange(nb), 8, 2)
    for t in range(0, 11):  # t - L <= k: every earlier block is kept
        assert list(sel[t, : cnt[t]]) == list(range(t + 1))


# ------------------------------------------------------------ row-max scores


def brute_rowmax_scores(q_group, proj, C, t, block):
    """u_i = sum_h q_{h,i} P (fp64, numpy), s_j = max_i u_i . c_j."""
    qg = widen(q_group)[:, t * block:(t + 1) * block]  # [G, B, 128]
    U = qg.sum(axis=0) @ np.asarray(proj, dtype=np.float64)
    return (U @ np.asarray(C, dtype=np.float64).T).max(axis=0)


@pytest.mark.parametrize("G,n,block,topk,n_local", [(2, 512, 64, 3, 1), (4, 1024, 128, 2, 2), (1, 640, 64, 20, 1)])
def test_rowmax_selection_matches_bruteforce(G, n, block, topk, n_local):
    g = torch.Generator().manual_seed(G * 1000 + n)
    q = torch.randn(G, n, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(n, 128, generator=g).to(torch.bfloat16)
    proj = torch.randn(128, 16, generator=g) / 11.3
    C = oracle.centroids(k, block, proj)
    nb = n // block
    sel, cnt, kth = oracle.select_rowmax(q, proj, C, np.arange(nb), block, topk, n_local)
    for t in range(nb):
        s = brute_rowmax_scores(q, proj, C, t, block)
        np.testing.assert_allclose(oracle.rowmax_scores(q, proj, C, t, block), s, rtol=1e-12, atol=1e-12)
        cands = list(range(1, t - n_local + 1))
        if len(cands) > topk:
            cands = sorted(cands, key=lambda j: (-s[j], j))[:topk]
        ref = sorted(set(cands) | {0} | set(range(max(0, t - n_local + 1), t + 1)))
        assert list(sel[t, :cnt[t]]) == ref and np.all(sel[t, cnt[t]:] == -1)


def test_rowmax_with_identical_rows_equals_mean_selection():
    # every row of a block equal (per head): the row maximum is the block mean,
    # so the scores and the selection are those of the query-block summaries
    G, n, block, topk, n_local = 3, 768, 64, 4, 2
    g = torch.Generator().manual_seed(5)
    rows = torch.randn(G, n // block, 1, 128, generator=g).expand(G, n // block, block, 128)
    q = rows.reshape(G, n, 128).to(torch.bfloat16)
    k = torch.randn(n, 128, generator=g).to(torch.bfloat16)
    proj = torch.randn(128, 16, generator=g) / 11.3
    C = oracle.centroids(k, block, proj)
    qb = oracle.qbar(q, block, proj)
    nb = n // block
    for t in range(nb):
        np.testing.assert_allclose(oracle.rowmax_scores(q, proj, C, t, block), oracle.scores(qb[t], C),
                                   rtol=1e-12, atol=1e-12)
    a = oracle.select_rowmax(q, proj, C, np.arange(nb), block, topk, n_local)
    b = oracle.select(qb, C, np.arange(nb), topk, n_local)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_rowmax_score_bounds_the_mean_score():
    G, n, block = 2, 512, 128
    g = torch.Generator().manual_seed(6)
    q = torch.randn(G, n, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(n, 128, generator=g).to(torch.bfloat16)
    proj = torch.randn(128, 16, generator=g) / 11.3
    C = oracle.centroids(k, block, proj)
    qb = oracle.qbar(q, block, proj)
    for t in range(n // block):
        assert np.all(oracle.rowmax_scores(q, proj, C, t, block) >= oracle.scores(qb[t], C) - 1e-12)


def test_per_head_selection_with_identical_heads_equals_the_shared_one():
    # every head of the group the same: the shared summary is G times each
    # head's own, so every head's own selection is the shared selection
    G, n, block, topk, n_local = 4, 1024, 64, 3, 2
    g = torch.Generator().manual_seed(9)
    q1 = torch.randn(1, n, 128, generator=g).to(torch.bfloat16)
    q = q1.expand(G, n, 128).contiguous()
    k = torch.randn(n, 128, generator=g).to(torch.bfloat16)
    proj = torch.randn(128, 16, generator=g) / 11.3
    C = oracle.centroids(k, block, proj)
    nb = n // block
    shared = oracle.qbar(q, block, proj)
    own = oracle.qbar(q[:1], block, proj)
    np.testing.assert_allclose(shared, G * own, rtol=1e-12, atol=1e-12)
    a = oracle.select(shared, C, np.arange(nb), topk, n_local)
    b = oracle.select(own, C, np.arange(nb), topk, n_local)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# --------------------------------------------------------------------- decode


@pytest.mark.parametrize("Lc", [1024, 1025])
def test_decode_equals_last_prefill_row(Lc):
    """The decode step is the prefill's row L_c - 1, also when that row opens
    a new query block (L_c = 1025: block 16, whose own centroid does not
    exist yet)."""
    block, G = 64, 4
    d = inputs.small_prefill(Lc, G, 1, [oracle.SPARSE], seed=31)
    q, k, v = d["q"][0], d["k"][0, 0], d["v"][0, 0]
    p = inputs.lowfreq_projector()
    C = oracle.centroids(k, block, p).astype(np.float32)
    out, sel, cnt, _ = oracle.decode_head(q[:, Lc - 1], k, v, C, p, oracle.SPARSE, 0, block, 4, 2)
    nb = (Lc + block - 1) // block
    t = nb - 1
    sel_full = np.full((nb, sel.shape[0]), -1, dtype=np.int32)
    cnt_full = np.ones(nb, dtype=np.int32)
    sel_full[:, 0] = 0
    sel_full[t] = sel
    cnt_full[t] = cnt
    for h in range(G):
        ref = oracle.attention_rows(q[h, Lc - 1:Lc], np.array([Lc - 1]), k, v, oracle.SPARSE, 0, block, sel_full,
                                    cnt_full)
        assert np.array_equal(out[h], ref[0])
    # the oracle's own selection is the brute-force one on the decode summary
    qb = oracle.project_rows(q[:, Lc - 1], p).sum(axis=0)
    assert list(sel[:cnt]) == brute_select(qb, C.astype(np.float64), t, 4, 2)


def test_decode_attends_to_a_given_selection_as_given():
    """A selection handed to the decode step is used as it is (not replaced
    by the oracle's own top-k): the output equals brute-force attention over
    exactly those blocks."""
    Lc, block, G, topk, n_local = 1000, 64, 2, 4, 2
    d = inputs.small_prefill(Lc, G, 1, [oracle.SPARSE], seed=37)
    q, k, v = d["q"][0], d["k"][0, 0], d["v"][0, 0]
    p = inputs.lowfreq_projector()
    C = oracle.centroids(k, block, p).astype(np.float32)
    given = [0, 3, 7, 14, 15]  # t = 999 // 64 = 15; block 15 holds keys 960..999
    _, own, own_cnt, _ = oracle.decode_head(q[:, Lc - 1], k, v, C, p, oracle.SPARSE, 0, block, topk, n_local)
    assert list(own[:own_cnt]) != given
    sel = np.full(topk + 1 + n_local, -1, dtype=np.int32)
    sel[:len(given)] = given
    out, sel_out, cnt_out, _ = oracle.decode_head(q[:, Lc - 1], k, v, C, p, oracle.SPARSE, 0, block, topk, n_local,
                                                  sel=sel, cnt=len(given))
    assert list(sel_out[:cnt_out]) == given
    j = np.arange(Lc)
    m = np.isin(j // block, given)[None, :]
    for h in range(G):
        ref = dense_reference(widen(q[h, Lc - 1:Lc]), widen(k), widen(v), m)
        assert np.max(np.abs(out[h] - ref[0])) <= 1e-12


def test_decode_swa_equals_window_row():
    Lc, G, W = 700, 2, 300
    d = inputs.small_prefill(Lc, G, 1, [oracle.SWA], seed=41)
    q, k, v = d["q"][0], d["k"][0, 0], d["v"][0, 0]
    C = np.zeros((Lc // 64, 16), dtype=np.float32)
    out, _, _, _ = oracle.decode_head(q[:, Lc - 1], k, v, C, inputs.lowfreq_projector(), oracle.SWA, W, 64, 4, 2)
    for h in range(G):
        ref = oracle.attention_rows(q[h, Lc - 1:Lc], np.array([Lc - 1]), k, v, oracle.SWA, W)
        assert np.array_equal(out[h], ref[0])


def test_decode_full_head_sees_whole_cache():
    Lc, G = 700, 2
    d = inputs.small_prefill(Lc, G, 1, [oracle.FULL], seed=43)
    q, k, v = d["q"][0], d["k"][0, 0], d["v"][0, 0]
    C = np.zeros((Lc // 64, 16), dtype=np.float32)
    out, _, _, _ = oracle.decode_head(q[:, Lc - 1], k, v, C, inputs.lowfreq_projector(), oracle.FULL, 10, 64, 4, 2)
    m = mask_matrix(Lc, oracle.FULL)[Lc - 1:Lc]
    for h in range(G):
        ref = dense_reference(widen(q[h, Lc - 1:Lc]), widen(k), widen(v), m)
        assert np.max(np.abs(out[h] - ref[0])) <= 1e-12


def _bf16_grid():
    """Every non-negative finite bf16 value (bit patterns 0x0000..0x7F7F) and
    2^128 standing for the next value up (infinity), as fp64."""
    bits = np.arange(0, 0x7F81, dtype=np.uint32) << 16
    vals = bits.view(np.float32).astype(np.float64)
    vals[-1] = 2.0 ** 128
    return vals


def brute_round_bf16(x, grid):
    """Nearest grid value by exact rational distance, ties to the even bit pattern."""
    from fractions import Fraction

    if np.isnan(x):
        return np.nan
    a = abs(x)
    j = int(np.searchsorted(grid, a, side="left"))
    if j == grid.size:  # beyond 2^128
        r = grid[-1]
    elif grid[j] == a:
        r = grid[j]
    else:
        lo, hi = grid[j - 1], grid[j]
        dl, dh = Fraction(a) - Fraction(lo), Fraction(hi) - Fraction(a)
        r = lo if dl < dh or (dl == dh and (j - 1) % 2 == 0) else hi
    r = np.inf if r == 2.0 ** 128 else r
    return -r if x < 0 else r


def test_round_bf16_matches_exact_nearest_even():
    grid = _bf16_grid()
    rng = np.random.default_rng(9)
    x = rng.standard_normal(3000) * np.exp2(rng.integers(-140, 130, 3000))
    # exact half-way points between neighbouring bf16 values, and just off them
    mids = (grid[1:-1:97] + grid[2::97]) / 2.0
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf), grid[:-1:211],
                        [0.0, -0.0, 2.0 ** -133, 3 * 2.0 ** -134, 2.0 ** -134, np.inf, -np.inf, np.nan,
                         (2.0 - 2.0 ** -8) * 2.0 ** 127, 3.4e38, 1e300]])
    # NaNs whose payload lies only in the low fraction bits (rounding the bits
    # alone would turn them into infinities)
    low_nan = np.array([0x7FF0000000000001, 0xFFF0000000000010, 0x7FF00000000FFFFF], dtype=np.uint64).view(np.float64)
    x = np.concatenate([x, low_nan])
    got = oracle.round_bf16(x)
    want = np.array([brute_round_bf16(v, grid) for v in x])
    assert np.array_equal(got, want, equal_nan=True)
    assert np.array_equal(np.signbit(got[x == 0]), np.signbit(x[x == 0]))


def test_round_bf16_rounds_once():
    # 1 + 2^-8 + 2^-30 lies above the half-way point between the bf16 values 1
    # and 1 + 2^-7; rounding to fp32 first would land exactly on that point and
    # then tie to 1.
    x = np.array([1 + 2.0 ** -8 + 2.0 ** -30, -(1 + 2.0 ** -8 + 2.0 ** -30), 1 + 2.0 ** -8])
    assert np.array_equal(oracle.round_bf16(x), [1 + 2.0 ** -7, -(1 + 2.0 ** -7), 1.0])


def test_selection_ties_at_the_cut_take_lower_indices():
    nb, topk, L = 40, 6, 2
    C = np.ones((nb, 16))
    qb = np.ones((nb, 16))
    C[30] = 2.0  # one clear winner, every other candidate ties
    sel, cnt, kth = oracle.select(qb, C, np.arange(nb), topk, L)
    t = 39
    assert list(sel[t, : cnt[t]]) == [0, 1, 2, 3, 4, 5, 30, 38, 39]
    assert kth[t] == 16.0


# ------------------------------------------------------------ KV-cache upkeep


def _cache_case(batch, H, cap, seed):
    d = inputs.small_prefill(cap, H, H, [oracle.SWA] * H, seed=seed)  # any bf16 keys/values of the right shape
    k = d["k"].expand(batch, -1, -1, -1).clone() if batch > 1 else d["k"]
    v = d["v"].expand(batch, -1, -1, -1).clone() if batch > 1 else d["v"]
    return k, v


@pytest.mark.parametrize("block", [64, 128])
def test_appending_one_row_at_a_time_builds_block_means(block):
    H, cap = 3, 5 * block + 17  # capacity not a multiple of the block
    kinds = [oracle.SPARSE, oracle.SWA, oracle.SPARSE]
    k_src, v_src = _cache_case(2, H, cap, seed=50 + block)
    k_src[1] = torch.roll(k_src[1], 7, dims=1)  # the two sequences differ
    p = inputs.random_projector(17)
    kc = np.zeros((2, H, cap, 128), dtype=np.uint16)
    vc = np.zeros((2, H, cap, 128), dtype=np.uint16)
    sentinel = -12345.0
    C = np.full((2, H, cap // block, 16), sentinel)
    kb, vb = oracle._bf16_bits(k_src), oracle._bf16_bits(v_src)
    for pos in range(cap):
        kc2, vc2, C2 = oracle.cache_append(kc, vc, C, kinds, pos, kb[:, :, pos], vb[:, :, pos], block, p)
        # only row pos changed in the caches
        changed = np.any(kc2 != kc, axis=-1) | np.any(vc2 != vc, axis=-1)
        assert not np.any(np.delete(changed, pos, axis=2))
        assert np.array_equal(kc2[:, :, pos], kb[:, :, pos]) and np.array_equal(vc2[:, :, pos], vb[:, :, pos])
        # a centroid changes only when its block completes, only for SPARSE heads
        diff = np.any(C2 != C, axis=-1)
        if (pos + 1) % block == 0:
            blk = (pos + 1) // block - 1
            expect = np.zeros_like(diff)
            expect[:, [0, 2], blk] = True
            assert np.array_equal(diff, expect)
        else:
            assert not diff.any()
        kc, vc, C = kc2, vc2, C2
    # after filling: complete blocks of SPARSE heads = numpy mean-then-project
    nbc = cap // block
    pn = p.double().numpy()
    for b in range(2):
        for h in range(H):
            if kinds[h] == oracle.SPARSE:
                ref = widen(k_src[b, h, : nbc * block]).reshape(nbc, block, 128).mean(axis=1) @ pn
                assert np.max(np.abs(C[b, h] - ref)) <= 1e-12
            else:
                assert np.all(C[b, h] == sentinel)
    # the bulk build agrees with the appended result, for every cache length
    for L in (0, block - 1, block, 3 * block + 5, cap):
        bulk = oracle.cache_centroids(k_src, L, kinds, block, p, C=np.full_like(C, sentinel))
        full = L // block
        assert np.array_equal(bulk[:, [0, 2], :full], C[:, [0, 2], :full])
        assert np.all(bulk[:, [0, 2], full:] == sentinel) and np.all(bulk[:, 1] == sentinel)


def test_cache_centroid_with_coordinate_projector_is_mean_of_coordinates():
    block, cap = 64, 256
    k_src, _ = _cache_case(1, 1, cap, seed=77)
    got = oracle.cache_centroids(k_src, cap, [oracle.SPARSE], block, inputs.lowfreq_projector())
    dims = list(range(56, 64)) + list(range(120, 128))
    ref = widen(k_src[0, 0])[:, dims].reshape(-1, block, 16).mean(axis=1)
    assert np.max(np.abs(got[0, 0] - ref)) <= 1e-15


# ------------------------------------------------------- dynamic selection


def pairwise_dynamic(qb, C, t, cap, n_local, mass, min_k, beta):
    """Dynamic selection without sorting: candidate j is kept iff the weight of
    the candidates ahead of it in (score desc, index asc) order is still below
    mass * Z; then the count is clamped by dropping/adding in that order."""
    s = C @ qb
    cands = list(range(1, t - n_local + 1))
    if not cands:
        return sorted(set([0] + list(range(max(0, t - n_local + 1), t + 1))))
    smax = max(s[j] for j in cands)
    w = {j: np.exp(beta * (s[j] - smax)) for j in cands}
    Z = sum(w.values())

    def ahead(i, j):
        return s[i] > s[j] or (s[i] == s[j] and i < j)

    rank = {j: sum(1 for i in cands if ahead(i, j)) for j in cands}
    kept = [j for j in cands if sum(w[i] for i in cands if ahead(i, j)) < mass * Z]
    n = len(kept)
    n = max(n, min(min_k, len(cands)))
    n = min(n, cap, len(cands))
    chosen = [j for j in cands if rank[j] < n]
    return sorted(set(chosen) | {0} | set(range(max(0, t - n_local + 1), t + 1)))


def _dyn_case(nb, seed):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(nb, 16)), rng.normal(size=(nb, 16))


@pytest.mark.parametrize("mass,beta,cap,min_k", [(0.5, 0.3, 40, 0), (0.9, 0.3, 40, 0), (0.9, 1.0, 8, 0),
                                                 (0.99, 0.05, 60, 3), (0.2, 2.0, 40, 5), (1.0, 0.3, 12, 0)])
def test_dynamic_selection_matches_pairwise_definition(mass, beta, cap, min_k):
    nb, n_local = 64, 2
    Q, C = _dyn_case(nb, 3)
    ts = np.arange(nb, dtype=np.int32)
    sel, cnt, lo, hi = oracle.select_dynamic(Q, C, ts, cap, n_local, mass, min_k, beta)
    for t in range(nb):
        ref = pairwise_dynamic(Q[t], C, t, cap, n_local, mass, min_k, beta)
        assert list(sel[t, :cnt[t]]) == ref, (t, list(sel[t, :cnt[t]]), ref)
        assert np.all(sel[t, cnt[t]:] == -1)


def test_dynamic_selection_with_equal_weights_takes_ceil_of_mass():
    """beta = 0: every candidate weighs the same, so n* = ceil(mass * m) and the
    set is the fixed top-n* of the scores."""
    nb, n_local = 48, 3
    Q, C = _dyn_case(nb, 5)
    for mass in (0.1, 0.25, 0.5, 0.77, 1.0):
        for t in (10, 30, 47):
            m = t - n_local
            n = int(np.ceil(mass * m - 1e-12))
            sel, cnt, _, _ = oracle.select_dynamic(Q[t:t + 1], C, [t], 1000, n_local, mass, 0, 0.0)
            fsel, fcnt, _ = oracle.select(Q[t:t + 1], C, [t], n, n_local)
            assert cnt[0] == 1 + n + n_local
            assert list(sel[0, :cnt[0]]) == list(fsel[0, :fcnt[0]])


def test_dynamic_selection_with_full_mass_equals_fixed_topk():
    nb, n_local, cap = 80, 4, 10
    Q, C = _dyn_case(nb, 8)
    ts = np.arange(nb, dtype=np.int32)
    sel, cnt, _, _ = oracle.select_dynamic(Q, C, ts, cap, n_local, 1.0, 0, 0.5)
    fsel, fcnt, _ = oracle.select(Q, C, ts, cap, n_local)
    for t in range(nb):
        if t - n_local > cap:  # more candidates than the cap: the fixed rule keeps exactly the cap
            assert list(sel[t, :cnt[t]]) == list(fsel[t, :fcnt[t]])


def test_dynamic_selection_stops_at_planted_mass():
    """Two dominant blocks hold almost all the mass: mass 0.9 keeps just them."""
    nb, n_local = 40, 2
    rng = np.random.default_rng(1)
    C = rng.normal(scale=0.01, size=(nb, 16))
    q = np.zeros(16)
    q[0] = 1.0
    C[7, 0] = C[23, 0] = 10.0
    sel, cnt, lo, hi = oracle.select_dynamic(q[None], C, [39], 16, n_local, 0.9, 0, 1.0)
    assert list(sel[0, :cnt[0]]) == [0, 7, 23, 38, 39]
    assert hi[0] >= 0.9 > lo[0]
    # min_k raises the count past the planted pair, cap lowers it
    sel, cnt, _, _ = oracle.select_dynamic(q[None], C, [39], 16, n_local, 0.9, 4, 1.0)
    assert cnt[0] == 1 + 4 + n_local
    sel, cnt, _, _ = oracle.select_dynamic(q[None], C, [39], 1, n_local, 0.9, 0, 1.0)
    assert list(sel[0, :cnt[0]]) == [0, 7, 38, 39]


# ------------------------------------------------------ k-means clustering


def _objective(X, mu, assign):
    return float(((X - mu[assign]) ** 2).sum())


def test_kmeans_recovers_planted_blobs_in_one_step():
    rng = np.random.default_rng(0)
    nc, per, r = 6, 40, 16
    centers = rng.normal(scale=20.0, size=(nc, r))
    X = np.concatenate([centers[c] + rng.normal(scale=0.1, size=(per, r)) for c in range(nc)])
    mu, assign = oracle.kmeans(X, nc, 1)  # the evenly spaced start puts one seed in each blob
    assert np.array_equal(assign, np.repeat(np.arange(nc), per))
    ref = X.reshape(nc, per, r).mean(axis=1)
    assert np.max(np.abs(mu - ref)) <= 1e-12


def test_kmeans_objective_never_increases_and_converges_to_nearest():
    rng = np.random.default_rng(1)
    X = rng.normal(size=(500, 16))
    prev = np.inf
    for it in range(1, 8):
        mu, assign = oracle.kmeans(X, 12, it)
        obj = _objective(X, mu, assign)
        assert obj <= prev + 1e-9
        prev = obj
    mu, assign = oracle.kmeans(X, 12, 200)
    mu2, assign2 = oracle.kmeans(X, 12, 201)
    assert np.array_equal(assign, assign2)  # converged
    d = ((X[:, None, :] - mu[None]) ** 2).sum(-1)
    assert np.array_equal(np.argmin(d, axis=1), assign)  # every point sits with its nearest centroid


def test_kmeans_degenerate_sizes():
    rng = np.random.default_rng(2)
    X = rng.normal(size=(9, 16))
    mu, assign = oracle.kmeans(X, 9, 3)  # one point per cluster
    assert np.array_equal(assign, np.arange(9)) and np.array_equal(mu, X)
    mu0, _ = oracle.kmeans(X, 3, 0)  # no iteration: the evenly spaced seeds
    assert np.array_equal(mu0, X[[1, 4, 7]])


def test_kmeans_ties_go_to_the_lower_index_and_an_empty_cluster_keeps_its_centroid():
    # Six points on a line (integers, so every distance is exact); the seeds
    # are rows 1, 3 and 5: the values 0, 4 and 4.  Clusters 1 and 2 start on
    # the same point, so every point nearer 4 ties between them and goes to
    # cluster 1, leaving cluster 2 empty; the point 2 ties between 0 and 4
    # and goes to cluster 0.
    X = np.zeros((6, 16))
    X[:, 0] = [2, 0, 8, 4, 3, 4]
    mu, assign = oracle.kmeans(X, 3, 1)
    assert assign.tolist() == [0, 0, 1, 1, 1, 1]
    assert mu[:, 0].tolist() == [1.0, 4.75, 4.0] and not mu[:, 1:].any()


def test_cluster_chunks_cover_members_once():
    rng = np.random.default_rng(3)
    assign = rng.integers(0, 5, size=700)
    assign[:300] = 2  # one cluster larger than two chunks
    members, offsets, chunks = oracle.cluster_chunks(assign, 128, 5)
    assert sorted(members.tolist()) == list(range(128, 828))
    seen = []
    for c, s0, n in chunks:
        assert 1 <= n <= 128 and offsets[c] <= s0 and s0 + n <= offsets[c + 1]
        block = members[s0:s0 + n]
        assert np.all(assign[block - 128] == c) and np.all(np.diff(block) > 0)
        seen.extend(block.tolist())
    assert sorted(seen) == list(range(128, 828))


def test_attention_over_key_list_matches_bruteforce_and_full_row():
    Lc, G = 700, 2
    d = inputs.small_prefill(Lc, G, 1, [oracle.FULL], seed=45)
    q, k, v = d["q"][0], d["k"][0, 0], d["v"][0, 0]
    rng = np.random.default_rng(4)
    keys = np.sort(rng.choice(Lc, size=150, replace=False))
    got = oracle.attention_keys(q[:, Lc - 1], k, v, keys)
    m = np.zeros((1, Lc), dtype=bool)
    m[0, keys] = True
    for h in range(G):
        ref = dense_reference(widen(q[h, Lc - 1:Lc]), widen(k), widen(v), m)
        assert np.max(np.abs(got[h] - ref[0])) <= 1e-12
    allk = oracle.attention_keys(q[:, Lc - 1], k, v, np.arange(Lc))
    for h in range(G):
        full = oracle.attention_rows(q[h, Lc - 1:Lc], np.array([Lc - 1]), k, v, oracle.FULL)
        assert np.max(np.abs(allk[h] - full[0])) <= 1e-12


def _python_scores(qb, C):
    """q . c_j as a plain fp64 sum in coordinate order, one chunk at a time."""
    out = []
    for row in C:
        acc = 0.0
        for a, b in zip(qb, row):
            acc += float(a) * float(b)
        out.append(acc)
    return out


@pytest.mark.parametrize("n,topk", [(50, 7), (50, 0), (12, 12), (12, 30), (1, 1), (300, 32)])
def test_topk_chunks_matches_full_sort(n, topk):
    """The clustered decode keeps the topk chunks by (score desc, chunk index
    asc), listed ascending: a full Python sort of exact ties and negative
    scores included."""
    rng = np.random.default_rng(n + topk)
    C = rng.standard_normal((n, 16))
    dup = rng.integers(0, n, size=n // 3)
    if dup.size:
        C[dup] = C[dup[0]]  # a crowd of exactly equal scores
    C[-1] = -C[0]
    qb = rng.standard_normal(16)
    s = _python_scores(qb, C)
    want = sorted(sorted(range(n), key=lambda j: (-s[j], j))[:topk])
    got = oracle.topk_chunks(qb, C, topk)
    assert got.tolist() == want


def test_topk_chunks_tie_order_is_by_index():
    C = np.ones((10, 16))
    C[6] = 2.0
    got = oracle.topk_chunks(np.ones(16), C, 4)
    assert got.tolist() == [0, 1, 2, 6]


@pytest.mark.parametrize("cache_len,clu_end,n_chosen", [(900, 700, 3), (900, 900, 3), (900, 700, 0),
                                                         (640, 640, 0), (1000, 128, 0)])
def test_decode_clustered_keys_is_sink_chunks_and_tail(cache_len, clu_end, n_chosen):
    """Brute force by a boolean mask over the cache: the sink block, every
    member of the chosen chunks and the unclustered tail [clu_end, cache_len),
    each key once."""
    block, nc = 128, 6
    rng = np.random.default_rng(cache_len + clu_end + n_chosen)
    n = clu_end - block
    assign = rng.integers(0, nc, size=max(n, 0))
    members, offsets, chunks = oracle.cluster_chunks(assign, block, nc, chunk=16)
    chosen = sorted(rng.choice(len(chunks), size=min(n_chosen, len(chunks)), replace=False).tolist()) \
        if len(chunks) else []
    mask = np.zeros(cache_len, dtype=bool)
    mask[:min(block, cache_len)] = True
    for x in chosen:
        _, s0, m = chunks[x]
        for key in members[s0:s0 + m]:
            assert block <= key < clu_end
            mask[key] = True
    mask[clu_end:cache_len] = True
    got = oracle.decode_clustered_keys(members, chunks, chosen, block, clu_end, cache_len)
    assert got.tolist() == np.nonzero(mask)[0].tolist()
    assert len(set(got.tolist())) == got.size
