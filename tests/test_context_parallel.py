"""Host logic of context-parallel prefill on CPU: the row partition, which
earlier K/V rows each rank's queries can see, and the exchange of those rows
and of the centroids between gloo ranks (world sizes 2 and 3)."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cp():
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import context_parallel as mod

    return mod


@pytest.mark.parametrize("seq,world", [(1024, 2), (1024, 3), (1000, 3), (128 * 7, 7), (1 << 20, 8)])
def test_ranges_cover_the_sequence_in_whole_tiles(cp, seq, world):
    r = cp.cp_ranges(seq, world)
    assert r[0][0] == 0 and r[-1][1] == seq and len(r) == world
    for (a, b), (c, d) in zip(r, r[1:]):
        assert b == c
    for a, b in r:
        assert a % 128 == 0 and (b % 128 == 0 or b == seq) and b > a
    sizes = [(b - a + 127) // 128 for a, b in r]
    assert max(sizes) - min(sizes) <= 1


def test_too_many_ranks_is_an_error(cp):
    with pytest.raises(ValueError):
        cp.cp_ranges(256, 3)


def random_selection(nb, kmax, n_local, rng):
    sel = np.full((nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros(nb, dtype=np.int32)
    for t in range(nb):
        pool = list(range(1, max(1, t - n_local + 1)))
        rng.shuffle(pool)
        chosen = sorted(set([0] + pool[: kmax - 1 - n_local] + list(range(max(0, t - n_local + 1), t + 1))))
        sel[t, :len(chosen)] = chosen
        cnt[t] = len(chosen)
    return sel, cnt


def visible_earlier_rows(kind, i_lo, i_hi, window, block, sel, cnt):
    """Rows j < i_lo visible to some query i in [i_lo, i_hi), straight from the rules."""
    rows = set()
    for i in range(i_lo, i_hi):
        for j in range(0, i_lo):
            if kind == 0:
                ok = i - window < j <= i
            elif kind == 1:
                ok = j <= i
            else:
                t = i // block
                ok = j <= i and (j // block) in set(sel[t, :cnt[t]].tolist())
            if ok:
                rows.add(j)
    return rows


@pytest.mark.parametrize("world", [2, 3])
def test_needs_are_exactly_the_visible_earlier_rows(cp, world):
    seq, block, window, n_local, kmax = 768, 64, 150, 2, 7
    kinds = [0, 1, 2]
    rng = np.random.default_rng(world)
    sel1, cnt1 = random_selection(seq // block, kmax, n_local, rng)
    sel = torch.from_numpy(sel1)[None, None]
    cnt = torch.from_numpy(cnt1)[None, None]
    for qb, qe in cp.cp_ranges(seq, world):
        needs = cp.kv_needs(kinds, window, block, (qb, qe), 1, sel, cnt, {2: 0})
        for h, kind in enumerate(kinds):
            want = visible_earlier_rows(kind, qb, qe, window, block, sel1, cnt1)
            got = set()
            for lo, hi in needs.get((0, h), []):
                assert lo < hi <= qb
                got |= set(range(lo, hi))
            assert got == want, (qb, h)


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _worker_exchange(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    from swa_hybrid_attention_b200 import context_parallel as cp

    _init(rank, world, port)
    try:
        B, H, seq, block = 2, 3, 1000, 64
        g = torch.Generator().manual_seed(11)
        K = torch.randn(B, H, seq, 128, generator=g).to(torch.bfloat16)
        V = torch.randn(B, H, seq, 128, generator=g).to(torch.bfloat16)
        ranges = cp.cp_ranges(seq, world)
        qb, qe = ranges[rank]
        # arbitrary needs: a few random intervals below qb per (b, h), per rank
        rng = np.random.default_rng(100 + rank)
        needs = {}
        for b in range(B):
            for h in range(H):
                if qb == 0 or rng.random() < 0.2:
                    continue
                iv = []
                for _ in range(3):
                    lo = int(rng.integers(0, qb))
                    iv.append((lo, int(min(qb, lo + rng.integers(1, 200)))))
                needs[(b, h)] = cp._merge(iv)
        sentinel = torch.tensor(-3.5, dtype=torch.bfloat16)
        kf = torch.full((B, H, qe, 128), float(sentinel))
        kf = kf.to(torch.bfloat16)
        vf = kf.clone()
        nbytes = cp.exchange_kv(K[:, :, qb:qe].contiguous(), V[:, :, qb:qe].contiguous(), needs, ranges, rank, kf, vf)
        ok = True
        want_rows = 0
        for b in range(B):
            for h in range(H):
                have = set(range(qb, qe))
                for lo, hi in needs.get((b, h), []):
                    have |= set(range(lo, hi))
                    want_rows += hi - lo
                for j in range(qe):
                    if j in have:
                        ok &= bool(torch.equal(kf[b, h, j], K[b, h, j]) and torch.equal(vf[b, h, j], V[b, h, j]))
                    else:
                        ok &= bool((kf[b, h, j] == sentinel).all() and (vf[b, h, j] == sentinel).all())
        ok &= nbytes == want_rows * 2 * 128 * 2
        # centroids: each rank writes its own blocks, then all hold every block
        C = torch.full((B, 2, seq // block, 16), -1.0)
        for blk in range(qb // block, qe // block):
            C[:, :, blk] = blk + 0.25
        cp.gather_centroids(C, ranges, rank, block)
        ok &= bool(torch.equal(C[0, 0, :, 0], torch.arange(seq // block, dtype=torch.float32) + 0.25))
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_delivers_exactly_the_requested_rows(cp, world):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_exchange, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    assert all(res[r] for r in range(world)), res


def test_overlapped_launch_is_the_shortest_prefix_covering_the_exchange(cp):
    """overlap_head_items picks how many of a rank's first local items the
    capped launch runs while the K/V exchange is in flight: the shortest
    prefix whose planned KV tiles reach 1.25 x the exchange time at the
    per-tile rate on the given number of CTAs (all local items if none
    does).  Item costs are the planner's tile counts: t + 1 for a full head,
    the window's tiles for a streaming head, min(t + 1, 1 + k + L) for a
    sparse head (the selected block count)."""
    from swa_hybrid_attention_b200 import rtp

    cfg = rtp.AttnConfig(1, 1 << 20, 32, 4, 8192, 128, 128, 8)
    rng = np.random.default_rng(3)
    kinds = rng.integers(0, 3, 400)
    ts = rng.integers(0, 8192, 400)
    items = np.stack([kinds, np.zeros(400), np.zeros(400), ts], axis=1).astype(np.int64)
    cost = []
    for kind, t in zip(kinds, ts):
        if kind == 1:
            cost.append(t + 1)
        elif kind == 0:
            lo = max(0, (128 * t - cfg.window + 1)) // 128
            cost.append(t - lo + 1)
        else:
            sel = t + 1 if t - cfg.n_local <= cfg.topk else 1 + cfg.topk + cfg.n_local
            cost.append(sel)
    tile_s, ctas = 2.4e-6, 132
    for exchange_s in (0.0, 1e-5, 3e-4, 5.7e-4, 1e-3, 1.0):
        n_local = 300
        n = cp.overlap_head_items(items, n_local, cfg, exchange_s, ctas, tile_s)
        budget = 1.25 * exchange_s / tile_s * ctas
        prefix = np.concatenate([[0], np.cumsum(cost[:n_local])])
        assert 0 <= n <= n_local
        if n < n_local:
            assert prefix[n] >= budget and (n == 0 or prefix[n - 1] < budget), (exchange_s, n)
        else:
            assert prefix[n_local - 1] < budget
    assert cp.overlap_head_items(items, 300, cfg, 0.0, ctas, tile_s) == 0
    assert cp.overlap_head_items(items, 300, cfg, 1.0, ctas, tile_s) == 300
