"""GPU k-means of the projected cached keys (rtp_cache_cluster) and decode
over clustered retrieval heads (rtp_sparse_decode_clustered), against the
CPU oracle (C ABI).

k-means assignments are decided by floating point and are not unique under
rounding, so the GPU clustering is checked for validity (each centroid is
the mean of its keys, members grouped stably, sorted K/V equal the cache
rows, bit-reproducible), for agreement with the oracle's Lloyd run on the
same keys (assignments and objective), and for exact recovery of planted
blobs.  The clustered decode is checked on a clustering computed by the
oracle and handed to the kernel, so no expected value comes from the GPU.
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import IDX_ABS, IDX_REL, O_MAX_ABS, O_MEAN_ABS, TIE_REL, cpu
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def rand_cache(B, H, cap, seed, device):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, H, cap, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, cap, 128, generator=g).to(torch.bfloat16)
    return k.to(device), v.to(device)


def objective(X, mu, assign):
    return float(((X - mu[assign]) ** 2).sum())


def check_clustering(rtp, cl, k, v, proj, kinds, block, nc, iters, min_agree=0.99):
    """Validity of the GPU clustering and agreement with the oracle's k-means."""
    B, H = k.shape[0], k.shape[1]
    n = cl.n
    for b in range(B):
        for h in range(H):
            if kinds[h] != 2:
                continue
            mem = cpu(cl.members[b, h]).numpy().astype(np.int64)
            off = cpu(cl.offsets[b, h]).numpy().astype(np.int64)
            assert sorted(mem.tolist()) == list(range(block, block + n))
            assert off[0] == 0 and off[-1] == n and np.all(np.diff(off) >= 0)
            assign = np.empty(n, dtype=np.int64)
            for c in range(nc):
                seg = mem[off[c]:off[c + 1]]
                assert np.all(np.diff(seg) > 0)  # stable: positions ascending inside a cluster
                assign[seg - block] = c
            # each non-empty centroid is the mean of its keys' projections
            X = oracle.project_rows(cpu(k[b, h, block:block + n]), cpu(proj))
            mu = cpu(cl.centroids[b, h]).double().numpy()
            for c in range(nc):
                if off[c + 1] > off[c]:
                    ref = X[mem[off[c]:off[c + 1]] - block].mean(axis=0)
                    assert np.all(np.abs(mu[c] - ref) <= IDX_ABS + IDX_REL * np.abs(ref)), c
            # the chunk table cuts each cluster's members into pieces of <= 128
            _, _, chunks = oracle.cluster_chunks(assign, block, nc)
            assert int(cl.n_chunks[b, h]) == len(chunks)
            cs = cpu(cl.chunk_start[b, h]).numpy()
            ln = cpu(cl.chunk_len[b, h]).numpy()
            cc = cpu(cl.chunk_centroids[b, h])
            for i, (c, s0, m) in enumerate(chunks):
                assert cs[i] == s0 and ln[i] == m
                assert torch.equal(cc[i], cpu(cl.centroids[b, h, c]))
            # K/V rows in cluster order
            idx = torch.from_numpy(mem).to(k.device)
            assert torch.equal(cl.k_sorted[b, h], k[b, h].index_select(0, idx))
            assert torch.equal(cl.v_sorted[b, h], v[b, h].index_select(0, idx))
            # agreement with the oracle's Lloyd run on the same keys
            mu_o, assign_o = oracle.kmeans(X, nc, iters)
            agree = float(np.mean(assign_o == assign))
            assert agree >= min_agree, agree
            og, oo = objective(X, mu, assign), objective(X, mu_o, assign_o)
            assert abs(og - oo) <= 1e-3 * oo, (og, oo)


@pytest.mark.parametrize("block,nc,iters", [(128, 24, 5), (64, 100, 3), (128, 1, 2), (64, 2048, 2)])
def test_kmeans_valid_and_agrees_with_oracle(rtp, cuda_device, block, nc, iters):
    kinds = [2, 0, 2]
    cap, clu_end = 4096, (3000 // block) * block
    if nc == 2048:
        cap, clu_end = 4352, 4288  # more keys than clusters
    k, v = rand_cache(2, 3, cap, 10 + nc, cuda_device)
    proj = inputs.random_projector(4, cuda_device)
    cl = rtp.cluster_cache(k, v, proj, kinds, clu_end=clu_end, n_clusters=nc, iters=iters, block=block)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    check_clustering(rtp, cl, k, v, proj, kinds, block, nc, iters, min_agree=0.97 if nc == 2048 else 0.99)
    # bit-reproducible
    cl2 = rtp.cluster_cache(k, v, proj, kinds, clu_end=clu_end, n_clusters=nc, iters=iters, block=block)
    torch.cuda.synchronize()
    for name in ("centroids", "members", "offsets", "chunk_start", "chunk_len", "n_chunks", "chunk_centroids"):
        assert torch.equal(getattr(cl, name), getattr(cl2, name)), name


def _against_exact_path(rtp, here, tmp_path, extra):
    import os
    import subprocess
    import sys

    import kmeans_cases

    out = tmp_path / "exact.pt"
    env = dict(os.environ, RTP_KMEANS_EXACT_ASSIGN="1")
    r = subprocess.run([sys.executable, kmeans_cases.__file__, str(out)] + extra, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    exact = torch.load(out)
    for name, fields in here.items():
        assert fields["status"] == rtp.RTP_OK and exact[name]["status"] == rtp.RTP_OK, name
        for f, t in fields.items():
            if f != "status":
                assert torch.equal(t, exact[name][f]), (name, f)


def test_tensor_core_assignment_equals_exact_path(rtp, cuda_device, tmp_path):
    """The assignment pass on tensor cores (fp16 distances, keys it cannot
    decide within its error bound re-scored in fp32) gives, key for key, the
    exact fp32 path's nearest centroid: whole clusterings are bit-identical to
    a run with RTP_KMEANS_EXACT_ASSIGN=1 (every key by the fp32 path), also
    with exact ties (duplicated keys) and values beyond fp16's range."""
    import kmeans_cases

    _against_exact_path(rtp, kmeans_cases.run_all(rtp, cuda_device), tmp_path, [])


@pytest.mark.slow
def test_tensor_core_assignment_equals_exact_path_full_size(rtp, cuda_device, tmp_path):
    """The same at the decode workload's full size: 8 x 262,144-row cache, 3
    clustered heads, 2048 clusters, 8 rounds (6.28M keys a round)."""
    import kmeans_cases

    _against_exact_path(rtp, kmeans_cases.run_full(rtp, cuda_device), tmp_path, ["--full"])


def test_kmeans_recovers_planted_blobs_exactly(rtp, cuda_device):
    block, nc, per = 128, 16, 96
    n = nc * per
    cap = block + n
    g = torch.Generator().manual_seed(3)
    k = torch.randn(1, 1, cap, 128, generator=g)
    dims = list(range(56, 64)) + list(range(120, 128))  # what the low-frequency projector keeps
    centers = torch.randn(nc, 16, generator=g) * 8.0
    for c in range(nc):
        rows = slice(block + c * per, block + (c + 1) * per)
        k[0, 0, rows][:, dims] = centers[c] + 0.05 * torch.randn(per, 16, generator=g)
    k = k.to(torch.bfloat16).to(cuda_device)
    v = torch.randn(1, 1, cap, 128, generator=g).to(torch.bfloat16).to(cuda_device)
    proj = inputs.lowfreq_projector(cuda_device)
    cl = rtp.cluster_cache(k, v, proj, [2], clu_end=cap, n_clusters=nc, iters=3, block=block)
    torch.cuda.synchronize()
    off = cpu(cl.offsets[0, 0]).numpy()
    assert np.array_equal(off, np.arange(nc + 1) * per)
    assert np.array_equal(cpu(cl.members[0, 0]).numpy(), np.arange(block, cap))
    X = oracle.project_rows(cpu(k[0, 0, block:]), cpu(proj))
    mu_o, assign_o = oracle.kmeans(X, nc, 3)
    assert np.array_equal(assign_o, np.repeat(np.arange(nc), per))
    mu = cpu(cl.centroids[0, 0]).double().numpy()
    assert np.all(np.abs(mu - mu_o) <= IDX_ABS + IDX_REL * np.abs(mu_o))


def clusters_from_oracle(rtp, k, v, proj, kinds, clu_end, nc, iters, block, in_place=False):
    """The oracle's clustering, laid out in the rtp_clusters arrays (in_place:
    without the cluster-ordered K/V copy)."""
    B, H = k.shape[0], k.shape[1]
    cl = rtp.Clusters(B, H, clu_end, nc, block, k.device, in_place=in_place)
    per_head = {}
    for b in range(B):
        for h in range(H):
            if kinds[h] != 2:
                continue
            X = oracle.project_rows(cpu(k[b, h, block:clu_end]), cpu(proj))
            mu, assign = oracle.kmeans(X, nc, iters)
            members, offsets, chunks = oracle.cluster_chunks(assign, block, nc)
            mu32 = torch.from_numpy(mu.astype(np.float32))
            cl.centroids[b, h] = mu32.to(k.device)
            cl.members[b, h] = torch.from_numpy(members.astype(np.int32)).to(k.device)
            cl.offsets[b, h] = torch.from_numpy(offsets.astype(np.int32)).to(k.device)
            if not in_place:
                idx = torch.from_numpy(members).to(k.device)
                cl.k_sorted[b, h] = k[b, h].index_select(0, idx)
                cl.v_sorted[b, h] = v[b, h].index_select(0, idx)
            cc = np.zeros((cl.max_chunks, 16), dtype=np.float32)
            for i, (c, s0, m) in enumerate(chunks):
                cl.chunk_start[b, h, i] = s0
                cl.chunk_len[b, h, i] = m
                cc[i] = mu[c]
            cl.chunk_centroids[b, h] = torch.from_numpy(cc).to(k.device)
            cl.n_chunks[b, h] = len(chunks)
            per_head[(b, h)] = (members, chunks, cc[:len(chunks)])
    return cl, per_head


DECODE_CASES = [
    # batch, hq, hkv, kinds, cap, cache_len, clu_end, nc, topk, window, block
    (2, 16, 2, [2, 0], 4096, 3000, 2560, 24, 6, 1000, 128),
    (1, 8, 2, [2, 2], 4096, 2560, 2560, 30, 40, 500, 128),     # no tail; top-k above 32 (radix path)
    (2, 8, 1, [2], 2048, 2047, 1280, 6, 64, 300, 64),          # top-k above the chunk count: every chunk
    (1, 32, 2, [2, 0], 4096, 4000, 3840, 40, 8, 2000, 128),    # group of 16
    (1, 8, 2, [2, 1], 3000, 2900, 2048, 16, 0, 100, 128),      # top-k 0: sink and tail only; a full head
]


@pytest.mark.parametrize("case", DECODE_CASES)
def test_clustered_decode_matches_oracle(rtp, cuda_device, case):
    B, Hq, Hkv, kinds, cap, Lc, clu_end, nc, topk, window, block = case
    G = Hq // Hkv
    k, v = rand_cache(B, Hkv, cap, Lc + nc, cuda_device)
    g = torch.Generator().manual_seed(7)
    q = torch.randn(B, Hq, 1, 128, generator=g).to(torch.bfloat16).to(cuda_device)
    proj = inputs.random_projector(9, cuda_device)
    cl, per_head = clusters_from_oracle(rtp, k, v, proj, kinds, clu_end, nc, 3, block)
    o, sel, cnt = rtp.sparse_decode_clustered_step(q, k, v, proj, kinds, cl, window=window, block=block, topk=topk,
                                                   cache_len=Lc, return_selection=True)
    # the same clustering without the K/V copy: member rows gathered in place
    cl_in, _ = clusters_from_oracle(rtp, k, v, proj, kinds, clu_end, nc, 3, block, in_place=True)
    o_in, sel_in, cnt_in = rtp.sparse_decode_clustered_step(q, k, v, proj, kinds, cl_in, window=window, block=block,
                                                            topk=topk, cache_len=Lc, return_selection=True)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    assert torch.equal(o_in, o) and torch.equal(sel_in, sel) and torch.equal(cnt_in, cnt)
    sel, cnt, o = cpu(sel).numpy(), cpu(cnt).numpy(), cpu(o)
    n_tail = (Lc - clu_end + 127) // 128
    errs = []
    for b in range(B):
        for h in range(Hkv):
            qg = cpu(q[b, h * G:(h + 1) * G, 0])
            kh, vh = cpu(k[b, h]), cpu(v[b, h])
            if kinds[h] == 2:
                members, chunks, cc = per_head[(b, h)]
                m = min(topk, len(chunks))
                assert cnt[b, h] == 1 + n_tail + m and sel[b, h, 0] == 0
                chosen = sel[b, h, 1:1 + m]
                assert sorted(set(chosen.tolist())) == sorted(chosen.tolist())
                qb = oracle.project_rows(qg, cpu(proj)).sum(axis=0)
                ref_sel = oracle.topk_chunks(qb, cc, m)
                if set(chosen.tolist()) != set(ref_sel.tolist()):
                    s = oracle.scores(qb, cc)
                    kth = np.sort(s)[::-1][m - 1]
                    for x in set(chosen.tolist()) ^ set(ref_sel.tolist()):
                        assert abs(s[x] - kth) <= TIE_REL * abs(kth), (b, h, x)
                keys = oracle.decode_clustered_keys(members, chunks, chosen, block, clu_end, Lc)
                ref = oracle.attention_keys(qg, kh[:Lc], vh[:Lc], keys)
            else:
                ref, _, _, _ = oracle.decode_head(qg, kh[:Lc], vh[:Lc], np.zeros((Lc // block, 16)), cpu(proj),
                                                  kinds[h], window, block, topk, 1)
            got = o[b, h * G:(h + 1) * G, 0].double().numpy()
            errs.append(np.abs(got - oracle.round_bf16(ref)))
    e = np.stack(errs)
    assert e.max() <= O_MAX_ABS and e.mean() <= O_MEAN_ABS, (e.max(), e.mean())


def test_gpu_clustering_then_decode_runs_clean(rtp, cuda_device):
    """The library's own clustering feeds its clustered decode: every selected
    chunk is valid and the output equals the oracle's attention over the keys
    that selection names."""
    B, Hq, Hkv, cap, Lc, clu_end, nc, topk, block = 2, 8, 2, 4096, 3500, 3072, 32, 8, 128
    kinds = [2, 0]
    k, v = rand_cache(B, Hkv, cap, 77, cuda_device)
    q = torch.randn(B, Hq, 1, 128, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).to(cuda_device)
    proj = inputs.random_projector(2, cuda_device)
    cl = rtp.cluster_cache(k, v, proj, kinds, clu_end=clu_end, n_clusters=nc, iters=4, block=block)
    o, sel, cnt = rtp.sparse_decode_clustered_step(q, k, v, proj, kinds, cl, window=800, block=block, topk=topk,
                                                   cache_len=Lc, return_selection=True)
    # in place: the same clustering (no K/V copy written) and the same step
    cl_in = rtp.cluster_cache(k, v, proj, kinds, clu_end=clu_end, n_clusters=nc, iters=4, block=block, in_place=True)
    o_in, sel_in, _ = rtp.sparse_decode_clustered_step(q, k, v, proj, kinds, cl_in, window=800, block=block,
                                                       topk=topk, cache_len=Lc, return_selection=True)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    for name in ("centroids", "members", "offsets", "chunk_start", "chunk_len", "n_chunks", "chunk_centroids"):
        assert torch.equal(getattr(cl, name), getattr(cl_in, name)), name
    assert torch.equal(o_in, o) and torch.equal(sel_in, sel)
    G = Hq // Hkv
    for b in range(B):
        n_ch = int(cl.n_chunks[b, 0])
        chosen = cpu(sel[b, 0, 1:1 + topk]).numpy()
        assert np.all((chosen >= 0) & (chosen < n_ch))
        mem = cpu(cl.members[b, 0]).numpy()
        starts, lens = cpu(cl.chunk_start[b, 0]).numpy(), cpu(cl.chunk_len[b, 0]).numpy()
        keys = list(range(block)) + list(range(clu_end, Lc))
        for x in chosen:
            keys += mem[starts[x]:starts[x] + lens[x]].tolist()
        # the keys the GPU names are checked against the oracle's attention over them
        ref = oracle.attention_keys(cpu(q[b, :G, 0]), cpu(k[b, 0, :Lc]), cpu(v[b, 0, :Lc]), np.sort(keys))
        got = cpu(o[b, :G, 0]).double().numpy()
        assert np.max(np.abs(got - oracle.round_bf16(ref))) <= O_MAX_ABS


@pytest.mark.slow
def test_clustered_decode_full_size_cache(rtp, cuda_device):
    """Two sequences of the 256K-token decode workload, clustered by the
    oracle (256 clusters, 2 rounds) and decoded with the clustered kernels."""
    w = inputs.workload(4)
    d = inputs.decode_step(w, cuda_device, batch=2)
    kinds, Lc, B = d["kinds"], d["cache_len"], w.block
    clu_end = (Lc // B - w.n_local) * B
    q, k, v, proj = d["q"], d["kcache"], d["vcache"], d["proj"]
    cl, per_head = clusters_from_oracle(rtp, k, v, proj, kinds, clu_end, 256, 2, B)
    o, sel, cnt = rtp.sparse_decode_clustered_step(q, k, v, proj, kinds, cl, window=w.window, block=B, topk=w.topk,
                                                   return_selection=True)
    cl.k_sorted = cl.v_sorted = None  # the same clustering, read in place
    o_in = rtp.sparse_decode_clustered_step(q, k, v, proj, kinds, cl, window=w.window, block=B, topk=w.topk)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    assert torch.equal(o_in, o)
    sel, cnt, o = cpu(sel).numpy(), cpu(cnt).numpy(), cpu(o)
    G = w.group
    n_tail = (Lc - clu_end + 127) // 128
    errs = []
    for b in range(2):
        for h, kind in enumerate(kinds):
            qg = cpu(q[b, h * G:(h + 1) * G, 0])
            kh, vh = cpu(k[b, h]), cpu(v[b, h])
            if kind == 2:
                members, chunks, cc = per_head[(b, h)]
                m = min(w.topk, len(chunks))
                assert cnt[b, h] == 1 + n_tail + m
                chosen = sel[b, h, 1:1 + m]
                qb = oracle.project_rows(qg, cpu(proj)).sum(axis=0)
                ref_sel = oracle.topk_chunks(qb, cc, m)
                if set(chosen.tolist()) != set(ref_sel.tolist()):
                    s = oracle.scores(qb, cc)
                    kth = np.sort(s)[::-1][m - 1]
                    for x in set(chosen.tolist()) ^ set(ref_sel.tolist()):
                        assert abs(s[x] - kth) <= TIE_REL * abs(kth)
                keys = oracle.decode_clustered_keys(members, chunks, chosen, B, clu_end, Lc)
                ref = oracle.attention_keys(qg, kh, vh, keys)
            else:
                ref, _, _, _ = oracle.decode_head(qg, kh, vh, np.zeros((Lc // B, 16)), cpu(proj), kind, w.window, B,
                                                  w.topk, w.n_local)
            errs.append(np.abs(o[b, h * G:(h + 1) * G, 0].double().numpy() - oracle.round_bf16(ref)))
    e = np.stack(errs)
    assert e.max() <= O_MAX_ABS and e.mean() <= O_MEAN_ABS, (e.max(), e.mean())
