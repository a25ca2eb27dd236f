"""GPU parity of the KV-cache maintenance calls (rtp_cache_centroids,
rtp_cache_append) against the CPU oracle, decode over a cache of larger
capacity, and the prefill -> centroids -> append -> decode sequence of the
full-prefill / sparse-decode variant (C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from helpers import IDX_ABS, IDX_REL, O_MAX_ABS, O_MEAN_ABS, TIE_REL, cpu
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu

SENTINEL = -7.25


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def random_cache(batch, H, cap, seed, device):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(batch, H, cap, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(batch, H, cap, 128, generator=g).to(torch.bfloat16)
    return k.to(device), v.to(device)


def assert_centroids_close(got, ref):
    assert np.all(np.abs(got - ref) <= IDX_ABS + IDX_REL * np.abs(ref)), np.max(np.abs(got - ref))


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("cache_len", [1, 63, 640, 2500, 3000])
def test_cache_centroids_parity(rtp, cuda_device, block, cache_len):
    kinds = [2, 0, 2, 1]
    cap = 3000  # not a multiple of either block size
    k, _ = random_cache(2, 4, cap, 100 + block, cuda_device)
    proj = inputs.random_projector(3, cuda_device)
    C = torch.full((2, 4, cap // block, 16), SENTINEL, dtype=torch.float32, device=cuda_device)
    cfg = rtp.AttnConfig(2, cap, 8, 4, 512, block, 8, 2)
    rtp.rtp_cache_centroids(cfg, kinds, cache_len, k, proj, C)
    torch.cuda.synchronize()
    got = cpu(C).double().numpy()
    ref = oracle.cache_centroids(cpu(k), cache_len, kinds, block, cpu(proj), C=np.full(got.shape, SENTINEL))
    written = ~(ref == SENTINEL)
    assert np.array_equal(got[~written], ref[~written])  # untouched entries, bit for bit
    assert_centroids_close(got[written], ref[written])
    assert written.sum() == 2 * 2 * (cache_len // block) * 16


def test_cache_centroids_equal_indexer_centroids(rtp, cuda_device):
    """Both paths sum in the same fixed order: identical fp32 centroids."""
    N, block = 4096, 128
    d = inputs.small_prefill(N, 8, 2, [2, 2], seed=21, device=cuda_device)
    proj = inputs.random_projector(8, cuda_device)
    cfg = rtp.AttnConfig(1, N, 8, 2, 1024, block, 8, 2)
    plan = rtp.Plan(cfg, [2, 2])
    bufs = plan.buffers(cuda_device)
    rtp.rtp_indexer_project(plan.handle, d["q"], d["k"], proj, bufs["centroids"], bufs["qbar"])
    C = torch.zeros(1, 2, N // block, 16, dtype=torch.float32, device=cuda_device)
    rtp.rtp_cache_centroids(cfg, [2, 2], N, d["k"], proj, C)
    torch.cuda.synchronize()
    plan.close()
    assert torch.equal(C, bufs["centroids"])


@pytest.mark.parametrize("block", [64, 128])
def test_cache_append_parity(rtp, cuda_device, block):
    kinds = [2, 0, 2]
    B, H = 2, 3
    cap = 5 * block + 17
    k, v = random_cache(B, H, cap, 7 + block, cuda_device)
    proj = inputs.random_projector(11, cuda_device)
    C = torch.full((B, H, cap // block, 16), SENTINEL, dtype=torch.float32, device=cuda_device)
    cfg = rtp.AttnConfig(B, cap, 2 * H, H, 256, block, 4, 2)
    g = torch.Generator().manual_seed(99)
    for pos in (0, 5, block - 2, block - 1, 3 * block - 1, 5 * block - 1, cap - 1):
        kn = torch.randn(B, H, 128, generator=g).to(torch.bfloat16).to(cuda_device)
        vn = torch.randn(B, H, 128, generator=g).to(torch.bfloat16).to(cuda_device)
        k0, v0, C0 = cpu(k).clone(), cpu(v).clone(), cpu(C).double().numpy()
        rtp.rtp_cache_append(cfg, kinds, pos, kn, vn, k, v, proj, C)
        torch.cuda.synchronize()
        rk, rv, rC = oracle.cache_append(k0, v0, C0, kinds, pos, cpu(kn), cpu(vn), block, cpu(proj))
        assert np.array_equal(oracle._bf16_bits(k), rk) and np.array_equal(oracle._bf16_bits(v), rv)
        got = cpu(C).double().numpy()
        changed = np.any(rC != C0, axis=-1)
        assert np.array_equal(got[~changed], C0[~changed])  # nothing else written
        if (pos + 1) % block == 0:
            assert changed.sum() == B * 2
            assert_centroids_close(got[changed], rC[changed])
        else:
            assert not changed.any()


def test_append_then_decode_matches_oracle_and_tight_cache(rtp, cuda_device):
    """Full-attention prefill of the retrieval head, K-cache centroids, then
    decode steps that append one token each and cross a block boundary."""
    block, window, topk, n_local = 64, 300, 4, 2
    N0, steps, cap = 1024, 66, 1536
    B, Hq, Hkv = 2, 16, 2
    prefill_kinds, decode_kinds = [1, 0], [2, 0]
    G = Hq // Hkv
    seqs = [inputs.small_prefill(N0 + steps, Hq, Hkv, prefill_kinds, seed=60 + b) for b in range(B)]
    q = torch.cat([s["q"] for s in seqs]).to(cuda_device)
    k = torch.cat([s["k"] for s in seqs]).to(cuda_device)
    v = torch.cat([s["v"] for s in seqs]).to(cuda_device)
    proj = inputs.lowfreq_projector(cuda_device)
    # prefill of the first N0 tokens with a dense retrieval head (no centroids needed)
    o_pre, _ = rtp.hybrid_prefill_layer(q[:, :, :N0].contiguous(), k[:, :, :N0].contiguous(),
                                        v[:, :, :N0].contiguous(), prefill_kinds, proj, window=window, block=block)
    assert torch.isfinite(o_pre.float()).all()
    cache = rtp.DecodeCache(B, Hkv, cap, decode_kinds, proj, block=block, device=cuda_device)
    cache.load(k[:, :, :N0], v[:, :, :N0])
    errs = []
    for s in range(steps):
        p = N0 + s
        cache.append(k[:, :, p], v[:, :, p])
        qs = q[:, :, p:p + 1].contiguous()
        o, sel, cnt = cache.decode(qs, window=window, topk=topk, n_local=n_local, return_selection=True)
        torch.cuda.synchronize()
        assert rtp.rtp_last_device_status() == rtp.RTP_OK
        Lc = p + 1
        if s in (0, 1, steps - 2, steps - 1) or (Lc % block) in (0, 1):
            # the same step over a tight copy of the cache: same kernels, same bits
            o_t, sel_t, cnt_t = rtp.sparse_decode_step(qs, cache.k[:, :, :Lc].contiguous(),
                                                       cache.v[:, :, :Lc].contiguous(),
                                                       cache.centroids[:, :, :Lc // block].contiguous(), proj,
                                                       decode_kinds, window=window, block=block, topk=topk,
                                                       n_local=n_local, return_selection=True)
            assert torch.equal(o, o_t) and torch.equal(sel, sel_t) and torch.equal(cnt, cnt_t)
        # the oracle, with its own centroids of the cached keys
        kc = cpu(cache.k[:, :, :Lc])
        vc = cpu(cache.v[:, :, :Lc])
        C_or = oracle.cache_centroids(kc, Lc, decode_kinds, block, cpu(proj))
        o_c, sel_c, cnt_c = cpu(o), cpu(sel).numpy(), cpu(cnt).numpy()
        for b in range(B):
            for h in range(Hkv):
                qg = cpu(qs[b, h * G:(h + 1) * G, 0])
                if decode_kinds[h] == 2:
                    Cf = C_or[b, h].astype(np.float32)
                    _, so, co, kth = oracle.decode_head(qg, kc[b, h], vc[b, h], Cf, cpu(proj), 2, window, block,
                                                        topk, n_local)
                    gsel = [int(x) for x in sel_c[b, h, :cnt_c[b, h]]]
                    assert cnt_c[b, h] == co and gsel == sorted(set(gsel))
                    if set(gsel) != set(so[:co].tolist()):
                        qb = oracle.project_rows(qg, cpu(proj)).sum(axis=0)
                        sc = oracle.scores(qb, C_or[b, h])
                        for blk in set(gsel) ^ set(so[:co].tolist()):
                            assert abs(sc[blk] - kth) <= TIE_REL * abs(kth)
                    ref, _, _, _ = oracle.decode_head(qg, kc[b, h], vc[b, h], Cf, cpu(proj), 2, window, block, topk,
                                                      n_local, sel=sel_c[b, h], cnt=cnt_c[b, h])
                else:
                    ref, _, _, _ = oracle.decode_head(qg, kc[b, h], vc[b, h], np.zeros((Lc // block, 16)),
                                                      cpu(proj), 0, window, block, topk, n_local)
                got = o_c[b, h * G:(h + 1) * G, 0].double().numpy()
                errs.append(np.abs(got - oracle.round_bf16(ref)))
    # the appended centroids equal a fresh build over the final cache, bit for bit
    C_fresh = torch.zeros_like(cache.centroids)
    rtp.rtp_cache_centroids(cache._cfg(), decode_kinds, cache.length, cache.k, proj, C_fresh)
    torch.cuda.synchronize()
    nfull = cache.length // block
    assert torch.equal(C_fresh[:, 0, :nfull], cache.centroids[:, 0, :nfull])
    e = np.stack(errs)
    assert e.max() <= O_MAX_ABS and e.mean() <= O_MEAN_ABS, (e.max(), e.mean())


def test_decode_noalloc_with_capacity(rtp, cuda_device):
    """The allocation-free entry point honours the capacity stride too."""
    block, window, topk, n_local = 128, 1000, 8, 2
    B, Hq, Hkv, Lc, cap = 2, 16, 2, 3000, 4096
    kinds = [2, 0]
    k, v = random_cache(B, Hkv, cap, 5, cuda_device)
    proj = inputs.random_projector(2, cuda_device)
    C = torch.zeros(B, Hkv, cap // block, 16, dtype=torch.float32, device=cuda_device)
    cfg = rtp.AttnConfig(B, cap, Hq, Hkv, window, block, topk, n_local)
    rtp.rtp_cache_centroids(cfg, kinds, Lc, k, proj, C)
    q = torch.randn(B, Hq, 1, 128, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16).to(cuda_device)
    o = torch.empty_like(q)
    sel = torch.full((B, Hkv, cfg.kmax), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=cuda_device)
    rtp.rtp_sparse_decode_noalloc(cfg, kinds, Lc, q, k, v, C, proj, o, sel, cnt)
    o_t, sel_t, cnt_t = rtp.sparse_decode_step(q, k[:, :, :Lc].contiguous(), v[:, :, :Lc].contiguous(),
                                               C[:, :, :Lc // block].contiguous(), proj, kinds, window=window,
                                               block=block, topk=topk, n_local=n_local, return_selection=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_t) and torch.equal(sel[:, 0], sel_t[:, 0]) and torch.equal(cnt[:, 0], cnt_t[:, 0])
