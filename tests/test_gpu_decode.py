"""GPU parity of the sparse decode step against the CPU oracle (C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from helpers import O_MAX_ABS, O_MEAN_ABS, TIE_REL, cpu
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def oracle_centroids(kc, kinds, block, proj):
    """Cached centroids of every retrieval head, computed by the oracle."""
    B, H, Lc = kc.shape[0], kc.shape[1], kc.shape[2]
    n = Lc // block  # complete blocks (at least one row is allocated: the call wants a centroid array)
    C = torch.zeros(B, H, max(1, n), 16, dtype=torch.float32)
    for b in range(B):
        for h in range(H):
            if kinds[h] == 2 and n:
                C[b, h, :n] = torch.from_numpy(oracle.centroids(cpu(kc[b, h]), block, cpu(proj)).astype(np.float32))
    return C


def check_decode(rtp, d, kinds, window, block, topk, n_local, device):
    q, kc, vc = d["q"].to(device), d["kcache"].to(device), d["vcache"].to(device)
    proj = d["proj"].to(device)
    C = oracle_centroids(kc, kinds, block, proj)
    o, sel, cnt = rtp.sparse_decode_step(q, kc, vc, C.to(device), proj, kinds, window=window, block=block, topk=topk,
                                         n_local=n_local, return_selection=True)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    Bt, Hq, Hkv, Lc = q.shape[0], q.shape[1], kc.shape[1], kc.shape[2]
    G = Hq // Hkv
    sel, cnt, o = cpu(sel).numpy(), cpu(cnt).numpy(), cpu(o)
    errs = []
    for b in range(Bt):
        for h in range(Hkv):
            qg = cpu(q[b, h * G:(h + 1) * G, 0])
            kh, vh = cpu(kc[b, h]), cpu(vc[b, h])
            if kinds[h] == 2:
                # the GPU's selection against the oracle's own
                _, so, co, kth = oracle.decode_head(qg, kh, vh, C[b, h], cpu(proj), 2, window, block, topk, n_local)
                g = [int(x) for x in sel[b, h, :cnt[b, h]]]
                assert g == sorted(set(g)) and cnt[b, h] == co
                if set(g) != set(so[:co].tolist()):
                    qb = oracle.project_rows(qg, cpu(proj)).sum(axis=0)
                    s = oracle.scores(qb, C[b, h].double().numpy())
                    for blk in set(g) ^ set(so[:co].tolist()):
                        assert abs(s[blk] - kth) <= TIE_REL * abs(kth)
                ref, _, _, _ = oracle.decode_head(qg, kh, vh, C[b, h], cpu(proj), 2, window, block, topk, n_local,
                                                  sel=sel[b, h], cnt=cnt[b, h])
            else:
                ref, _, _, _ = oracle.decode_head(qg, kh, vh, C[b, h], cpu(proj), kinds[h], window, block, topk,
                                                  n_local)
            got = o[b, h * G:(h + 1) * G, 0].double().numpy()
            err = np.abs(got - oracle.round_bf16(ref))
            errs.append(err)
    e = np.stack(errs)
    assert e.max() <= O_MAX_ABS and e.mean() <= O_MEAN_ABS, (e.max(), e.mean())


DECODE_CASES = [
    # batch, hq, hkv, kinds, cache_len, window, block, topk, n_local
    (2, 16, 2, [2, 0], 4096, 1000, 128, 4, 2),
    (2, 8, 4, [2, 2, 0, 1], 3000, 512, 64, 6, 2),    # ragged last block, full head, block 64
    (1, 4, 1, [2], 640, 100, 128, 8, 1),            # fewer candidates than top-k
    (3, 32, 4, [2, 0, 2, 2], 8192, 2048, 128, 16, 4),
    # top-k 32 (bitonic path) with more candidates than one scoring round per CTA
    (1, 8, 2, [2, 0], 196608, 4096, 64, 32, 4),
    # top-k above 32 (radix path): one round, then several rounds per CTA
    (1, 8, 2, [2, 0], 8192, 1024, 128, 40, 2),
    (1, 4, 1, [2], 196608, 128, 64, 48, 2),
    # group of 16 query heads per KV head (two tiles of 8 heads in the attention MMAs)
    (2, 32, 2, [2, 0], 4096, 1000, 128, 4, 2),
]


@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_small(rtp, cuda_device, case):
    B, hq, hkv, kinds, Lc, window, block, topk, n_local = case
    w = inputs.Workload(4, "t", B, 1, hq, hkv, 1, window, block, topk, n_local, "lowfreq", 0, [kinds],
                        cache_len=Lc, decode=True)
    d = inputs.decode_step(w, "cpu")
    check_decode(rtp, d, kinds, window, block, topk, n_local, cuda_device)


SHORT_CACHE_CASES = [
    # batch, hq, hkv, kinds, cache_len, window, block, topk, n_local
    (1, 8, 2, [2, 0], 1, 100, 64, 4, 2),    # a single cached token
    (1, 8, 2, [2, 1], 63, 100, 64, 4, 2),   # no complete block yet; a full head
    (1, 8, 2, [2, 0], 64, 32, 64, 4, 2),    # exactly one block; window shorter than the cache
    (2, 8, 2, [2, 0], 65, 64, 64, 4, 1),    # the new token opens block 1
    (1, 4, 1, [2], 300, 64, 64, 1, 1),      # top-k 1
]


@pytest.mark.parametrize("case", SHORT_CACHE_CASES, ids=[f"len{c[4]}-k{c[7]}" for c in SHORT_CACHE_CASES])
def test_decode_short_caches(rtp, cuda_device, case):
    B, hq, hkv, kinds, Lc, window, block, topk, n_local = case
    w = inputs.Workload(4, "t", B, 1, hq, hkv, 1, window, block, topk, n_local, "lowfreq", 0, [kinds],
                        cache_len=Lc, decode=True)
    d = inputs.decode_step(w, "cpu")
    check_decode(rtp, d, kinds, window, block, topk, n_local, cuda_device)


@pytest.mark.slow
def test_decode_full_size(rtp, cuda_device):
    w = inputs.workload(4)
    d = inputs.decode_step(w, cuda_device)
    check_decode(rtp, d, w.kinds[0], w.window, w.block, w.topk, w.n_local, cuda_device)


def test_decode_workspace_reuse_and_arbitrary_contents(rtp, cuda_device):
    """The workspace holds only scratch of the step that uses it: one
    workspace, first filled with arbitrary bytes, then reused for steps on
    alternating inputs, gives every step exactly the output and selection of
    a call on a fresh workspace (nothing of the previous step is taken for
    this step's)."""
    kinds, B, hq, hkv, Lc, window, block, topk, n_local = [2, 0, 2, 2], 2, 16, 4, 8192, 1024, 128, 12, 3
    steps = []
    for seed in (7, 8):
        w = inputs.Workload(60 + seed, "t", B, 1, hq, hkv, 1, window, block, topk, n_local, "lowfreq", 0, [kinds],
                            cache_len=Lc, decode=True)
        d = inputs.decode_step(w, "cpu")
        d = {k: (v.to(cuda_device) if torch.is_tensor(v) else v) for k, v in d.items()}
        d["C"] = oracle_centroids(d["kcache"], kinds, block, d["proj"]).to(cuda_device)
        ref = rtp.sparse_decode_step(d["q"], d["kcache"], d["vcache"], d["C"], d["proj"], kinds, window=window,
                                     block=block, topk=topk, n_local=n_local, return_selection=True)
        steps.append((d, ref))
    cfg = rtp.AttnConfig(B, Lc, hq, hkv, window, block, topk, n_local)
    ws_bytes = rtp.rtp_decode_workspace_bytes(cfg, kinds, Lc)
    g = torch.Generator(device="cpu").manual_seed(3)
    for fill in ("random", "ones"):
        if fill == "random":
            ws = torch.randint(0, 256, (ws_bytes,), dtype=torch.uint8, generator=g).to(cuda_device)
        else:
            ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device=cuda_device)
        for i in (0, 1, 0, 1, 1, 0):
            d, (ro, rsel, rcnt) = steps[i]
            o = torch.empty_like(d["q"])
            sel = torch.full((B, hkv, cfg.kmax), -1, dtype=torch.int32, device=cuda_device)
            cnt = torch.zeros(B, hkv, dtype=torch.int32, device=cuda_device)
            rtp.rtp_sparse_decode(cfg, kinds, Lc, d["q"], d["kcache"], d["vcache"], d["C"], d["proj"], o, ws,
                                  ws_bytes, sel, cnt)
            torch.cuda.synchronize()
            assert torch.equal(o, ro), (fill, i)
            assert torch.equal(cnt, rcnt) and torch.equal(sel, rsel), (fill, i)
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
