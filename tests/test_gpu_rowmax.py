"""GPU parity of the row-max block selection (rtp_block_select_rowmax)
against the CPU oracle, and of the prefill on its selection (C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from helpers import TIE_REL, check_prefill_rows, cpu
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu

S, W, F = inputs.SPARSE, inputs.SWA, inputs.FULL


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def check_rowmax_rows(sel_gpu, cnt_gpu, q_group, proj, C, t_list, block, topk, n_local):
    """GPU rows against the oracle's row-max selection: equal sets, or every
    differing block is a near-tie of the k-th score (the GPU scores in fp32).
    Returns the number of near-tie rows."""
    sel_o, cnt_o, kth = oracle.select_rowmax(q_group, proj, C, t_list, block, topk, n_local)
    near = 0
    for r, t in enumerate(t_list):
        n = int(cnt_gpu[r])
        g = [int(x) for x in sel_gpu[r][:n]]
        assert g == sorted(set(g)), (t, g)
        assert n == int(cnt_o[r]), (t, n, int(cnt_o[r]))
        assert 0 in g and all(b in g for b in range(max(0, t - n_local + 1), t + 1)), (t, g)
        assert all(x == -1 for x in sel_gpu[r][n:])
        o = set(int(x) for x in sel_o[r][:n])
        if set(g) != o:
            s = oracle.rowmax_scores(q_group, proj, C, t, block)
            for b in set(g) ^ o:
                assert abs(s[b] - kth[r]) <= TIE_REL * abs(kth[r]), (t, b, s[b], kth[r])
            near += 1
    return near


CASES = [
    # seq, hq, hkv, kinds, window, block, topk, n_local
    (2048, 8, 2, [S, W], 512, 64, 6, 2),
    (4096, 16, 4, [S, W, S, F], 1024, 128, 5, 2),
    (3072, 8, 1, [S], 256, 64, 12, 1),
    (1536, 32, 4, [S, S, W, S], 300, 128, 3, 1),  # group of 8
    (640, 4, 1, [S], 128, 64, 16, 2),  # fewer candidates than top-k in every block
    (32768, 16, 2, [S, W], 1024, 128, 32, 4),  # 256 blocks: many candidates per query block
]


@pytest.mark.parametrize("case", CASES, ids=[f"n{c[0]}-h{c[1]}x{c[2]}-b{c[5]}-k{c[6]}" for c in CASES])
def test_rowmax_selection_and_prefill(rtp, cuda_device, case):
    n, hq, hkv, kinds, window, block, topk, n_local = case
    d = inputs.small_prefill(n, hq, hkv, kinds, seed=n + hq)
    q, k, v, proj = (d[x].to(cuda_device) for x in ("q", "k", "v", "proj"))
    cfg = rtp.AttnConfig(1, n, hq, hkv, window, block, topk, n_local)
    plan = rtp.Plan(cfg, kinds)
    bufs = plan.buffers(cuda_device)
    o = torch.full_like(q, float("nan"))
    plan.run(q, k, v, proj, o, bufs, score="rowmax")
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    G, nb = hq // hkv, n // block
    slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
    for kvh, s in slot_of.items():
        C = oracle.centroids(cpu(k[0, kvh]), block, cpu(proj))
        check_rowmax_rows(cpu(bufs["sel"][0, s]).numpy(), cpu(bufs["sel_cnt"][0, s]).numpy(),
                          cpu(q[0, kvh * G:(kvh + 1) * G]), cpu(proj), C, np.arange(nb), block, topk, n_local)
    rows = np.unique(np.concatenate([np.arange(0, n, 97), np.arange(n - 64, n)]))
    check_prefill_rows(o, q, k, v, kinds, G, window, block, bufs["sel"], bufs["sel_cnt"], slot_of,
                       lambda hq_: rows)
    plan.close()


def test_rowmax_on_query_ranges_equals_whole_sequence(rtp, cuda_device):
    """Plans over query ranges (context parallelism) write the same rows, bit
    for bit, as the whole-sequence plan."""
    n, hq, hkv, kinds, window, block, topk, n_local = 4096, 8, 2, [S, W], 1024, 128, 4, 2
    d = inputs.small_prefill(n, hq, hkv, kinds, seed=77)
    q, k, v, proj = (d[x].to(cuda_device) for x in ("q", "k", "v", "proj"))
    cfg = rtp.AttnConfig(1, n, hq, hkv, window, block, topk, n_local)
    whole = rtp.Plan(cfg, kinds)
    bufs = whole.buffers(cuda_device)
    rtp.rtp_indexer_project(whole.handle, q, k, proj, bufs["centroids"], bufs["qbar"])
    rtp.rtp_block_select_rowmax(whole.handle, q, proj, bufs["centroids"], bufs["sel"], bufs["sel_cnt"])
    sel2 = torch.full_like(bufs["sel"], -9)
    cnt2 = torch.full_like(bufs["sel_cnt"], -9)
    for qb, qe in ((0, 1024), (1024, 2560), (2560, 4096)):
        p = rtp.Plan(cfg, kinds, q_range=(qb, qe))
        rtp.rtp_block_select_rowmax(p.handle, q[:, :, qb:qe].contiguous(), proj, bufs["centroids"], sel2, cnt2)
        torch.cuda.synchronize()
        p.close()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    assert torch.equal(sel2, bufs["sel"]) and torch.equal(cnt2, bufs["sel_cnt"])
    whole.close()


def test_rowmax_finds_a_planted_needle_the_mean_misses(rtp, cuda_device):
    """One query row aligned with the keys of a distant block j, while every
    row of the query block leans a little towards another block m: the mean
    over the rows prefers m, the row maximum keeps j (top-k 1)."""
    n, hq, hkv, block, topk, n_local = 4096, 4, 1, 128, 1, 1
    d = inputs.small_prefill(n, hq, hkv, [S], seed=5)
    q, k, v, proj = d["q"].clone(), d["k"].clone(), d["v"], d["proj"]
    t, j, m, i = 30, 7, 12, 30 * 128 + 77  # query block, needle block, competitor block, query row
    d1 = torch.zeros(128)
    d1[120:124] = 1.0  # both directions inside the low-frequency coordinates the projector keeps
    d2 = torch.zeros(128)
    d2[124:128] = 1.0
    k[0, 0, j * block:(j + 1) * block] += (6.0 * d1).to(torch.bfloat16)
    k[0, 0, m * block:(m + 1) * block] += (6.0 * d2).to(torch.bfloat16)
    for h in range(hq):
        q[0, h, t * block:(t + 1) * block] += (1.0 * d2).to(torch.bfloat16)
        q[0, h, i] += (6.0 * d1).to(torch.bfloat16)
    q, k, v, proj = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), proj.to(cuda_device)
    cfg = rtp.AttnConfig(1, n, hq, hkv, 256, block, topk, n_local)
    plan = rtp.Plan(cfg, [S])
    bufs = plan.buffers(cuda_device)
    rtp.rtp_indexer_project(plan.handle, q, k, proj, bufs["centroids"], bufs["qbar"])
    rtp.rtp_block_select(plan.handle, bufs["qbar"], bufs["centroids"], bufs["sel"], bufs["sel_cnt"])
    mean_sel = set(bufs["sel"][0, 0, t, :int(bufs["sel_cnt"][0, 0, t])].tolist())
    rtp.rtp_block_select_rowmax(plan.handle, q, proj, bufs["centroids"], bufs["sel"], bufs["sel_cnt"])
    row_sel = set(bufs["sel"][0, 0, t, :int(bufs["sel_cnt"][0, 0, t])].tolist())
    torch.cuda.synchronize()
    plan.close()
    assert mean_sel == {0, m, t} and row_sel == {0, j, t}, (sorted(mean_sel), sorted(row_sel))


@pytest.mark.parametrize("tied", ["some", "all"])
def test_rowmax_exact_ties_take_the_lower_blocks(rtp, cuda_device, tied):
    """Blocks with identical keys have identical centroids and scores.  With
    a crowd of them at the cut (or every block identical, so that every
    candidate is re-scored exactly), the kept ones are the lowest-indexed, as
    in the oracle."""
    n, hq, hkv, block, topk, n_local = 8192, 8, 1, 128, 7, 2
    d = inputs.small_prefill(n, hq, hkv, [S], seed=9)
    k = d["k"].clone()
    nb = n // block
    src = k[0, 0, 3 * block:4 * block].clone()
    copies = range(1, nb) if tied == "all" else range(5, nb, 3)
    for b in copies:
        k[0, 0, b * block:(b + 1) * block] = src
    q, k, v, proj = (x.to(cuda_device) for x in (d["q"], k, d["v"], d["proj"]))
    cfg = rtp.AttnConfig(1, n, hq, hkv, 256, block, topk, n_local)
    plan = rtp.Plan(cfg, [S])
    bufs = plan.buffers(cuda_device)
    rtp.rtp_indexer_project(plan.handle, q, k, proj, bufs["centroids"], bufs["qbar"])
    rtp.rtp_block_select_rowmax(plan.handle, q, proj, bufs["centroids"], bufs["sel"], bufs["sel_cnt"])
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    C = oracle.centroids(cpu(k[0, 0]), block, cpu(proj))
    check_rowmax_rows(cpu(bufs["sel"][0, 0]).numpy(), cpu(bufs["sel_cnt"][0, 0]).numpy(), cpu(q[0]), cpu(proj), C,
                      np.arange(nb), block, topk, n_local)
    if tied == "all":
        # every candidate scores the same: blocks 1..topk are kept
        for t in range(topk + n_local + 1, nb):
            got = bufs["sel"][0, 0, t, :int(bufs["sel_cnt"][0, 0, t])].tolist()
            assert got == [0] + list(range(1, topk + 1)) + list(range(t - n_local + 1, t + 1)), (t, got)
    plan.close()


def test_rowmax_centroids_beyond_fp16_range(rtp, cuda_device):
    """Keys scaled so that centroid entries exceed fp16's range (2^15 and
    more): the tensor-core approximation is not used and every candidate is
    scored exactly; the selection still equals the oracle's."""
    n, hq, hkv, block, topk, n_local = 4096, 8, 1, 128, 5, 2
    d = inputs.small_prefill(n, hq, hkv, [S], seed=13)
    k = (d["k"].float() * 1.0e5).to(torch.bfloat16)
    q, k, proj = d["q"].to(cuda_device), k.to(cuda_device), d["proj"].to(cuda_device)
    cfg = rtp.AttnConfig(1, n, hq, hkv, 256, block, topk, n_local)
    plan = rtp.Plan(cfg, [S])
    bufs = plan.buffers(cuda_device)
    rtp.rtp_indexer_project(plan.handle, q, k, proj, bufs["centroids"], bufs["qbar"])
    assert float(bufs["centroids"].abs().max()) >= 32768.0
    rtp.rtp_block_select_rowmax(plan.handle, q, proj, bufs["centroids"], bufs["sel"], bufs["sel_cnt"])
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    C = oracle.centroids(cpu(k[0, 0]), block, cpu(proj))
    check_rowmax_rows(cpu(bufs["sel"][0, 0]).numpy(), cpu(bufs["sel_cnt"][0, 0]).numpy(), cpu(q[0]), cpu(proj), C,
                      np.arange(n // block), block, topk, n_local)
    plan.close()
