"""GPU parity of the per-head selection (rtp_indexer_project_heads,
rtp_block_select_heads, rtp_hybrid_prefill_heads) against the CPU oracle
(C ABI): every query head selects its own blocks."""

import numpy as np
import pytest
import torch

import oracle
from helpers import IDX_ABS, IDX_REL, O_MAX_ABS, O_MEAN_ABS, check_selection_rows, cpu
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu

S, W, F = inputs.SPARSE, inputs.SWA, inputs.FULL
MODE = {S: oracle.SPARSE, W: oracle.SWA, F: oracle.FULL}


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def run(rtp, d, window, topk, n_local, device):
    q, k, v, proj = (d[x].to(device) for x in ("q", "k", "v", "proj"))
    cfg = rtp.AttnConfig(1, q.shape[2], q.shape[1], k.shape[1], window, 128, topk, n_local)
    plan = rtp.Plan(cfg, d["kinds"])
    bufs = plan.buffers(device, per_head=True)
    o = torch.full_like(q, float("nan"))
    plan.run(q, k, v, proj, o, bufs, score="heads")
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    return q, k, v, proj, o, bufs, plan


CASES = [
    # seq, hq, hkv, kinds, window, topk, n_local
    (2048, 8, 2, [S, W], 512, 4, 2),
    (4096, 16, 2, [S, S], 1024, 6, 1),
    (3072, 8, 4, [S, W, F, S], 300, 3, 2),  # group of 2
    (1024, 8, 1, [S], 256, 16, 1),  # fewer candidates than top-k: every head keeps all blocks
]


@pytest.mark.parametrize("case", CASES, ids=[f"n{c[0]}-h{c[1]}x{c[2]}-k{c[5]}" for c in CASES])
def test_per_head_selection_and_prefill(rtp, cuda_device, case):
    n, hq, hkv, kinds, window, topk, n_local = case
    d = inputs.small_prefill(n, hq, hkv, kinds, seed=3 * n + hq)
    q, k, v, proj, o, bufs, plan = run(rtp, d, window, topk, n_local, cuda_device)
    G, nb = hq // hkv, n // 128
    slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
    rows = np.unique(np.concatenate([np.arange(0, n, 61), np.arange(n - 40, n)]))
    errs = []
    for hqi in range(hq):
        kvh, g = hqi // G, hqi % G
        kh, vh = cpu(k[0, kvh]), cpu(v[0, kvh])
        sel = cnt = None
        if kinds[kvh] == S:
            s = slot_of[kvh]
            C = oracle.centroids(kh, 128, cpu(proj))
            Qh = oracle.qbar(cpu(q[0, hqi:hqi + 1]), 128, cpu(proj))
            gq = cpu(bufs["qbar_heads"][0, s, g]).double().numpy()
            assert np.all(np.abs(gq - Qh) <= IDX_ABS + IDX_REL * np.abs(Qh)), np.max(np.abs(gq - Qh))
            sel = cpu(bufs["sel_heads"][0, s, g]).numpy()
            cnt = cpu(bufs["cnt_heads"][0, s, g]).numpy()
            check_selection_rows(sel, cnt, Qh, C, np.arange(nb), topk, n_local)
        ref = oracle.attention_rows(cpu(q[0, hqi][torch.from_numpy(rows).to(q.device)]), rows, kh, vh,
                                    MODE[kinds[kvh]], window, 128, sel, cnt)
        got = o[0, hqi, torch.from_numpy(rows).to(q.device)].double().cpu().numpy()
        errs.append(np.abs(got - oracle.round_bf16(ref)))
    e = np.stack(errs)
    assert e.max() <= O_MAX_ABS and e.mean() <= O_MEAN_ABS, (e.max(), e.mean())
    plan.close()


def test_equal_head_lists_reproduce_the_shared_selection_bitwise(rtp, cuda_device):
    """Per-head lists that all equal the shared one: the per-head prefill does
    exactly the shared prefill's work and writes the same bits."""
    n, hq, hkv, kinds, window, topk, n_local = 4096, 8, 2, [S, W], 1024, 5, 2
    d = inputs.small_prefill(n, hq, hkv, kinds, seed=11)
    q, k, v, proj = (d[x].to(cuda_device) for x in ("q", "k", "v", "proj"))
    cfg = rtp.AttnConfig(1, n, hq, hkv, window, 128, topk, n_local)
    plan = rtp.Plan(cfg, kinds)
    bufs = plan.buffers(cuda_device, per_head=True)
    o1 = torch.empty_like(q)
    plan.run(q, k, v, proj, o1, bufs)
    G = hq // hkv
    sel_h = bufs["sel"].unsqueeze(2).expand(-1, -1, G, -1, -1).contiguous()
    cnt_h = bufs["sel_cnt"].unsqueeze(2).expand(-1, -1, G, -1).contiguous()
    o2 = torch.empty_like(q)
    rtp.rtp_hybrid_prefill_heads(plan.handle, q, k, v, sel_h, cnt_h, o2)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    assert torch.equal(o1, o2)
    plan.close()


def test_per_head_selection_needs_whole_sequence_block_128(rtp, cuda_device):
    kinds = [S, W]
    cfg64 = rtp.AttnConfig(1, 1024, 8, 2, 256, 64, 4, 1)
    p64 = rtp.Plan(cfg64, kinds)
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_block_select_heads(p64.handle, 16, 16, 16, 16)
    assert e.value.status == rtp.RTP_ERR_UNSUPPORTED
    p64.close()
    cfg = rtp.AttnConfig(1, 1024, 8, 2, 256, 128, 4, 1)
    pr = rtp.Plan(cfg, kinds, q_range=(0, 512))
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_hybrid_prefill_heads(pr.handle, 16, 16, 16, 16, 16, 16)
    assert e.value.status == rtp.RTP_ERR_UNSUPPORTED
    pr.close()
