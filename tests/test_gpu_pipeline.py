"""Prefill from host memory through the chunked pipeline
(rtp_hybrid_prefill_host) equals the device-resident layer bit for bit."""

import pytest
import torch

from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


CASES = [
    # seq, hq, hkv, kinds, window, block, topk, n_local, chunks
    (2048, 8, 4, [2, 0, 1, 0], 300, 64, 4, 2, 3),
    (1984, 4, 2, [0, 2], 200, 64, 3, 2, 4),     # ragged last tile
    (4096, 16, 2, [2, 1], 700, 128, 6, 2, 1),   # one chunk
    (4096, 8, 2, [0, 0], 500, 128, 4, 2, 32),   # no retrieval head; one tile per chunk
]


@pytest.mark.parametrize("case", CASES)
def test_host_pipeline_equals_device_layer(rtp, cuda_device, case):
    seq, hq, hkv, kinds, window, block, topk, n_local, chunks = case
    d = inputs.small_prefill(seq, hq, hkv, kinds, seed=seq + chunks, device=cuda_device)
    q = torch.cat([d["q"], torch.roll(d["q"], 3, dims=2)]).contiguous()
    k = torch.cat([d["k"], torch.roll(d["k"], 5, dims=2)]).contiguous()
    v = torch.cat([d["v"], torch.roll(d["v"], 7, dims=2)]).contiguous()
    proj = inputs.random_projector(3, cuda_device)
    cfg = rtp.AttnConfig(2, seq, hq, hkv, window, block, topk, n_local)
    plan = rtp.Plan(cfg, kinds)
    bufs = plan.buffers(cuda_device)
    o_ref = torch.empty_like(q)
    plan.run(q, k, v, proj, o_ref, bufs)
    torch.cuda.synchronize()
    plan.close()
    hq_, hk_, hv_ = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.full(q.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    pl = rtp.HostPipeline(cfg, kinds, chunks, device=cuda_device)
    pl.run(hq_, hk_, hv_, proj, ho)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    assert torch.equal(ho, o_ref.cpu())
    if 2 in kinds:
        assert torch.equal(pl.bufs["sel"], bufs["sel"]) and torch.equal(pl.bufs["sel_cnt"], bufs["sel_cnt"])
    pl.close()


@pytest.mark.slow
def test_host_pipeline_full_size_1m_layer(rtp, cuda_device):
    """The 1M-token layer from pinned host memory in 16 chunks equals the device-resident layer."""
    w = inputs.workload(3)
    d = inputs.prefill_layer(w, 0, cuda_device)
    cfg = rtp.AttnConfig(1, w.seq, w.n_q_heads, w.n_kv_heads, w.window, w.block, w.topk, w.n_local)
    plan = rtp.Plan(cfg, d["kinds"])
    bufs = plan.buffers(cuda_device)
    o_ref = torch.empty_like(d["q"])
    plan.run(d["q"], d["k"], d["v"], d["proj"], o_ref, bufs)
    torch.cuda.synchronize()
    plan.close()
    hq_, hk_, hv_ = (x.cpu().pin_memory() for x in (d["q"], d["k"], d["v"]))
    ho = torch.empty(d["q"].shape, dtype=torch.bfloat16).pin_memory()
    pl = rtp.HostPipeline(cfg, d["kinds"], 16, device=cuda_device)
    pl.run(hq_, hk_, hv_, d["proj"], ho)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    assert torch.equal(ho.to(cuda_device), o_ref)
    pl.close()
