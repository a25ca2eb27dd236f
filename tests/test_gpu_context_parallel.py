"""Context-parallel prefill on one GPU (C ABI).

1. Emulated ranks in one process: each rank's ranged plan runs the indexer
   on its own rows, selection on its own query blocks and the prefill on K/V
   buffers that hold only its own rows and the earlier rows kv_needs lists
   (every other row is finite garbage).  Centroids, summaries, selections and
   outputs must equal the single-GPU layer bit for bit: a missing row would
   change the output, and the kernels compute each tile the same way.
2. Two real ranks (processes) on the same GPU running cp_prefill_layer over a
   gloo group with host staging: the whole driver, collectives included.
   No kernel waits on another rank; the ranks only meet in host collectives.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GARBAGE = 3.0


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


@pytest.fixture(scope="module")
def cp(rtp):
    from swa_hybrid_attention_b200 import context_parallel as mod

    return mod


def reference(rtp, q, k, v, proj, cfg, kinds, dynamic):
    plan = rtp.Plan(cfg, kinds)
    bufs = plan.buffers(q.device)
    o = torch.empty_like(q)
    plan.run(q, k, v, proj, o, bufs, dynamic=dynamic)
    torch.cuda.synchronize()
    plan.close()
    return o, bufs


def emulate(rtp, cp, q, k, v, proj, cfg, kinds, world, dynamic, split=False):
    """split: each rank's plan is split at its first row (rtp_route_heads_split)
    and run as the overlapped driver runs it: its local items (the first on a
    capped grid) while every row outside its own is still garbage, then the
    fetched rows arrive and the remaining items run."""
    ranges = cp.cp_ranges(cfg.seq, world)
    plans = [rtp.Plan(cfg, kinds, q_range=r, key_begin=r[0] if split else None) for r in ranges]
    bufs = plans[0].buffers(q.device)  # whole-sequence layout, shared: each rank writes only its own part
    for b in bufs.values():
        b.fill_(-9)
    slot_of = {h: s for s, h in enumerate(plans[0].slot_heads)}
    for p, (qb, qe) in zip(plans, ranges):
        if p.n_sparse:
            rtp.rtp_indexer_project(p.handle, q[:, :, qb:qe].contiguous(), k[:, :, qb:qe].contiguous(), proj,
                                    bufs["centroids"], bufs["qbar"])
    o = torch.full_like(q, float("nan"))
    fetched = []
    for p, (qb, qe) in zip(plans, ranges):
        sel = cnt = None
        if p.n_sparse:
            if dynamic is None:
                rtp.rtp_block_select(p.handle, bufs["qbar"], bufs["centroids"], bufs["sel"], bufs["sel_cnt"])
            else:
                rtp.rtp_block_select_dynamic(p.handle, bufs["qbar"], bufs["centroids"], dynamic["mass"], 0,
                                             dynamic["beta"], bufs["sel"], bufs["sel_cnt"])
            sel, cnt = bufs["sel"].cpu(), bufs["sel_cnt"].cpu()
        needs = cp.kv_needs(kinds, cfg.window, cfg.block, (qb, qe), cfg.batch, sel, cnt, slot_of)
        kf = torch.full((cfg.batch, cfg.n_kv_heads, qe, 128), GARBAGE, dtype=torch.bfloat16, device=q.device)
        vf = kf.clone()
        kf[:, :, qb:qe] = k[:, :, qb:qe]
        vf[:, :, qb:qe] = v[:, :, qb:qe]
        fetched.append(sum(hi - lo for iv in needs.values() for lo, hi in iv))
        o_loc = torch.empty_like(q[:, :, qb:qe])
        q_loc = q[:, :, qb:qe].contiguous()
        sel_d = bufs["sel"] if p.n_sparse else None
        cnt_d = bufs["sel_cnt"] if p.n_sparse else None
        if split:
            check_split(rtp, p, cfg, kinds, qb)
            head = p.n_local // 3
            rtp.rtp_hybrid_prefill_items(p.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc, 0, head, 5)
            rtp.rtp_hybrid_prefill_items(p.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc, head, p.n_local, 0)
        for (b, h), iv in needs.items():
            for lo, hi in iv:
                kf[b, h, lo:hi] = k[b, h, lo:hi]
                vf[b, h, lo:hi] = v[b, h, lo:hi]
        if split:
            rtp.rtp_hybrid_prefill_items(p.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc, p.n_local, p.n_items, 0)
        else:
            rtp.rtp_hybrid_prefill(p.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc)
        o[:, :, qb:qe] = o_loc
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    for p in plans:
        p.close()
    return o, bufs, fetched


def check_split(rtp, p, cfg, kinds, key_begin):
    """The split plan holds the ranged plan's items; the first n_local are
    exactly those whose earliest visible key is at or after key_begin."""
    items = rtp.rtp_plan_work_items(p.handle)
    ranged = rtp.Plan(cfg, kinds, q_range=p.q_range)
    ref = rtp.rtp_plan_work_items(ranged.handle)
    ranged.close()
    assert sorted(map(tuple, items.tolist())) == sorted(map(tuple, ref.tolist()))

    def local(it):
        kind, t = int(it[0]) & 0xFF, int(it[3])
        first = max(0, 128 * t - cfg.window + 1) if kind == 0 else 0
        return first >= key_begin

    flags = [local(it) for it in items]
    assert flags == [True] * p.n_local + [False] * (p.n_items - p.n_local)


CASES = [
    # seq, hq, hkv, kinds, window, block, topk, n_local, world, dynamic
    (2048, 8, 4, [2, 0, 1, 0], 300, 64, 4, 2, 2, None),
    (2048, 8, 4, [2, 0, 1, 0], 300, 64, 4, 2, 4, None),
    (1984, 4, 2, [0, 2], 200, 64, 3, 2, 3, None),         # ragged last tile on the last rank
    (4096, 16, 2, [2, 1], 700, 128, 6, 2, 4, None),       # group 8, block 128
    (4096, 8, 2, [2, 0], 1000, 128, 8, 2, 3, dict(mass=0.6, beta=20.0)),
    (1024, 4, 1, [1], 64, 128, 2, 1, 8, None),            # one tile per rank
]


@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
@pytest.mark.parametrize("case", CASES)
def test_emulated_ranks_equal_single_gpu_bit_for_bit(rtp, cp, cuda_device, case, split):
    seq, hq, hkv, kinds, window, block, topk, n_local, world, dynamic = case
    d = inputs.small_prefill(seq, hq, hkv, kinds, seed=seq + world, device=cuda_device)
    d["k"] = torch.cat([d["k"], torch.roll(d["k"], 5, dims=2)])  # two sequences
    d["v"] = torch.cat([d["v"], torch.roll(d["v"], 9, dims=2)])
    d["q"] = torch.cat([d["q"], torch.roll(d["q"], 3, dims=2)])
    q, k, v = d["q"].contiguous(), d["k"].contiguous(), d["v"].contiguous()
    proj = inputs.random_projector(7, cuda_device)
    cfg = rtp.AttnConfig(2, seq, hq, hkv, window, block, topk, n_local)
    o_ref, b_ref = reference(rtp, q, k, v, proj, cfg, kinds, dynamic)
    o, bufs, fetched = emulate(rtp, cp, q, k, v, proj, cfg, kinds, world, dynamic, split)
    if 2 in kinds:
        assert torch.equal(bufs["centroids"], b_ref["centroids"]) and torch.equal(bufs["qbar"], b_ref["qbar"])
        assert torch.equal(bufs["sel"], b_ref["sel"]) and torch.equal(bufs["sel_cnt"], b_ref["sel_cnt"])
    assert torch.equal(o, o_ref)
    assert fetched[0] == 0 and all(f > 0 for f in fetched[1:])


def _worker(rank, world, port, seq, q_out, overlap):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from swa_hybrid_attention_b200 import context_parallel as cp
        from swa_hybrid_attention_b200 import inputs as inp
        from swa_hybrid_attention_b200 import rtp

        d = inp.small_prefill(seq, 8, 4, [2, 0, 1, 0], seed=77, device="cuda")
        cfg = rtp.AttnConfig(1, seq, 8, 4, 300, 64, 4, 2)
        qb, qe = cp.cp_ranges(seq, world)[rank]
        o_loc, info = cp.cp_prefill_layer(d["q"][:, :, qb:qe].contiguous(), d["k"][:, :, qb:qe].contiguous(),
                                          d["v"][:, :, qb:qe].contiguous(), [2, 0, 1, 0],
                                          inp.random_projector(7, "cuda"), cfg, overlap=overlap)
        torch.cuda.synchronize()
        q_out.put((rank, o_loc.cpu().view(torch.int16).numpy(), info["bytes_received"],
                   rtp.rtp_last_device_status()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("overlap", [True, False], ids=["overlap", "serial"])
def test_two_processes_with_gloo_staging(rtp, cp, cuda_device, overlap):
    seq, world = 2048, 2
    d = inputs.small_prefill(seq, 8, 4, [2, 0, 1, 0], seed=77, device=cuda_device)
    cfg = rtp.AttnConfig(1, seq, 8, 4, 300, 64, 4, 2)
    o_ref, _ = reference(rtp, d["q"], d["k"], d["v"], inputs.random_projector(7, cuda_device), cfg, [2, 0, 1, 0],
                         None)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seq, q_out, overlap)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, o_bits, nbytes, status = q_out.get(timeout=300)
        res[r] = (o_bits, nbytes, status)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    ranges = cp.cp_ranges(seq, world)
    ref_bits = o_ref.cpu().view(torch.int16).numpy()
    for r, (qb, qe) in enumerate(ranges):
        o_bits, nbytes, status = res[r]
        assert status == rtp.RTP_OK
        assert np.array_equal(o_bits, ref_bits[:, :, qb:qe])
    assert res[0][1] == 0 and res[1][1] > 0
