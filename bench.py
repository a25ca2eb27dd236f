"""Benchmark of the headwise hybrid attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Primary workload: one 1M-token V2 prefill layer (32 q / 4 kv heads, kv0 a
block-sparse retrieval head with block 128, top-k 128 + sink + 8 local and
1024 planted needles, kv1-3 SWA window 8192).  A step is one pass of the
attention path over that layer: rtp_indexer_project + rtp_block_select +
rtp_hybrid_prefill (the routing plan is built once, before timing).  Inputs
(8.6 GB of Q) are far larger than L2, so no flush is needed between steps.

`value` is effective throughput in TFLOP/s: algorithmic attention FLOPs
(4 * 128 per visible (query, key) pair) of all ranks / step time (max over
ranks).  Each rank runs its own independent layer (weak scaling, no data-path
collective).  Secondary lines: the 48-layer 128K V2 prefill pass and the
8 x 256K decode step.  With --impl reference the CPU oracle is timed on a
bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from swa_hybrid_attention_b200 import inputs  # noqa: E402

METRIC = "headwise sparse prefill attention ms and TFLOP/s at 128K/1M; % BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TILE_FLOPS = 2 * 2 * 128 * 128 * 128  # QK^T + PV of one 128x128 tile for one head


# ---------------------------------------------------------------- accounting


def selected_count(t: int, topk: int, n_local: int) -> int:
    ncand = max(0, t - n_local)
    return 1 + topk + n_local if ncand > topk else t + 1


def algorithmic_pairs(kind: int, n: int, window: int, block: int, topk: int, n_local: int) -> int:
    """Visible (query, key) pairs of one query head."""
    if kind == inputs.FULL:
        return n * (n + 1) // 2
    if kind == inputs.SWA:
        w = min(window, n)
        return w * (w + 1) // 2 + (n - w) * w
    nb = n // block
    tot = 0
    for t in range(nb):
        c = selected_count(t, topk, n_local)
        tot += block * block * (c - 1) + block * (block + 1) // 2
    return tot


def layer_flops(w, kinds) -> tuple[float, float]:
    """(algorithmic, executed) attention FLOPs of one layer."""
    G = w.group
    algo = sum(algorithmic_pairs(k, w.seq, w.window, w.block, w.topk, w.n_local) for k in kinds) * G * 4 * 128
    nqt = (w.seq + 127) // 128
    tiles = 0
    for k in kinds:
        for t in range(nqt):
            if k == inputs.FULL:
                tiles += t + 1
            elif k == inputs.SWA:
                first = 128 * t - w.window + 1
                lo = 0 if first <= 0 else first // 128
                tiles += t - lo + 1
            elif w.block == 128:
                tiles += selected_count(t, w.topk, w.n_local)
            else:
                tiles += (selected_count(2 * t, w.topk, w.n_local) + selected_count(2 * t + 1, w.topk, w.n_local) + 1) // 2
    return float(algo), float(tiles * G * TILE_FLOPS)


def decode_work(w, kinds, Lc) -> tuple[int, int]:
    """(algorithmic bytes, FLOPs) of one decode step: per sequence, the K/V
    rows every head reads (kmax selected blocks of a retrieval head, the
    window of a streaming head), the retrieval heads' cached centroids, and
    q and o."""
    ns = sum(1 for k in kinds if k == inputs.SPARSE)
    nsw = len(kinds) - ns
    keys = ns * w.kmax * w.block + nsw * min(w.window, Lc)
    bytes_ = w.batch * (keys * 128 * 2 * 2 + ns * (Lc // w.block) * 16 * 4 + w.n_q_heads * 128 * 2 * 2)
    return bytes_, w.batch * keys * w.group * 4 * 128


def indexer_bytes(w, kinds) -> float:
    ns = sum(1 for k in kinds if k == inputs.SPARSE)
    nb = w.seq // w.block
    return float(ns * (w.seq * 128 * 2 * (1 + w.group) + 2 * nb * 16 * 4))


def prefill_traffic(w):
    """DRAM bytes per launch of the prefill kernel for the 1M-token layer, from
    the committed ncu summary (captured at 128K and scaled by length); None
    for any other length."""
    p = os.path.join(ROOT, "profiles", "hybrid_prefill_kernel.md")
    if w.seq != 1048576 or not os.path.exists(p):
        return None
    for line in open(p):
        if line.startswith("prefill_traffic_bytes_per_launch_1m:"):
            return float(line.split(":")[1])
    return None


def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# -------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples nvidia-smi clocks / throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", *sel], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ distributed


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _collective_device():
    import torch.distributed as dist

    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank value (the step time) over all ranks."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=_collective_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_units(n_units: int, rank: int, world: int) -> list:
    """Contiguous share of n_units independent units (layers, sequences) for a rank."""
    per, extra = divmod(n_units, world)
    start = rank * per + min(rank, extra)
    return list(range(start, start + per + (1 if rank < extra else 0)))


def rank_layer(rank: int) -> int:
    """Each rank times its own independent layer of the primary workload (weak scaling)."""
    return rank


# ---------------------------------------------------------------- our arm


def make_layer(rtp, w, layer, device):
    d = inputs.prefill_layer(w, layer, device)
    cfg = rtp.AttnConfig(w.batch, w.seq, w.n_q_heads, w.n_kv_heads, w.window, w.block, max(w.topk, 0),
                         max(w.n_local, 1))
    plan = rtp.Plan(cfg, d["kinds"])
    bufs = plan.buffers(device)
    return d, plan, bufs


def time_primary(rtp, w, layer, steps, warmup, device, world):
    d, plan, bufs = make_layer(rtp, w, layer, device)
    q, k, v, proj = d["q"], d["k"], d["v"], d["proj"]
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        plan.run(q, k, v, proj, o, bufs, stream)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status(stream) == rtp.RTP_OK
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    sampler = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(steps):
        e = ev[s]
        e[0].record(stream)
        if plan.n_sparse:
            rtp.rtp_indexer_project(plan.handle, q, k, proj, bufs["centroids"], bufs["qbar"], stream)
        e[1].record(stream)
        if plan.n_sparse:
            rtp.rtp_block_select(plan.handle, bufs["qbar"], bufs["centroids"], bufs["sel"], bufs["sel_cnt"], stream)
        e[2].record(stream)
        rtp.rtp_hybrid_prefill(plan.handle, q, k, v, bufs["sel"] if plan.n_sparse else None,
                               bufs["sel_cnt"] if plan.n_sparse else None, o, stream)
        e[3].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    status = rtp.rtp_last_device_status(stream)
    total_ms = start.elapsed_time(end)
    per = {"indexer": [], "select": [], "prefill": []}
    for e in ev:
        per["indexer"].append(e[0].elapsed_time(e[1]))
        per["select"].append(e[1].elapsed_time(e[2]))
        per["prefill"].append(e[2].elapsed_time(e[3]))
    launches = steps * (3 if plan.n_sparse else 1)
    res = dict(total_ms=total_ms, per=per, clocks=clocks, status=status, launches=launches,
               kinds=d["kinds"], q=q, k=k, v=v, proj=proj, o=o, plan=plan, bufs=bufs, needles=d["needles"])
    return res


def needle_recall(needles, slot_of, sel, cnt, block) -> float | None:
    """Fraction of planted needles whose key block is selected for the
    query block of their target query (a diagnostic, not a pinned value)."""
    if not needles:
        return None
    sel_c, cnt_c = sel.cpu(), cnt.cpu()
    hit = 0
    for kvh, _, tq, j in needles:
        t = tq // block
        row = sel_c[0, slot_of[kvh], t, :int(cnt_c[0, slot_of[kvh], t])]
        hit += int((row == j // block).any())
    return hit / len(needles)


def time_dynamic(rtp, w, res, device, points=((0.9, None), (0.99, None), (0.9, 100.0)), reps=2):
    """The layer of the main step with the dynamic (mass-threshold) selection
    in place of the fixed top-k (cap = the workload's top-k, default beta):
    selection and prefill times, blocks kept, and the executed FLOPs of the
    prefill on that selection."""
    plan, bufs = res["plan"], res["bufs"]
    if not plan.n_sparse:
        return None
    q, k, v, o = res["q"], res["k"], res["v"], res["o"]
    stream = torch.cuda.current_stream()
    beta0 = rtp.default_selection_beta(plan.cfg)
    slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
    B, G = w.block, w.group
    nb = w.seq // B
    out = {"cap": w.topk, "default_beta": beta0, "min_k": 0,
           "fixed_needle_recall": needle_recall(res["needles"], slot_of, bufs["sel"], bufs["sel_cnt"], B)}
    for mass, beta in points:
        beta = beta0 if beta is None else beta
        sel, cnt = torch.empty_like(bufs["sel"]), torch.empty_like(bufs["sel_cnt"])
        for _ in range(2):
            rtp.rtp_block_select_dynamic(plan.handle, bufs["qbar"], bufs["centroids"], mass, 0, beta, sel, cnt,
                                         stream)
            rtp.rtp_hybrid_prefill(plan.handle, q, k, v, sel, cnt, o, stream)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
        torch.cuda.synchronize()
        for e in ev:
            e[0].record(stream)
            rtp.rtp_block_select_dynamic(plan.handle, bufs["qbar"], bufs["centroids"], mass, 0, beta, sel, cnt,
                                         stream)
            e[1].record(stream)
            rtp.rtp_hybrid_prefill(plan.handle, q, k, v, sel, cnt, o, stream)
            e[2].record(stream)
        torch.cuda.synchronize()
        sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        pre_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
        c = cnt.cpu().long()  # [batch][n_sparse][nb]
        # executed tiles of the sparse heads: one 128-key tile per selected block (block 128)
        sparse_pairs = float(((c - 1) * B * B + B * (B + 1) // 2).sum()) * G
        other_pairs = sum(algorithmic_pairs(kd, w.seq, w.window, B, w.topk, w.n_local)
                          for kd in res["kinds"] if kd != inputs.SPARSE) * G
        flops = (sparse_pairs + other_pairs) * 4 * 128
        out[f"mass_{mass}_beta_{beta:.4g}"] = {
            "select_ms": sel_ms, "prefill_ms": pre_ms,
            "mean_blocks_per_query_block": float(c.float().mean()),
            "fixed_blocks_per_query_block": float(np.mean([selected_count(t, w.topk, w.n_local) for t in range(nb)])),
            "algorithmic_tflops": flops / (pre_ms * 1e-3) / 1e12,
            "needle_recall": needle_recall(res["needles"], slot_of, sel, cnt, B)}
    # the fixed top-k on row-max scores (largest low-rank logit over a query
    # block's rows instead of the block mean); same budget, so the prefill
    # time only moves with the tiles' masks
    sel, cnt = torch.empty_like(bufs["sel"]), torch.empty_like(bufs["sel_cnt"])
    for _ in range(2):
        rtp.rtp_block_select_rowmax(plan.handle, q, res["proj"], bufs["centroids"], sel, cnt, stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    torch.cuda.synchronize()
    for e in ev:
        e[0].record(stream)
        rtp.rtp_block_select_rowmax(plan.handle, q, res["proj"], bufs["centroids"], sel, cnt, stream)
        e[1].record(stream)
        rtp.rtp_hybrid_prefill(plan.handle, q, k, v, sel, cnt, o, stream)
        e[2].record(stream)
    torch.cuda.synchronize()
    out["rowmax_scores"] = {
        "select_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
        "prefill_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
        "needle_recall": needle_recall(res["needles"], slot_of, sel, cnt, B)}
    # one selection per query head (same top-k per head); the pair of heads
    # in a CTA streams the union of its two lists
    if B == 128 and G % 2 == 0:
        qh = torch.empty(w.batch, plan.n_sparse, G, nb, 16, dtype=torch.float32, device=device)
        sh = torch.empty(w.batch, plan.n_sparse, G, nb, plan.cfg.kmax, dtype=torch.int32, device=device)
        ch = torch.empty(w.batch, plan.n_sparse, G, nb, dtype=torch.int32, device=device)
        for _ in range(2):
            rtp.rtp_indexer_project_heads(plan.handle, q, res["proj"], qh, stream)
            rtp.rtp_block_select_heads(plan.handle, qh, bufs["centroids"], sh, ch, stream)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
        torch.cuda.synchronize()
        for e in ev:
            e[0].record(stream)
            rtp.rtp_indexer_project_heads(plan.handle, q, res["proj"], qh, stream)
            rtp.rtp_block_select_heads(plan.handle, qh, bufs["centroids"], sh, ch, stream)
            e[1].record(stream)
            rtp.rtp_hybrid_prefill_heads(plan.handle, q, k, v, sh, ch, o, stream)
            e[2].record(stream)
        torch.cuda.synchronize()
        hit = 0
        sh_c, ch_c = sh.cpu(), ch.cpu()
        for kvh, hq_, tq, j in res["needles"]:
            t = tq // B
            row = sh_c[0, slot_of[kvh], hq_ % G, t, :int(ch_c[0, slot_of[kvh], hq_ % G, t])]
            hit += int((row == j // B).any())
        out["per_head"] = {
            "select_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
            "prefill_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
            "needle_recall": hit / len(res["needles"]) if res["needles"] else None}
        del qh, sh, ch
    return out


def time_selection_variants(rtp, w, device, reps=2):
    """The selection variants alone on the layer (profiling entry): the
    indexer, then `reps` times each of the row-max selection, the per-head
    summaries + selection, the fixed top-k selection and the dynamic
    (mass 0.9, default beta, cap = top-k) selection; mean ms per call."""
    d, plan, _ = make_layer(rtp, w, 0, device)
    bufs = plan.buffers(device, per_head=True)
    q, proj = d["q"], d["proj"]
    stream = torch.cuda.current_stream()
    beta = rtp.default_selection_beta(plan.cfg)
    rtp.rtp_indexer_project(plan.handle, q, d["k"], proj, bufs["centroids"], bufs["qbar"], stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]
    for e in ev:
        e[0].record(stream)
        rtp.rtp_block_select_rowmax(plan.handle, q, proj, bufs["centroids"], bufs["sel"], bufs["sel_cnt"], stream)
        e[1].record(stream)
        rtp.rtp_indexer_project_heads(plan.handle, q, proj, bufs["qbar_heads"], stream)
        rtp.rtp_block_select_heads(plan.handle, bufs["qbar_heads"], bufs["centroids"], bufs["sel_heads"],
                                   bufs["cnt_heads"], stream)
        e[2].record(stream)
        rtp.rtp_block_select(plan.handle, bufs["qbar"], bufs["centroids"], bufs["sel"], bufs["sel_cnt"], stream)
        e[3].record(stream)
        rtp.rtp_block_select_dynamic(plan.handle, bufs["qbar"], bufs["centroids"], 0.9, 0, beta, bufs["sel"],
                                     bufs["sel_cnt"], stream)
        e[4].record(stream)
    torch.cuda.synchronize()
    out = {"workload": w.name, "rowmax_select_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
           "per_head_summaries_and_select_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
           "fixed_select_ms": statistics.mean(e[2].elapsed_time(e[3]) for e in ev),
           "dynamic_select_ms": statistics.mean(e[3].elapsed_time(e[4]) for e in ev),
           "status": rtp.status_str(rtp.rtp_last_device_status(stream))}
    plan.close()
    return out


def time_cp_projection(rtp, w, res, device, world=8, link_gbs=770.0, reserve_sms=16):
    """Context-parallel prefill of the main layer split over `world` ranks,
    projected from one GPU.  Each rank's work is timed here on its own rows
    (its K/V buffer holds every row it may read), as one ranged launch and as
    the overlapped driver runs it (context_parallel.cp_prefill_layer): a head
    of the split plan's local tiles on reserve_sms fewer CTAs, sized to the
    exchange, then every other tile in one launch.  The K/V bytes a rank
    would receive are counted from its heads' row needs and selection;
    transfer time = bytes / the measured peer-copy bandwidth.  With overlap a
    rank takes head + rest + the part of the transfer the head does not
    hide.  Not a multi-GPU measurement."""
    from swa_hybrid_attention_b200 import context_parallel as cp

    plan, bufs = res["plan"], res["bufs"]
    q, k, v = res["q"], res["k"], res["v"]
    cfg = plan.cfg
    stream = torch.cuda.current_stream()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
    sel = bufs["sel"].cpu() if plan.n_sparse else None
    cnt = bufs["sel_cnt"].cpu() if plan.n_sparse else None
    sel_d = bufs["sel"] if plan.n_sparse else None
    cnt_d = bufs["sel_cnt"] if plan.n_sparse else None
    # every rank's inputs first, then all ranks' launches back to back, twice
    # (the second pass is timed), so that each launch runs at the clocks of a
    # long busy stretch like the single-GPU layer rather than as a short burst
    setup = []
    for qb, qe in cp.cp_ranges(cfg.seq, world):
        pr = rtp.Plan(cfg, res["kinds"], q_range=(qb, qe), key_begin=qb)
        needs = cp.kv_needs(res["kinds"], cfg.window, cfg.block, (qb, qe), cfg.batch, sel, cnt, slot_of)
        kv_bytes = sum(hi - lo for iv in needs.values() for lo, hi in iv) * 2 * 128 * 2
        transfer_s = kv_bytes / (link_gbs * 1e9)
        head = cp.overlap_head_items(rtp.rtp_plan_work_items(pr.handle), pr.n_local, cfg, transfer_s,
                                     sms - reserve_sms) if qb > 0 else 0
        # the rank's own Q rows and the K/V rows before its end (a rank's buffer)
        tensors = (q[:, :, qb:qe].contiguous(), k[:, :, :qe].contiguous(), v[:, :, :qe].contiguous())
        setup.append((pr, qb, qe, kv_bytes, head, tensors, torch.empty_like(tensors[0])))
    ranks = []
    for pass_ in range(2):
        evs = []
        for pr, qb, qe, kv_bytes, head, (q_loc, k_loc, v_loc), o_loc in setup:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(stream)
            rtp.rtp_hybrid_prefill(pr.handle, q_loc, k_loc, v_loc, sel_d, cnt_d, o_loc, stream)
            e[1].record(stream)
            rtp.rtp_hybrid_prefill_items(pr.handle, q_loc, k_loc, v_loc, sel_d, cnt_d, o_loc, 0, head,
                                         sms - reserve_sms, stream)
            e[2].record(stream)
            rtp.rtp_hybrid_prefill_items(pr.handle, q_loc, k_loc, v_loc, sel_d, cnt_d, o_loc, head, pr.n_items, 0,
                                         stream)
            e[3].record(stream)
            evs.append(e)
        torch.cuda.synchronize()
        if pass_ == 1:
            for (pr, qb, qe, kv_bytes, head, _, _), e in zip(setup, evs):
                transfer = kv_bytes / (link_gbs * 1e9) * 1e3
                head_ms, rest_ms = e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])
                exposed = max(0.0, transfer - head_ms)
                ranks.append({"q_rows": qe - qb, "prefill_ms": e[0].elapsed_time(e[1]), "kv_bytes_in": kv_bytes,
                              "transfer_ms": transfer, "items": pr.n_items, "local_items": pr.n_local,
                              "head_items": head, "head_ms": head_ms, "rest_ms": rest_ms,
                              "exposed_transfer_ms": exposed, "overlapped_ms": head_ms + exposed + rest_ms})
    for pr, *_ in setup:
        pr.close()
    del setup
    torch.cuda.empty_cache()
    return {"world": world, "ranks": ranks, "compute_ms_max": max(r["prefill_ms"] for r in ranks),
            "kv_bytes_in_max": max(r["kv_bytes_in"] for r in ranks), "link_gbs": link_gbs,
            "reserve_sms": reserve_sms,
            "projected_ms_no_overlap": max(r["prefill_ms"] + r["transfer_ms"] for r in ranks),
            "projected_ms_overlap": max(r["overlapped_ms"] for r in ranks),
            "exposed_transfer_ms_max": max(r["exposed_transfer_ms"] for r in ranks),
            "note": "projection from one GPU: per-rank prefill timed on its own rows (all ranks back to back, "
                    "second pass), as one launch and as the overlapped split (a capped launch of local tiles "
                    "during the exchange, then every other tile); K/V transfer = bytes / measured 770 GB/s peer "
                    "copy; the indexer, selection and centroid all-gather (<1 ms) are not included"}


def time_e2e(rtp, w, res, steps, device, chunks=16):
    """The same layer from pinned host buffers through the public host entry
    point (rtp_hybrid_prefill_host: chunked, uploads / kernels / downloads
    overlapped), copies inside the timed region; plus, for context, the
    serial form (all uploads, the layer, the download) on one stream."""
    q, k, v = res["q"], res["k"], res["v"]
    plan, bufs, proj = res["plan"], res["bufs"], res["proj"]
    try:
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        ho = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    except RuntimeError as e:
        return {"error": f"pinned host allocation failed: {e}"}
    hq.copy_(q)
    hk.copy_(k)
    hv.copy_(v)
    stream = torch.cuda.current_stream()
    algo, _ = layer_flops(w, res["kinds"])

    def timed(fn):
        times = []
        for _ in range(steps + 1):
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        return statistics.median(times[1:])

    pl = rtp.HostPipeline(plan.cfg, res["kinds"], chunks, device=device)
    t = timed(lambda: pl.run(hq, hk, hv, proj, ho, stream))
    status = rtp.rtp_last_device_status(stream)
    pl.close()
    del pl
    torch.cuda.empty_cache()
    dq, dk, dv, do = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(q)

    def serial():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        plan.run(dq, dk, dv, proj, do, bufs, stream)
        ho.copy_(do, non_blocking=True)

    t_serial = timed(serial)
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
    d2h = ho.numel() * 2
    del hq, hk, hv, ho, dq, dk, dv, do
    return {"value": algo / (t * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": t, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "api": f"rtp_hybrid_prefill_host, {chunks} chunks",
            "status": rtp.status_str(status), "serial_ms_per_step": t_serial,
            "serial_note": "uploads, layer and download one after another on one stream"}


def time_layers(rtp, wid, steps, device):
    """A 48-layer prefill pass (one pass = all layers, buffers per layer):
    the 128K V2 model (workload 2) or the 32K V1 model (workload 1)."""
    w = inputs.workload(wid)
    layers = []
    for l in range(w.layers):
        d, plan, bufs = make_layer(rtp, w, l, device)
        layers.append((d, plan, bufs))
    o = torch.empty_like(layers[0][0]["q"])
    stream = torch.cuda.current_stream()

    def one_pass():
        for d, plan, bufs in layers:
            plan.run(d["q"], d["k"], d["v"], d["proj"], o, bufs, stream)

    for _ in range(1):
        one_pass()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one_pass()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # each kernel separately: one more pass with events between the calls
    evs = []
    for d, plan, bufs in layers:
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        sel = bufs["sel"] if plan.n_sparse else None
        cnt = bufs["sel_cnt"] if plan.n_sparse else None
        e[0].record(stream)
        if plan.n_sparse:
            rtp.rtp_indexer_project(plan.handle, d["q"], d["k"], d["proj"], bufs["centroids"], bufs["qbar"], stream)
        e[1].record(stream)
        if plan.n_sparse:
            rtp.rtp_block_select(plan.handle, bufs["qbar"], bufs["centroids"], sel, cnt, stream)
        e[2].record(stream)
        rtp.rtp_hybrid_prefill(plan.handle, d["q"], d["k"], d["v"], sel, cnt, o, stream)
        e[3].record(stream)
        evs.append(e)
    torch.cuda.synchronize()
    kernels = {name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) for i, name in
               enumerate(("indexer", "select", "prefill"))}
    algo = sum(layer_flops(w, w.kinds[l])[0] for l in range(w.layers))
    execd = sum(layer_flops(w, w.kinds[l])[1] for l in range(w.layers))
    status = rtp.rtp_last_device_status(stream)
    for _, plan, _ in layers:
        plan.close()
    del layers
    torch.cuda.empty_cache()
    return {"workload": w.name, "layers": w.layers, "ms_per_pass": ms, "ms_per_layer": ms / w.layers,
            "kernels_ms_per_pass": kernels,
            "tflops_effective": algo / (ms * 1e-3) / 1e12, "tflops_executed": execd / (ms * 1e-3) / 1e12,
            "status": rtp.status_str(status)}


def time_decode(rtp, steps, device):
    w = inputs.workload(4)
    d = inputs.decode_step(w, device)
    kinds = d["kinds"]
    Lc = d["cache_len"]
    # cached centroids: the library's bulk build over the whole cache (timed below)
    cfg = rtp.AttnConfig(w.batch, Lc, w.n_q_heads, w.n_kv_heads, w.window, w.block, w.topk, w.n_local)
    C = torch.zeros(w.batch, w.n_kv_heads, Lc // w.block, 16, dtype=torch.float32, device=device)
    rtp.rtp_cache_centroids(cfg, kinds, Lc, d["kcache"], d["proj"], C)
    ws_bytes = rtp.rtp_decode_workspace_bytes(cfg, kinds, Lc)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    o = torch.empty_like(d["q"])
    stream = torch.cuda.current_stream()
    args = (cfg, kinds, Lc, d["q"], d["kcache"], d["vcache"], C, d["proj"], o, ws, ws_bytes)
    # L2 flush (the selected K/V of one step, 95 MB, would otherwise stay in the 126 MB L2): write
    # 256 MB, then read another 256 MB so that L2 holds clean lines of unrelated data; with the
    # write alone L2 would start the step full of dirty lines whose write-back the step would pay.
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    flush_read = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    for _ in range(5):
        rtp.rtp_sparse_decode(*args, stream=stream)
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.zero_()
        flush_read.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        rtp.rtp_sparse_decode(*args, stream=stream)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in times)
    status = rtp.rtp_last_device_status(stream)
    rotating = time_decode_rotating(rtp, w, d, C, cfg, steps, stream)
    upkeep = time_cache_upkeep(rtp, w, d, C, cfg, flush, flush_read, steps, stream)
    clustered = time_clustered_decode(rtp, w, d, flush, flush_read, steps, stream)
    bytes_, flops = decode_work(w, kinds, Lc)
    return {"workload": w.name, "ms_per_step": ms, "algorithmic_bytes": bytes_, "gb_s": bytes_ / (ms * 1e-3) / 1e9,
            "tflops_effective": flops / (ms * 1e-3) / 1e12, "l2": "flushed before each step (256 MB write, then 256 MB read)",
            "launches_per_step": 3, "status": rtp.status_str(status), "rotating": rotating,
            "cache_upkeep": upkeep, "clustered": clustered}


def time_decode_rotating(rtp, w, d, C, cfg, steps, stream, n_problems=4):
    """The decode step with inputs larger than L2 instead of a flush: four
    independent problems (the cache rolled along its rows by different
    offsets, so each selects other blocks and streams other rows) taken in
    turn, so that the three steps between two visits of a problem stream
    ~285 MB of other K/V through the 126 MB L2.  Each step's K/V and
    centroids come from DRAM as with the flush; the kernels' code, launch
    parameters and address translations stay warm, as in a decode loop that
    runs the same kernels layer after layer."""
    kinds, Lc = d["kinds"], d["cache_len"]
    probs = [(d["q"], d["kcache"], d["vcache"], C)]
    for r in range(1, n_problems):
        shift = r * 37 * w.block + 5 * r
        kc = torch.roll(d["kcache"], shifts=shift, dims=2)
        vc = torch.roll(d["vcache"], shifts=shift, dims=2)
        Cr = torch.zeros_like(C)
        rtp.rtp_cache_centroids(cfg, kinds, Lc, kc, d["proj"], Cr)
        probs.append((torch.roll(d["q"], shifts=r, dims=1).contiguous(), kc, vc, Cr))
    ws_bytes = rtp.rtp_decode_workspace_bytes(cfg, kinds, Lc)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=d["q"].device)
    outs = [torch.empty_like(d["q"]) for _ in probs]

    def step(i):
        q, kc, vc, Cr = probs[i % n_problems]
        rtp.rtp_sparse_decode(cfg, kinds, Lc, q, kc, vc, Cr, d["proj"], outs[i % n_problems], ws, ws_bytes,
                              stream=stream)

    for i in range(3 * n_problems):
        step(i)
    torch.cuda.synchronize()
    times = []
    for i in range(max(steps, 4 * n_problems)):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step(i)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in times)
    status = rtp.rtp_last_device_status(stream)
    del probs, outs, ws
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "problems": n_problems, "status": rtp.status_str(status),
            "l2": "no flush: four independent problems in turn, ~285 MB of other K/V between two visits of one"}


def time_kmeans_one_sequence(rtp, device, n_clusters=2048, iters=8):
    """k-means of one sequence of the decode workload's cache (3 clustered
    heads, 262,144 rows each): a small case for profiling the clustering
    kernels; warm, median of 5 runs after one, in place (no K/V copy)."""
    w = inputs.workload(4)
    d = inputs.decode_step(w, device, batch=1)
    Lc = d["cache_len"]
    clu_end = (Lc // w.block - w.n_local) * w.block
    runs = []
    for i in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        rtp.cluster_cache(d["kcache"], d["vcache"], d["proj"], d["kinds"], clu_end=clu_end, n_clusters=n_clusters,
                          iters=iters, block=w.block, in_place=True)
        b.record()
        torch.cuda.synchronize()
        if i > 0:
            runs.append(a.elapsed_time(b))
    return {"ms": statistics.median(runs), "clusters": n_clusters, "rounds": iters, "keys_per_head": clu_end - w.block,
            "heads": sum(1 for k in d["kinds"] if k == inputs.SPARSE), "status": rtp.status_str(rtp.rtp_last_device_status()),
            "note": "includes the arrays' allocation by cluster_cache (outside the kernels)"}


def time_clustered_decode(rtp, w, d, flush, flush_read, steps, stream, n_clusters=2048, iters=8):
    """Decode with k-means-clustered retrieval heads on the decode workload:
    the clustering of rows [block, clu_end) of every retrieval head (clu_end
    leaves the last n_local blocks as the unclustered tail), then the decode
    step selecting top-k chunks of <= 128 keys (L2 flushed as for the main
    decode step)."""
    kinds, Lc = d["kinds"], d["cache_len"]
    B = w.block
    clu_end = (Lc // B - w.n_local) * B
    ns = sum(1 for k in kinds if k == inputs.SPARSE)
    # k-means, warm: the clusters' arrays and the workspace are allocated once,
    # outside the timed region; the median of 5 timed runs after a warm-up
    ccfg = rtp.AttnConfig(w.batch, Lc, w.n_kv_heads, w.n_kv_heads, 1, B, 0, 1)
    cl = rtp.Clusters(w.batch, w.n_kv_heads, clu_end, n_clusters, B, d["kcache"].device)
    km_ws_bytes = rtp.rtp_cache_cluster_workspace_bytes(ccfg, clu_end)
    km_ws = torch.empty(km_ws_bytes, dtype=torch.uint8, device=d["kcache"].device)
    km_runs = []
    for i in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        rtp.rtp_cache_cluster(ccfg, kinds, iters, d["kcache"], d["vcache"], d["proj"], cl, km_ws, km_ws_bytes,
                              stream)
        b.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            km_runs.append(a.elapsed_time(b))
    km_ms = statistics.median(km_runs)
    # the same clustering in place (no cluster-ordered K/V copy written)
    cl_in = rtp.Clusters(w.batch, w.n_kv_heads, clu_end, n_clusters, B, d["kcache"].device, in_place=True)
    km_in_runs = []
    for i in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        rtp.rtp_cache_cluster(ccfg, kinds, iters, d["kcache"], d["vcache"], d["proj"], cl_in, km_ws, km_ws_bytes,
                              stream)
        b.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            km_in_runs.append(a.elapsed_time(b))
    del km_ws
    cfg = rtp.AttnConfig(w.batch, Lc, w.n_q_heads, w.n_kv_heads, w.window, B, w.topk, w.n_local)
    ws_bytes = rtp.rtp_decode_clustered_workspace_bytes(cfg, kinds, Lc, clu_end)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=d["q"].device)
    o = torch.empty_like(d["q"])
    cnt = torch.zeros(w.batch, w.n_kv_heads, dtype=torch.int32, device=d["q"].device)
    if ws_bytes == 0:
        raise RuntimeError("clustered decode: rejected configuration")
    sel = torch.full((w.batch, w.n_kv_heads, 1 + (Lc - clu_end + 127) // 128 + w.topk), -1,
                     dtype=torch.int32, device=d["q"].device)
    args = (cfg, kinds, Lc, d["q"], d["kcache"], d["vcache"], d["proj"], cl, o, ws, ws_bytes, sel, cnt)
    for _ in range(5):
        rtp.rtp_sparse_decode_clustered(*args, stream=stream)
    torch.cuda.synchronize()
    ev = []
    for _ in range(steps):
        flush.zero_()
        flush_read.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        rtp.rtp_sparse_decode_clustered(*args, stream=stream)
        e1.record(stream)
        ev.append((e0, e1))
    torch.cuda.synchronize()
    ms = statistics.median(x.elapsed_time(y) for x, y in ev)
    # in place: the decode gathers member rows from the cache
    args_in = (cfg, kinds, Lc, d["q"], d["kcache"], d["vcache"], d["proj"], cl_in, o, ws, ws_bytes, sel, cnt)
    for _ in range(5):
        rtp.rtp_sparse_decode_clustered(*args_in, stream=stream)
    torch.cuda.synchronize()
    ev_in = []
    for _ in range(steps):
        flush.zero_()
        flush_read.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        rtp.rtp_sparse_decode_clustered(*args_in, stream=stream)
        e1.record(stream)
        ev_in.append((e0, e1))
    torch.cuda.synchronize()
    ms_in = statistics.median(x.elapsed_time(y) for x, y in ev_in)
    rtp.rtp_sparse_decode_clustered(*args, stream=stream)  # leave the copy-based selection in sel / cnt
    status = rtp.rtp_last_device_status(stream)
    # keys read: every retrieval head's sink block, tail and selected chunks, every window head's window
    sel_c, cnt_c = sel.cpu(), cnt.cpu()
    lens = cl.chunk_len.cpu()
    keys = 0
    for bb in range(w.batch):
        for h, kind in enumerate(kinds):
            if kind == inputs.SPARSE:
                m = int(cnt_c[bb, h]) - 1 - (Lc - clu_end + 127) // 128
                keys += B + (Lc - clu_end) + sum(int(lens[bb, h, int(x)]) for x in sel_c[bb, h, 1:1 + m])
            else:
                keys += min(w.window, Lc)
    bytes_ = keys * 128 * 2 * 2 + w.batch * ns * cl.max_chunks * 16 * 4 + w.batch * w.n_q_heads * 128 * 2 * 2
    chunks = cl.n_chunks.cpu()[:, [h for h, k in enumerate(kinds) if k == inputs.SPARSE]].float()
    copy_bytes = 2 * w.batch * ns * (clu_end - B) * 128 * 2
    return {"n_clusters": n_clusters, "iters": iters, "clu_end": clu_end, "kmeans_ms": km_ms,
            "kmeans_ms_runs": km_runs,
            "in_place": {"kmeans_ms": statistics.median(km_in_runs), "ms_per_step": ms_in,
                         "copy_bytes_saved": copy_bytes,
                         "note": "no cluster-ordered K/V copy: the decode gathers member rows (16-byte cp.async)"},
            "mean_chunks_per_head": float(chunks.mean()), "ms_per_step": ms, "algorithmic_bytes": bytes_,
            "gb_s": bytes_ / (ms * 1e-3) / 1e9, "status": rtp.status_str(status)}


def time_cache_upkeep(rtp, w, d, C, cfg, flush, flush_read, steps, stream):
    """The KV-cache calls on the decode workload: the bulk centroid build over
    every cached block, and one append (new K/V row; the row completes a block,
    so its centroid is recomputed for each retrieval head).  The appended row
    is the cache's own last row, so the cache keeps its contents."""
    kinds, Lc = d["kinds"], d["cache_len"]
    ns = sum(1 for k in kinds if k == inputs.SPARSE)

    def timed(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = []
        for _ in range(n):
            flush.zero_()
            flush_read.sum()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    build_ms = timed(lambda: rtp.rtp_cache_centroids(cfg, kinds, Lc, d["kcache"], d["proj"], C, stream=stream), 10)
    build_bytes = w.batch * ns * (Lc // w.block) * (w.block * 128 * 2 + 16 * 4)
    k_new = d["kcache"][:, :, Lc - 1].contiguous()
    v_new = d["vcache"][:, :, Lc - 1].contiguous()
    app_ms = timed(lambda: rtp.rtp_cache_append(cfg, kinds, Lc - 1, k_new, v_new, d["kcache"], d["vcache"],
                                                d["proj"], C, stream=stream), min(steps, 64))
    app_bytes = w.batch * w.n_kv_heads * 4 * 128 * 2 + w.batch * ns * (w.block * 128 * 2 + 16 * 4)
    k_mid = d["kcache"][:, :, Lc - 2].contiguous()
    v_mid = d["vcache"][:, :, Lc - 2].contiguous()
    row_ms = timed(lambda: rtp.rtp_cache_append(cfg, kinds, Lc - 2, k_mid, v_mid, d["kcache"], d["vcache"],
                                                d["proj"], C, stream=stream), min(steps, 64))
    return {"append_row_only_us": row_ms * 1e3,"centroid_build_ms": build_ms, "centroid_build_algorithmic_bytes": build_bytes,
            "centroid_build_gb_s": build_bytes / (build_ms * 1e-3) / 1e9,
            "append_us": app_ms * 1e3, "append_algorithmic_bytes": app_bytes,
            "append_note": "row completes a block: its centroid is recomputed for every retrieval head"}


# ---------------------------------------------------------------- oracle arm


class OracleSample:
    """The CPU oracle timed on a bounded sample of one layer of workload w.

    Prepared once: the layer's inputs (generated on the device) and, for the
    retrieval head, its K/V and block centroids over all keys on the host.
    A step then runs the oracle for random query rows of every head: for the
    retrieval group the summaries and selection of the rows' query blocks,
    then exact attention; it keeps going until `budget_s` has passed.
    """

    def __init__(self, w, layer, device):
        import oracle

        self.oracle = oracle
        self.w = w
        self.d = inputs.prefill_layer(w, layer, device)
        self.device = device
        self.threads = int(os.environ.get("ORACLE_THREADS", os.cpu_count() or 1))
        self.k_cpu = {h: self.d["k"][0, h].cpu() for h in range(w.n_kv_heads)}
        self.v_cpu = {h: self.d["v"][0, h].cpu() for h in range(w.n_kv_heads)}
        self.proj = self.d["proj"].cpu()
        t0 = time.perf_counter()
        self.C = {h: oracle.centroids(self.k_cpu[h], w.block, self.proj)
                  for h, kind in enumerate(self.d["kinds"]) if kind == inputs.SPARSE}
        self.centroid_seconds = time.perf_counter() - t0

    def step(self, budget_s: float, seed: int):
        oracle, w, d = self.oracle, self.w, self.d
        rng = np.random.default_rng(seed)
        G, B, n = w.group, w.block, w.seq
        rows_per_head = max(8, self.threads)
        flops, done_rows = 0.0, 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < budget_s:
            for hq in range(w.n_q_heads):
                kvh = hq // G
                kind = d["kinds"][kvh]
                rows = np.sort(rng.integers(0, n, rows_per_head))
                qr = d["q"][0, hq][torch.from_numpy(rows).to(self.device)].cpu()
                if kind == inputs.SPARSE:
                    ts = np.unique(rows // B).astype(np.int32)
                    qb = np.zeros((n // B, 16))
                    for t in ts:
                        qb[t] = oracle.qbar(d["q"][0, kvh * G:(kvh + 1) * G, t * B:(t + 1) * B].cpu(), B,
                                            self.proj)[0]
                    sel_rows, cnt_rows, _ = oracle.select(qb[ts], self.C[kvh], ts, w.topk, w.n_local)
                    sel = np.full((n // B, w.kmax), -1, dtype=np.int32)
                    cnt = np.zeros(n // B, dtype=np.int32)
                    sel[ts] = sel_rows
                    cnt[ts] = cnt_rows
                    oracle.attention_rows(qr, rows, self.k_cpu[kvh], self.v_cpu[kvh], oracle.SPARSE, 0, B, sel, cnt)
                    for r in rows:
                        t = r // B
                        flops += (int(cnt[t] - 1) * B + (r - t * B + 1)) * 4 * 128
                else:
                    mode = oracle.SWA if kind == inputs.SWA else oracle.FULL
                    oracle.attention_rows(qr, rows, self.k_cpu[kvh], self.v_cpu[kvh], mode, w.window)
                    for r in rows:
                        vis = r + 1 if mode == oracle.FULL else min(r + 1, w.window)
                        flops += vis * 4 * 128
                done_rows += len(rows)
        secs = time.perf_counter() - t0
        desc = (f"{done_rows} random query rows (every head) of one {w.name} layer: exact attention, plus query "
                f"summaries and selection of their query blocks; the retrieval head's centroids over all {n} keys "
                f"took a further {self.centroid_seconds:.1f} s once, not counted")
        return flops / secs / 1e12, secs, desc


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = inputs.workload(3)
    device = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    sample = OracleSample(w, 0, device)
    vals = []
    for s in range(args.warmup + args.steps):
        val, secs, desc = sample.step(args.ref_step_seconds, seed=s)
        if s >= args.warmup:
            vals.append((val, secs))
    value = statistics.median(v for v, _ in vals)
    ms = statistics.median(s for _, s in vals) * 1e3
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "seq": w.seq, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
                       "kinds": w.kinds[0], "block": w.block, "topk": w.topk, "n_local": w.n_local,
                       "window": w.window},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": sample.threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def secondary_summary(sec: dict) -> dict:
    """The secondary figures in a few short keys (ms unless named _us)."""
    out = {}
    d = sec.get("decode_8x256k") or {}
    if "ms_per_step" in d:
        out["decode_8x256k_us"] = round(d["ms_per_step"] * 1e3, 2)
        out["decode_hbm_frac"] = round(d["gb_s"] / 6552.6, 3) if "gb_s" in d else None
        if (d.get("rotating") or {}).get("ms_per_step"):
            out["decode_rotating_us"] = round(d["rotating"]["ms_per_step"] * 1e3, 2)
        c = d.get("clustered") or {}
        if "ms_per_step" in c:
            out["clustered_decode_us"] = round(c["ms_per_step"] * 1e3, 2)
        if "in_place" in c:
            out["clustered_in_place_decode_us"] = round(c["in_place"]["ms_per_step"] * 1e3, 2)
            out["kmeans_in_place_ms"] = round(c["in_place"]["kmeans_ms"], 2)
        if "kmeans_ms" in c:
            out["kmeans_ms"] = round(c["kmeans_ms"], 2)
    for key, name in (("v2_128k_48_layers", "v2_128k_ms_per_layer"), ("v1_32k_48_layers", "v1_32k_ms_per_layer")):
        if "ms_per_layer" in sec.get(key, {}):
            out[name] = round(sec[key]["ms_per_layer"], 3)
            out[name.replace("ms_per_layer", "tflops_executed")] = round(sec[key]["tflops_executed"], 1)
    cp = sec.get("context_parallel_projection") or {}
    for key in ("projected_ms_no_overlap", "projected_ms_overlap", "exposed_transfer_ms_max"):
        if key in cp:
            out["cp8_" + key] = round(cp[key], 3)
    dyn = sec.get("dynamic_selection") or {}
    for key in ("rowmax_scores", "per_head"):
        if key in dyn:
            out[key + "_select_ms"] = round(dyn[key]["select_ms"], 3)
            out[key + "_prefill_ms"] = round(dyn[key]["prefill_ms"], 2)
    return out


def run_ours(args, rank, world, local):
    from swa_hybrid_attention_b200 import build

    if rank == 0:
        build.build()
    barrier(world)
    from swa_hybrid_attention_b200 import rtp

    device = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    if args.only == "decode":
        if rank == 0:
            print(json.dumps({"decode_8x256k": time_decode(rtp, args.decode_steps, device)}), flush=True)
        return
    if args.only == "kmeans":
        if rank == 0:
            print(json.dumps({"kmeans_one_sequence": time_kmeans_one_sequence(rtp, device)}), flush=True)
        return
    w = inputs.workload(3)
    if args.seq:
        # same head structure at a shorter length (profiling runs)
        w.seq = args.seq
        w.name = f"{w.name}@{args.seq}"
        w.needles = max(1, w.needles * args.seq // 1048576)
    if args.only == "selection":
        if rank == 0:
            print(json.dumps({"selection_variants": time_selection_variants(rtp, w, device)}), flush=True)
        return
    res = time_primary(rtp, w, rank_layer(rank), args.steps, args.warmup, device, world)
    algo, execd = layer_flops(w, res["kinds"])
    step_ms = max_over_ranks(res["total_ms"] / args.steps, world)
    pre_ms = statistics.mean(res["per"]["prefill"])
    idx_ms = statistics.mean(res["per"]["indexer"])
    sel_ms = statistics.mean(res["per"]["select"])
    value = world * algo / (step_ms * 1e-3) / 1e12
    achieved = execd / (pre_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    traffic = prefill_traffic(w)
    extra = {}
    if args.only == "cp":
        if rank == 0:
            print(json.dumps({"context_parallel_projection": time_cp_projection(rtp, w, res, device)}), flush=True)
        return
    if not args.no_secondary and world == 1:
        extra["dynamic"] = time_dynamic(rtp, w, res, device)
        extra["cp"] = time_cp_projection(rtp, w, res, device)
    if not args.no_e2e:
        e2e = time_e2e(rtp, w, res, max(2, min(args.steps, 3)), device, args.e2e_chunks)
        # whole job: every rank's layer, over the slowest rank's time (every rank
        # takes part in the reduction, also one whose pinned allocation failed)
        t_max = max_over_ranks(e2e.get("ms_per_step", float("inf")), world)
        if "error" not in e2e:
            e2e["value"] = world * algo / (t_max * 1e-3) / 1e12
            e2e["ms_per_step"] = t_max
            e2e["h2d_bytes_per_step"] *= world
            e2e["d2h_bytes_per_step"] *= world
        extra["e2e"] = e2e
    for key in ("q", "k", "v", "o"):
        res[key] = None
    res["plan"].close()
    torch.cuda.empty_cache()
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(w, 0, device)
        val, secs, desc = sample.step(args.cpu_seconds, seed=0)
        cpu_base = {"value": val, "unit": "TFLOP/s", "cores": sample.threads, "kind": "oracle", "sample": desc}
        del sample
        torch.cuda.empty_cache()
    secondary = {}
    if not args.no_secondary and world == 1:
        secondary["v2_128k_48_layers"] = time_layers(rtp, 2, 2, device)
        secondary["v1_32k_48_layers"] = time_layers(rtp, 1, 3, device)
        secondary["decode_8x256k"] = time_decode(rtp, args.decode_steps, device)
        if extra.get("dynamic"):
            secondary["dynamic_selection"] = extra["dynamic"]
        if extra.get("cp"):
            secondary["context_parallel_projection"] = extra["cp"]
    if rank != 0:
        return
    clocks = res["clocks"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "seq": w.seq, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
                   "kinds": res["kinds"], "block": w.block, "topk": w.topk, "n_local": w.n_local,
                   "window": w.window, "needles": w.needles, "l2": "inputs larger than L2 (Q 8.6 GB), no flush",
                   "parallelism": f"independent layer per rank x{world}"},
        "roofline": {"bound": "tensor", "kernel": "hybrid_prefill_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} (sustained bf16, kernel timed inside back-to-back steps)",
                     "executed_flops_per_launch": execd, "ms_per_launch": pre_ms},
        "kernels_ms": {"indexer": idx_ms, "select": sel_ms, "prefill": pre_ms},
        "algorithmic_flops_per_step": algo, "executed_flops_per_step": execd,
        "tflops_executed": execd / (step_ms * 1e-3) / 1e12,
        "indexer_gb_s": indexer_bytes(w, res["kinds"]) / (idx_ms * 1e-3) / 1e9,
        "gpu_launches": res["launches"],
        "device_status": rtp.status_str(res["status"]),
    }
    if clocks:
        line["clocks"] = clocks
    if "e2e" in extra:
        line["e2e"] = extra["e2e"]
    if cpu_base:
        line["cpu_baseline"] = cpu_base
    if secondary:
        line["secondary"] = secondary
        line["summary"] = secondary_summary(secondary)  # last, short: the end of the line carries the key figures
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=16, help="chunks of the host-memory pipeline (e2e)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=10.0)
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--seq", type=int, default=0, help="override the primary workload's length (profiling)")
    ap.add_argument("--only", choices=["all", "decode", "selection", "cp", "kmeans"], default="all",
                    help="run only part of the bench (decode step; selection variants, for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_setup(args.gpus) if torch.cuda.is_available() else (0, 1, 0)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
