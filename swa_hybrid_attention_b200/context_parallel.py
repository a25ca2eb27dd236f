"""Context-parallel prefill of one layer over the ranks of a process group.

RTPurbo page, "RTP-LLM：RTPurbo 在长文上的极致性能优化": with head-wise
sparsity, tensor parallelism (heads split over GPUs) leaves GPUs unevenly
loaded, so the engine uses context parallelism: every GPU computes the
attention of all heads for its own part of the context, and communication
overlaps computation.

Rank r owns the query rows [begin_r, end_r) (a contiguous run of 128-row
tiles) and holds Q, K and V of those rows.  Its attention needs, for every
(sequence, KV head), some earlier K/V rows owned by lower ranks:
  * streaming (SWA) heads: the window before begin_r, [begin_r - W + 1, begin_r);
  * full heads: every earlier row, [0, begin_r);
  * sparse heads: the earlier blocks its query blocks selected; selection
    needs the centroids of every earlier block, which are all-gathered first
    (16 fp32 per block).
The rows are requested from their owners and delivered with two all-to-alls
(request lists, then payload); received rows land in this GPU's memory
before any kernel reads them (no kernel reads another GPU's memory).  The
attention itself is the library's prefill on a split ranged plan
(rtp_route_heads_split), so a rank computes exactly the tiles the
single-GPU prefill would compute for its rows, bit for bit.

Overlap: the plan's work list starts with the tiles whose visible keys are
all this rank's own rows (streaming heads whose window starts inside the
range).  The first of them run on the compute stream, on all but a few SMs
so that the collectives' kernels have SMs to run on (a prefill CTA holds an
SM's registers), while the exchange runs on a side stream; as many as take
about as long as the exchange.  Every other tile — the remaining local ones
and those that need fetched rows (full and sparse heads always see row 0;
streaming tiles near the range's start) — runs in one launch once the
exchange is done.

This module is host-side orchestration: which rows to fetch, and the
collectives (torch.distributed, NCCL on GPUs; gloo with host staging where
no NCCL group exists).  The attention, indexer and selection run in the
library's kernels.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import rtp

SWA, FULL, SPARSE = 0, 1, 2


# ------------------------------------------------------------------ layout


def cp_ranges(seq: int, world: int) -> list:
    """Query rows of each rank: contiguous runs of whole 128-row tiles, as
    even as the tile count allows (the last run may end in a partial tile)."""
    tiles = (seq + 127) // 128
    if world < 1 or tiles < world:
        raise ValueError(f"{tiles} query tiles cannot be shared by {world} ranks")
    return [(128 * (r * tiles // world), min(seq, 128 * ((r + 1) * tiles // world))) for r in range(world)]


def _merge(intervals: list) -> list:
    out = []
    for lo, hi in sorted(intervals):
        if hi <= lo:
            continue
        if out and lo <= out[-1][1]:
            out[-1] = (out[-1][0], max(out[-1][1], hi))
        else:
            out.append((lo, hi))
    return out


def kv_needs(kinds, window: int, block: int, q_range: tuple, batch: int, sel=None, cnt=None,
             slot_of: dict | None = None) -> dict:
    """Earlier K/V rows the queries of q_range can see, per (sequence, KV head).

    sel / cnt: this range's selection (host int tensors [batch][n_sparse][nb][kmax]
    and [batch][n_sparse][nb], whole-sequence layout; only the range's rows
    are read) for the sparse heads.  Returns {(b, h): [(lo, hi), ...]}, sorted
    disjoint row intervals below q_range[0]; heads that need nothing are absent.
    """
    qb, qe = q_range
    needs = {}
    for b in range(batch):
        for h, kind in enumerate(kinds):
            iv = []
            if kind == SWA:
                lo = max(0, qb - window + 1)
                if lo < qb:
                    iv = [(lo, qb)]
            elif kind == FULL:
                if qb > 0:
                    iv = [(0, qb)]
            else:
                s = slot_of[h]
                t_lo, t_hi = qb // block, (qe + block - 1) // block
                blocks = set()
                for t in range(t_lo, t_hi):
                    n = int(cnt[b, s, t])
                    for e in range(n):
                        blk = int(sel[b, s, t, e])
                        if 0 <= blk and (blk + 1) * block <= qb:
                            blocks.add(blk)
                iv = _merge([(blk * block, (blk + 1) * block) for blk in blocks])
            if iv:
                needs[(b, h)] = iv
    return needs


def split_by_owner(needs: dict, ranges: list) -> list:
    """Per owner rank: int64 tensor [n, 4] of requests (b, h, lo, hi), each
    inside that owner's rows, in a fixed order."""
    per = [[] for _ in ranges]
    for (b, h) in sorted(needs):
        for lo, hi in needs[(b, h)]:
            for s, (ob, oe) in enumerate(ranges):
                a, z = max(lo, ob), min(hi, oe)
                if a < z:
                    per[s].append((b, h, a, z))
    return [torch.tensor(p, dtype=torch.int64).reshape(-1, 4) for p in per]


# -------------------------------------------------------------- transport


def _staged(group) -> bool:
    return dist.get_backend(group) == "gloo"


def _all_to_all(out: torch.Tensor, inp: torch.Tensor, out_splits: list, in_splits: list, group) -> None:
    """all_to_all_single on flat tensors; through host memory for gloo.
    bf16 payloads (even-sized pieces: whole K and V rows) travel as pairs of
    16-bit patterns in int32 words, which every backend supports."""
    if out.dtype == torch.bfloat16:
        assert all(n % 2 == 0 for n in out_splits + in_splits)
        out, inp = out.view(torch.int32), inp.view(torch.int32)
        out_splits, in_splits = [n // 2 for n in out_splits], [n // 2 for n in in_splits]
    if _staged(group) and inp.is_cuda:
        o = torch.empty(out.shape, dtype=out.dtype)
        dist.all_to_all_single(o, inp.cpu(), out_splits, in_splits, group=group)
        out.copy_(o)
    else:
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=group)


def _all_gather(parts: list, x: torch.Tensor, group) -> None:
    if _staged(group) and x.is_cuda:
        host = [torch.empty(p.shape, dtype=p.dtype) for p in parts]
        dist.all_gather(host, x.cpu(), group=group)
        for p, h in zip(parts, host):
            p.copy_(h)
    else:
        dist.all_gather(parts, x, group=group)


def exchange_kv(k_loc: torch.Tensor, v_loc: torch.Tensor, needs: dict, ranges: list, rank: int, kf: torch.Tensor,
                vf: torch.Tensor, group=None, copy_own: bool = True) -> int:
    """Fill kf / vf ([batch][H][>= end][128]) with the rows in `needs`,
    fetched from their owners, and (copy_own) this rank's own rows.  k_loc /
    v_loc hold this rank's rows [begin, end).  Every rank of the group must
    call it (it runs three all-to-alls).  Returns the payload bytes received."""
    world = len(ranges)
    dev = k_loc.device
    qb, qe = ranges[rank]
    if copy_own:
        kf[:, :, qb:qe].copy_(k_loc)
        vf[:, :, qb:qe].copy_(v_loc)
    reqs = split_by_owner(needs, ranges)
    assert reqs[rank].numel() == 0, "a rank never needs rows it owns from itself"
    # 1. how many requests go to / come from each rank
    send_n = torch.tensor([r.shape[0] for r in reqs], dtype=torch.int64, device=dev)
    recv_n = torch.empty_like(send_n)
    _all_to_all(recv_n, send_n, [1] * world, [1] * world, group)
    recv_n = recv_n.tolist()
    # 2. the request lists
    send_req = torch.cat(reqs).reshape(-1).to(dev)
    recv_req = torch.empty(4 * sum(recv_n), dtype=torch.int64, device=dev)
    _all_to_all(recv_req, send_req, [4 * n for n in recv_n], [4 * r.shape[0] for r in reqs], group)
    got = recv_req.reshape(-1, 4).tolist()
    # 3. payload: for each request, its K rows then its V rows
    row = k_loc.shape[-1]
    pieces, send_sizes = [], []
    i = 0
    for s in range(world):
        size = 0
        for b, h, lo, hi in got[i:i + recv_n[s]]:
            assert qb <= lo < hi <= qe, "request outside the owner's rows"
            pieces.append(k_loc[b, h, lo - qb:hi - qb].reshape(-1))
            pieces.append(v_loc[b, h, lo - qb:hi - qb].reshape(-1))
            size += 2 * (hi - lo) * row
        send_sizes.append(size)
        i += recv_n[s]
    send = torch.cat(pieces) if pieces else torch.empty(0, dtype=k_loc.dtype, device=dev)
    recv_sizes = [int(2 * (r[:, 3] - r[:, 2]).sum()) * row if r.numel() else 0 for r in reqs]
    recv = torch.empty(sum(recv_sizes), dtype=k_loc.dtype, device=dev)
    _all_to_all(recv, send, recv_sizes, send_sizes, group)
    # 4. place the received rows
    off = 0
    for s in range(world):
        for b, h, lo, hi in reqs[s].tolist():
            n = (hi - lo) * row
            kf[b, h, lo:hi].copy_(recv[off:off + n].view(hi - lo, row))
            vf[b, h, lo:hi].copy_(recv[off + n:off + 2 * n].view(hi - lo, row))
            off += 2 * n
    return recv.numel() * recv.element_size()


def gather_centroids(centroids: torch.Tensor, ranges: list, rank: int, block: int, group=None) -> None:
    """All-gather the centroid blocks each rank computed for its own rows
    (whole-sequence layout [batch][n_sparse][nb][16]; rank r wrote blocks
    begin_r/block .. end_r/block - 1)."""
    spans = [(qb // block, qe // block) for qb, qe in ranges]
    width = max(hi - lo for lo, hi in spans)
    lo, hi = spans[rank]
    mine = torch.zeros(centroids.shape[0], centroids.shape[1], width, centroids.shape[3], dtype=centroids.dtype,
                       device=centroids.device)
    mine[:, :, :hi - lo].copy_(centroids[:, :, lo:hi])
    parts = [torch.empty_like(mine) for _ in ranges]
    _all_gather(parts, mine.contiguous(), group)
    for (a, z), p in zip(spans, parts):
        centroids[:, :, a:z].copy_(p[:, :, :z - a])


# ------------------------------------------------------------------ layer


# Planner cost of one work item, in KV tiles of 128 keys (the same count the
# library's longest-first ordering uses), for sizing the overlapped launch.
def _item_tiles(item, cfg: rtp.AttnConfig) -> int:
    kind, t = int(item[0]) & 0xFF, int(item[3])
    if kind == FULL:
        return t + 1
    if kind == SWA:
        first = 128 * t - cfg.window + 1
        return t - (0 if first <= 0 else first // 128) + 1
    return min(t + 1, cfg.topk + 1 + cfg.n_local)


def overlap_head_items(items, n_local: int, cfg: rtp.AttnConfig, exchange_s: float, ctas: int,
                       tile_s: float = 2.4e-6) -> int:
    """How many of the first local items the capped launch should run so that
    it lasts a little longer than the exchange (a quarter more): ctas CTAs,
    each taking a KV tile of one query-head pair in about tile_s seconds (the
    prefill kernel's measured rate on B200: ~2.4 us per pair-tile per SM)."""
    budget = 1.25 * exchange_s / tile_s * ctas
    acc = 0
    for i in range(n_local):
        if acc >= budget:
            return i
        acc += _item_tiles(items[i], cfg)
    return n_local


def cp_prefill_layer(q_loc, k_loc, v_loc, kinds, proj, cfg: rtp.AttnConfig, group=None, dynamic: dict | None = None,
                     stream=None, overlap: bool = True, reserve_sms: int = 16, link_gbs: float = 770.0) -> tuple:
    """One layer of context-parallel prefill on this rank.

    cfg describes the whole sequence (cfg.seq = total tokens); q_loc, k_loc,
    v_loc hold this rank's rows of cp_ranges(cfg.seq, world)[rank].  Returns
    (o_loc, info) with o_loc the attention output of this rank's rows and
    info the bytes received, the rows fetched and the work split.
    overlap: while the exchange is in flight (side stream), run tiles that
    need no fetched row, on reserve_sms fewer CTAs, as many as the exchange's
    duration at link_gbs allows; the rest after it.  stream: a torch.cuda.Stream
    (None: the current stream); everything this rank queues goes on it, the
    exchange on a side stream joined before the remote tiles.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ranges = cp_ranges(cfg.seq, world)
    qb, qe = ranges[rank]
    assert q_loc.shape[2] == qe - qb and k_loc.shape[2] == qe - qb
    dev = q_loc.device
    comp = torch.cuda.current_stream(dev) if stream is None else stream
    plan = rtp.Plan(cfg, kinds, comp, q_range=(qb, qe), key_begin=qb)
    try:
        with torch.cuda.stream(comp):
            bufs = plan.buffers(dev)
            slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
            sel = cnt = None
            if plan.n_sparse:
                rtp.rtp_indexer_project(plan.handle, q_loc, k_loc, proj, bufs["centroids"], bufs["qbar"], comp)
                gather_centroids(bufs["centroids"], ranges, rank, cfg.block, group)
                if dynamic is None:
                    rtp.rtp_block_select(plan.handle, bufs["qbar"], bufs["centroids"], bufs["sel"],
                                         bufs["sel_cnt"], comp)
                else:
                    beta = dynamic.get("beta")
                    rtp.rtp_block_select_dynamic(plan.handle, bufs["qbar"], bufs["centroids"], dynamic["mass"],
                                                 dynamic.get("min_k", 0),
                                                 rtp.default_selection_beta(cfg) if beta is None else beta,
                                                 bufs["sel"], bufs["sel_cnt"], comp)
                sel, cnt = bufs["sel"].cpu(), bufs["sel_cnt"].cpu()
            needs = kv_needs(kinds, cfg.window, cfg.block, (qb, qe), cfg.batch, sel, cnt, slot_of)
            rows = sum(hi - lo for iv in needs.values() for lo, hi in iv)
            kf = torch.empty(cfg.batch, cfg.n_kv_heads, qe, 128, dtype=k_loc.dtype, device=dev)
            vf = torch.empty_like(kf)
            kf[:, :, qb:qe].copy_(k_loc)
            vf[:, :, qb:qe].copy_(v_loc)
            o_loc = torch.empty_like(q_loc)
            sel_d = bufs["sel"] if plan.n_sparse else None
            cnt_d = bufs["sel_cnt"] if plan.n_sparse else None
            n_loc, n_all = plan.n_local, plan.n_items
            n_head = 0
            if overlap and world > 1 and n_loc > 0:
                sms = torch.cuda.get_device_properties(dev).multi_processor_count
                ctas = max(1, sms - reserve_sms)
                exchange_s = 2 * rows * 128 * k_loc.element_size() / (link_gbs * 1e9)
                n_head = overlap_head_items(rtp.rtp_plan_work_items(plan.handle), n_loc, cfg, exchange_s, ctas)
                side = torch.cuda.Stream(dev)
                side.wait_stream(comp)
                # queued before the exchange, whose host side blocks on its own stream only
                rtp.rtp_hybrid_prefill_items(plan.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc, 0, n_head, ctas, comp)
                with torch.cuda.stream(side):
                    received = exchange_kv(k_loc, v_loc, needs, ranges, rank, kf, vf, group, copy_own=False)
                comp.wait_stream(side)
                # the rest, local and remote tiles in one launch (one tail instead of two)
                rtp.rtp_hybrid_prefill_items(plan.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc, n_head, n_all, 0, comp)
            else:
                received = exchange_kv(k_loc, v_loc, needs, ranges, rank, kf, vf, group, copy_own=False)
                rtp.rtp_hybrid_prefill(plan.handle, q_loc, kf, vf, sel_d, cnt_d, o_loc, comp)
        return o_loc, {"bytes_received": received, "rows_fetched": rows, "q_range": (qb, qe), "items": n_all,
                       "local_items": n_loc, "head_items": n_head}
    finally:
        plan.close()
