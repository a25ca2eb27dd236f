"""Comparison helpers shared by the GPU parity tests (test code only)."""

from __future__ import annotations

import numpy as np
import torch

import oracle

# Acceptance bounds: bf16 in/out, fp32 accumulation, against the fp64 oracle
# rounded once to bf16, on the GPU's own selection.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
# Selections must be equal except for blocks whose oracle score is within
# this relative distance of the k-th kept score (fp32 vs fp64 near-ties).
TIE_REL = 1e-5
# Indexer outputs (fp32 sums of up to 8 x 128 rows) against fp64.
IDX_ABS = 2e-4
IDX_REL = 2e-4

MODE_OF_KIND = {0: oracle.SWA, 1: oracle.FULL, 2: oracle.SPARSE}


def cpu(x):
    return x.detach().cpu()


def check_indexer(centroids_gpu, qbar_gpu, q, k, proj, slot_heads, block, group):
    """Centroids and query summaries of every slot against the oracle (fp64)."""
    C_all, Q_all = [], []
    for s, kvh in enumerate(slot_heads):
        C = oracle.centroids(cpu(k[0, kvh]), block, cpu(proj))
        Qb = oracle.qbar(cpu(q[0, kvh * group:(kvh + 1) * group]), block, cpu(proj))
        gc = cpu(centroids_gpu[0, s]).double().numpy()
        gq = cpu(qbar_gpu[0, s]).double().numpy()
        assert np.all(np.abs(gc - C) <= IDX_ABS + IDX_REL * np.abs(C)), np.max(np.abs(gc - C))
        assert np.all(np.abs(gq - Qb) <= IDX_ABS + IDX_REL * np.abs(Qb)), np.max(np.abs(gq - Qb))
        C_all.append(C)
        Q_all.append(Qb)
    return C_all, Q_all


def check_selection_rows(sel_gpu, cnt_gpu, Qb, C, t_list, topk, n_local):
    """GPU selection rows (for query blocks t_list) against the oracle's.

    Equal sets, or every differing block is a near-tie of the k-th score.
    Also checks the GPU rows are ascending, unique, and contain the sink and
    local blocks.  Returns the number of near-tie rows.
    """
    sel_o, cnt_o, kth = oracle.select(Qb[t_list], C, t_list, topk, n_local)
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
            s = oracle.scores(Qb[t], C)
            for b in set(g) ^ o:
                assert abs(s[b] - kth[r]) <= TIE_REL * abs(kth[r]), (t, b, s[b], kth[r])
            near += 1
    return near


def check_prefill_rows(o_gpu, q, k, v, kinds, group, window, block, sel_gpu, cnt_gpu, slot_of, rows_of_head,
                       scale=None):
    """O rows of every query head against the oracle on the GPU's selection."""
    worst = 0.0
    kv_cpu = {}
    for hq in range(q.shape[1]):
        kvh = hq // group
        if kvh not in kv_cpu:
            kv_cpu.clear()
            kv_cpu[kvh] = (cpu(k[0, kvh]), cpu(v[0, kvh]))
        k_h, v_h = kv_cpu[kvh]
        mode = MODE_OF_KIND[kinds[kvh]]
        rows = np.asarray(rows_of_head(hq), dtype=np.int64)
        sel = cnt = None
        if mode == oracle.SPARSE:
            sel = cpu(sel_gpu[0, slot_of[kvh]]).numpy()
            cnt = cpu(cnt_gpu[0, slot_of[kvh]]).numpy()
        if rows.size == 0:
            continue
        qr = cpu(q[0, hq][torch.from_numpy(rows).to(q.device)])
        ref = oracle.attention_rows_mm(qr, rows, k_h, v_h, mode, window, block, sel, cnt, scale)
        ref = oracle.round_bf16(ref)
        got = cpu(o_gpu[0, hq][torch.from_numpy(rows).to(o_gpu.device)]).double().numpy()
        err = np.abs(got - ref)
        assert np.all(np.isfinite(got)), hq
        assert err.max() <= O_MAX_ABS, (hq, mode, float(err.max()), rows[np.unravel_index(err.argmax(), err.shape)[0]])
        assert err.mean() <= O_MEAN_ABS, (hq, mode, float(err.mean()))
        worst = max(worst, float(err.max()))
    return worst
