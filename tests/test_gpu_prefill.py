"""GPU parity of the prefill path (indexer, selection, hybrid attention)
against the CPU oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
from helpers import check_indexer, check_prefill_rows, check_selection_rows, cpu
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def run_layer(rtp, d, window, block, topk, n_local, device, scale=0.0):
    q, k, v = d["q"].to(device), d["k"].to(device), d["v"].to(device)
    proj = d["proj"].to(device)
    cfg = rtp.AttnConfig(q.shape[0], q.shape[2], q.shape[1], k.shape[1], window, block, topk, n_local, scale)
    plan = rtp.Plan(cfg, d["kinds"])
    bufs = plan.buffers(device)
    o = torch.full_like(q, float("nan"))
    plan.run(q, k, v, proj, o, bufs)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    return q, k, v, proj, o, bufs, plan


def full_check(rtp, d, window, block, topk, n_local, device, scale=0.0):
    q, k, v, proj, o, bufs, plan = run_layer(rtp, d, window, block, topk, n_local, device, scale)
    group = q.shape[1] // k.shape[1]
    n = q.shape[2]
    nb = n // block
    slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
    if plan.n_sparse:
        C, Qb = check_indexer(bufs["centroids"], bufs["qbar"], q, k, proj, plan.slot_heads, block, group)
        for s in range(plan.n_sparse):
            check_selection_rows(cpu(bufs["sel"][0, s]).numpy(), cpu(bufs["sel_cnt"][0, s]).numpy(), Qb[s], C[s],
                                 np.arange(nb), topk, n_local)
    check_prefill_rows(o, q, k, v, d["kinds"], group, window, block, bufs["sel"], bufs["sel_cnt"], slot_of,
                       lambda hq: np.arange(n), None if scale == 0.0 else scale)
    plan.close()
    return o


def test_tiny_v2_layer(rtp, cuda_device):
    w = inputs.workload(0)
    d = inputs.prefill_layer(w, 0, "cpu")
    full_check(rtp, d, w.window, w.block, w.topk, w.n_local, cuda_device)


EDGE_CASES = [
    # seq, hq, hkv, kinds, window, block, topk, n_local
    (64, 2, 1, [2], 64, 64, 2, 1),              # one block of 64: half a query tile, sink only
    (64, 4, 2, [0, 1], 16, 64, 1, 1),           # one block of 64, SWA and full
    (128, 2, 1, [1], 64, 128, 2, 1),            # one tile, full
    (128, 2, 1, [0], 1, 128, 2, 1),             # window 1: each row sees itself
    (192, 2, 1, [2], 64, 64, 1, 1),             # ragged last 128-row tile, block 64
    (640, 4, 2, [0, 1], 100, 64, 2, 2),         # SWA window not a tile multiple
    (640, 4, 2, [0, 1], 128, 128, 2, 2),        # window = one tile
    (640, 4, 2, [0, 1], 129, 128, 2, 2),        # window = tile + 1
    (640, 4, 2, [0, 2], 5000, 128, 1, 1),       # window > seq (SWA == full)
    (1024, 16, 2, [2, 0], 256, 128, 2, 1),      # group 8, sparse block 128
    (1024, 4, 2, [2, 2], 256, 64, 3, 2),        # two sparse slots, block 64
    (1024, 4, 1, [2], 256, 128, 0, 1),          # top-k 0: sink + diagonal only
    (1024, 4, 1, [2], 256, 128, 64, 1),         # top-k >= blocks: full causal
    (1984, 8, 2, [2, 0], 300, 64, 5, 2),        # 31 blocks of 64: ragged tile
]


@pytest.mark.parametrize("case", EDGE_CASES, ids=[f"n{c[0]}-h{c[1]}x{c[2]}-k{''.join(map(str, c[3]))}-w{c[4]}-b{c[5]}"
                                                  for c in EDGE_CASES])
def test_edge_shapes(rtp, cuda_device, case):
    seq, hq, hkv, kinds, window, block, topk, n_local = case
    d = inputs.small_prefill(seq, hq, hkv, kinds, seed=100 + seq + hq)
    full_check(rtp, d, window, block, topk, n_local, cuda_device)


def test_batch_two_and_scale(rtp, cuda_device):
    d0 = inputs.small_prefill(512, 4, 2, [2, 0], seed=5)
    d1 = inputs.small_prefill(512, 4, 2, [2, 0], seed=6)
    d = dict(q=torch.cat([d0["q"], d1["q"]]), k=torch.cat([d0["k"], d1["k"]]), v=torch.cat([d0["v"], d1["v"]]),
             proj=d0["proj"], kinds=[2, 0])
    q, k, v, proj, o, bufs, plan = run_layer(rtp, d, 200, 64, 2, 2, cuda_device, scale=0.05)
    for b in range(2):
        db = d0 if b == 0 else d1
        sub = dict(centroids=bufs["centroids"][b:b + 1], sel=bufs["sel"][b:b + 1], sel_cnt=bufs["sel_cnt"][b:b + 1])
        check_prefill_rows(o[b:b + 1], db["q"], db["k"], db["v"], [2, 0], 2, 200, 64, sub["sel"], sub["sel_cnt"],
                           {0: 0}, lambda hq: np.arange(512), 0.05)
    plan.close()


@pytest.mark.parametrize("scale", [0.5, 2.0])
def test_growing_maximum(rtp, cuda_device, scale):
    """Key norms ramp up along the sequence and the softmax scale is large, so
    a row's maximum keeps growing, also between the two 64-key halves of a
    tile: every reference move, O rescale and recomputed chunk of P is taken,
    including the one that waits for the tile's first half to pass its P V."""
    n = 1024
    d = inputs.small_prefill(n, 6, 3, [2, 0, 1], seed=9)
    ramp = torch.linspace(0.25, 2.0, n).view(1, 1, n, 1)
    d["k"] = (d["k"].float() * ramp).to(torch.bfloat16)
    full_check(rtp, d, 300, 128, 2, 1, cuda_device, scale=scale)


def test_deterministic(rtp, cuda_device):
    w = inputs.workload(0)
    d = inputs.prefill_layer(w, 0, "cpu")
    outs = []
    for _ in range(2):
        q, k, v, proj, o, bufs, plan = run_layer(rtp, d, w.window, w.block, w.topk, w.n_local, cuda_device)
        outs.append((o.clone(), bufs["sel"].clone(), bufs["centroids"].clone()))
        plan.close()
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


def kind_blocks(nb, topk, n_local, rng, n_random=64):
    """Query blocks checked at full size for one head kind: 0, 1, k+L, k+L+1,
    the last, and n_random more drawn without replacement."""
    fixed = [min(nb - 1, b) for b in (0, 1, topk + n_local, topk + n_local + 1, nb - 1)]
    rand = rng.choice(nb, size=min(n_random, nb), replace=False).tolist()
    return sorted(set(fixed) | set(int(b) for b in rand))


def sampled_check(rtp, w, layer, device, check_o=True):
    """A full-size layer through the library, against the oracle:
      * centroids and query summaries of every retrieval slot, in full;
      * the selection of every query block, in full;
      * O: per head kind present in the layer, every row of the query blocks
        {0, 1, k+L, k+L+1, last} and 64 random ones, for all G query heads of
        every KV head of that kind, plus every needle's target row."""
    d = inputs.prefill_layer(w, layer, device)
    q, k, v, proj, o, bufs, plan = run_layer(rtp, d, w.window, w.block, w.topk, w.n_local, device)
    G, n, B = w.group, w.seq, w.block
    nb = n // B
    rng = np.random.default_rng(1000 * w.wid + layer + 17)
    slot_of = {h: s for s, h in enumerate(plan.slot_heads)}
    if plan.n_sparse:
        C, Qb = check_indexer(bufs["centroids"], bufs["qbar"], q, k, proj, plan.slot_heads, B, G)
        for s, kvh in enumerate(plan.slot_heads):
            sel = cpu(bufs["sel"][0, s]).numpy()
            cnt = cpu(bufs["sel_cnt"][0, s]).numpy()
            near = check_selection_rows(sel, cnt, Qb[s], C[s], np.arange(nb), w.topk, w.n_local)
            hits = sum(1 for (h, qh, tq, j) in d["needles"] if h == kvh and (j // B) in set(sel[tq // B][:cnt[tq // B]]))
            tot = sum(1 for x in d["needles"] if x[0] == kvh)
            print(f"layer {layer} slot {s}: {near} near-tie rows of {nb}; needle recall {hits}/{tot}")
    if check_o:
        blocks_of_kind = {kind: kind_blocks(nb, w.topk, w.n_local, rng) for kind in set(d["kinds"])}
        needle_rows = {}
        for (_, qh, tq, _) in d["needles"]:
            needle_rows.setdefault(qh, set()).add(int(tq))

        def rows_of_head(hq):
            blocks = blocks_of_kind[d["kinds"][hq // G]]
            rows = set((np.asarray(blocks)[:, None] * B + np.arange(B)[None, :]).reshape(-1).tolist())
            return np.array(sorted(rows | needle_rows.get(hq, set())), dtype=np.int64)

        worst = check_prefill_rows(o, q, k, v, d["kinds"], G, w.window, B, bufs["sel"], bufs["sel_cnt"], slot_of,
                                   rows_of_head)
        print(f"layer {layer}: O max |err| {worst:.3e} on {sum(rows_of_head(h).size for h in range(q.shape[1]))} rows")
    plan.close()


@pytest.mark.slow
def test_full_size_1m_v2_layer(rtp, cuda_device):
    sampled_check(rtp, inputs.workload(3), 0, cuda_device)


@pytest.mark.slow
def test_full_size_128k_v2_every_layer(rtp, cuda_device):
    """Every layer of the 48-layer 128K V2 model with a retrieval head:
    indexer and selection in full; O rows on the first, a middle and the last
    such layer."""
    w = inputs.workload(2)
    layers = [l for l in range(w.layers) if 2 in w.kinds[l]]
    o_layers = {layers[0], layers[len(layers) // 2], layers[-1]}
    for layer in layers:
        sampled_check(rtp, w, layer, cuda_device, check_o=layer in o_layers)
        torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_size_32k_v1_layers(rtp, cuda_device):
    """The 48-layer 32K V1 model (no indexer): O rows on three layers with a
    full-attention head and on one with streaming heads only, if any."""
    w = inputs.workload(1)
    full = [l for l in range(w.layers) if 1 in w.kinds[l]]
    layers = {full[0], full[len(full) // 2], full[-1]}
    swa_only = [l for l in range(w.layers) if 1 not in w.kinds[l]]
    if swa_only:
        layers.add(swa_only[0])
    for layer in sorted(layers):
        sampled_check(rtp, w, layer, cuda_device)
        torch.cuda.empty_cache()
