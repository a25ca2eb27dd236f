"""The seeded synthetic workloads are the ones the design states.

Five workloads stand in for the configurations the method is evaluated on:
a tiny 2K V2 layer; the 48-layer 32K V1 model and 128K V2 model (29 of the
192 (layer, KV head) slots retrieval heads, chosen by randperm(192, seed 0),
the rest streaming heads with an 8192-token window); one 1M-token V2 layer
(KV head 0 retrieval, three streaming heads); and an 8-sequence decode step
over 256K-token caches (3 of 4 KV heads retrieval, randperm(4, seed 0)).
Generation is seeded and reproducible, and V is not rotated.
"""

import torch

from swa_hybrid_attention_b200 import inputs

SWA, FULL, SPARSE = inputs.SWA, inputs.FULL, inputs.SPARSE


def slots(w, kind):
    return [(layer, h) for layer in range(w.layers) for h in range(w.n_kv_heads) if w.kinds[layer][h] == kind]


def test_model_workloads_route_29_of_192_slots_to_retrieval_heads():
    w1, w2 = inputs.workload(1), inputs.workload(2)
    for w, kind, seq in ((w1, FULL, 32768), (w2, SPARSE, 131072)):
        assert (w.layers, w.n_q_heads, w.n_kv_heads, w.seq, w.window, w.block) == (48, 32, 4, seq, 8192, 128)
        assert len(slots(w, kind)) == 29
        assert len(slots(w, SWA)) == 192 - 29
    assert slots(w1, FULL) == slots(w2, SPARSE)  # the same routing map for V1 and V2
    perm = torch.randperm(192, generator=torch.Generator().manual_seed(0))[:29].tolist()
    assert sorted(slots(w1, FULL)) == sorted((s // 4, s % 4) for s in perm)
    assert (w2.topk, w2.n_local, w2.projector, w2.needles) == (64, 4, "random", 256)


def test_million_token_layer_and_decode_workloads():
    w3 = inputs.workload(3)
    assert (w3.seq, w3.layers, w3.kinds, w3.block, w3.topk, w3.n_local) == \
        (1 << 20, 1, [[SPARSE, SWA, SWA, SWA]], 128, 128, 8)
    assert (w3.projector, w3.needles, w3.window, w3.group) == ("lowfreq", 1024, 8192, 8)
    w4 = inputs.workload(4)
    assert (w4.batch, w4.cache_len, w4.block, w4.topk, w4.n_local, w4.window) == (8, 262144, 128, 32, 4, 8192)
    assert sorted(w4.kinds[0]) == [SWA, SPARSE, SPARSE, SPARSE]
    perm = torch.randperm(4, generator=torch.Generator().manual_seed(0))[:3].tolist()
    assert [h for h in range(4) if w4.kinds[0][h] == SPARSE] == sorted(perm)
    w0 = inputs.workload(0)
    assert (w0.seq, w0.n_q_heads, w0.n_kv_heads, w0.kinds, w0.block, w0.topk, w0.n_local, w0.window) == \
        (2048, 8, 2, [[SPARSE, SWA]], 64, 16, 2, 512)


def test_low_frequency_projector_keeps_the_eight_slowest_rotary_pairs():
    p = inputs.lowfreq_projector()
    rows, cols = torch.nonzero(p, as_tuple=True)
    assert rows.tolist() == list(range(56, 64)) + list(range(120, 128))
    assert cols.tolist() == list(range(16)) and bool((p[rows, cols] == 1.0).all())


def test_generation_is_seeded_and_values_are_not_rotated():
    a = inputs.small_prefill(256, 4, 2, [SPARSE, SWA], seed=9)
    b = inputs.small_prefill(256, 4, 2, [SPARSE, SWA], seed=9)
    c = inputs.small_prefill(256, 4, 2, [SPARSE, SWA], seed=10)
    for t in ("q", "k", "v"):
        assert torch.equal(a[t], b[t]) and not torch.equal(a[t], c[t])
        assert a[t].dtype == torch.bfloat16
    plain = inputs.small_prefill(256, 4, 2, [SPARSE, SWA], seed=9, rotate=False)
    assert torch.equal(plain["v"], a["v"])  # V is never rotated
    assert not torch.equal(plain["k"], a["k"]) and torch.equal(plain["k"][:, :, 0], a["k"][:, :, 0])  # position 0


def test_rotary_encoding_rotates_pairs_i_and_i_plus_64():
    """Rotate-half pairs (i, i + 64) turned by position * 1e6^(-2i/128): as
    complex numbers x_i + 1j x_(i+64) multiplied by exp(1j * angle); the
    rotation keeps each pair's norm, and the scores q.k of two rotated rows
    depend only on the difference of their positions."""
    torch.manual_seed(0)
    n = 300
    x = torch.randn(n, 128, dtype=torch.float64)
    cos, sin = inputs.rope_tables(n, "cpu")
    y = inputs.apply_rope_fp32(x.float(), cos, sin).double()
    i = torch.arange(64, dtype=torch.float64)
    ang = torch.arange(n, dtype=torch.float64)[:, None] * 1e6 ** (-2.0 * i / 128)[None, :]
    z = torch.complex(x[:, :64], x[:, 64:]) * torch.exp(1j * ang)
    assert torch.allclose(y[:, :64], z.real, atol=1e-5) and torch.allclose(y[:, 64:], z.imag, atol=1e-5)
    assert torch.allclose(y[:, :64] ** 2 + y[:, 64:] ** 2, x[:, :64] ** 2 + x[:, 64:] ** 2, rtol=1e-5, atol=1e-5)
    q, k = torch.randn(128, dtype=torch.float64), torch.randn(128, dtype=torch.float64)
    qs = inputs.apply_rope_fp32(q.float().expand(n, 128), cos, sin).double()
    ks = inputs.apply_rope_fp32(k.float().expand(n, 128), cos, sin).double()
    s1 = (qs[200] * ks[150]).sum()  # offset 50
    s2 = (qs[80] * ks[30]).sum()
    assert abs(float(s1 - s2)) <= 1e-4
