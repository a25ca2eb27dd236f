"""Seeded synthetic workloads for the headwise hybrid attention path.

This module only *makes data*: Q/K/V with rotary position encoding already
applied, the low-rank projector, planted "needle" keys and the per-(layer,
KV-head) routing map.  It holds none of the attention arithmetic, so both the
CUDA library and the CPU oracle can be fed from it without sharing any of
the method's code.

Workloads (sizes follow the configurations the method is evaluated on):

  0  tiny V2 layer: seq 2048, 8 q / 2 kv heads, kv0 retrieval (block 64,
     top-k 16, 1 sink, 2 local, low-frequency projector), kv1 SWA window 512.
  1  Qwen3-30B-A3B-shaped V1 prefill: 48 layers x (32 q / 4 kv), seq 32768,
     29 of 192 (layer, kv) slots full attention, the rest SWA window 8192.
  2  same map at seq 131072 in V2 mode: retrieval heads use a random
     N(0, 1/128) projector, block 128, top-k 64 + sink + 4 local, 256 needles.
  3  one 1M-token V2 layer: kv0 retrieval (low-frequency projector, block 128,
     top-k 128 + sink + 8 local, 1024 needles), kv1-3 SWA window 8192.
  4  decode step: 8 sequences x 262144-token cache (4 kv / 32 q heads),
     3 of 4 kv heads retrieval (block 128, top-k 32 + sink + 4 local), the
     other SWA window 8192.

Head kinds: 0 = SWA (streaming head), 1 = full causal (V1 retrieval head),
2 = block-sparse (V2 retrieval head).

Rotary encoding ("RoPE"): theta_i = base^(-2i/D), base 1e6, rotate-half
pairing of dims (i, i+D/2), position = token index.  Pre-rotation values are
N(0,1) fp32; rotation is done in fp32 and the result is rounded once to bf16.
The low-frequency projector keeps the 8 slowest rotary pairs
(dims 56..63 and 120..127), the pages' reason being that retrieval heads live
on the low-frequency rotary components.

Seeds: tensor t of layer l in workload w draws from a generator seeded with
1000*w + 10*l + t (t: Q=0, K=1, V=2, projector=3, needles=4).  Large tensors
are generated one head at a time on the target device.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SWA, FULL, SPARSE = 0, 1, 2
HEAD_DIM = 128
RANK = 16
ROPE_BASE = 1.0e6


@dataclass
class Workload:
    wid: int
    name: str
    batch: int
    seq: int
    n_q_heads: int
    n_kv_heads: int
    layers: int
    window: int
    block: int
    topk: int
    n_local: int
    projector: str  # "lowfreq" or "random"
    needles: int = 0
    kinds: list = field(default_factory=list)  # [layers][n_kv_heads]
    cache_len: int = 0  # decode only
    decode: bool = False

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def kmax(self) -> int:
        return self.topk + 1 + self.n_local


def _randperm(n: int, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randperm(n, generator=g)


def _layered_map(layers: int, hkv: int, n_retrieval: int, retrieval_kind: int) -> list:
    slots = _randperm(layers * hkv, 0)[:n_retrieval].tolist()
    kinds = [[SWA] * hkv for _ in range(layers)]
    for s in slots:
        kinds[s // hkv][s % hkv] = retrieval_kind
    return kinds


def workload(wid: int) -> Workload:
    """The five seeded workloads (see module docstring)."""
    if wid == 0:
        return Workload(0, "tiny-v2-2k", 1, 2048, 8, 2, 1, 512, 64, 16, 2, "lowfreq", 0, [[SPARSE, SWA]])
    if wid == 1:
        return Workload(1, "qwen3-30b-a3b-v1-32k", 1, 32768, 32, 4, 48, 8192, 128, 0, 1, "none", 0,
                        _layered_map(48, 4, 29, FULL))
    if wid == 2:
        return Workload(2, "qwen3-30b-a3b-v2-128k", 1, 131072, 32, 4, 48, 8192, 128, 64, 4, "random", 256,
                        _layered_map(48, 4, 29, SPARSE))
    if wid == 3:
        return Workload(3, "v2-1m-layer", 1, 1048576, 32, 4, 1, 8192, 128, 128, 8, "lowfreq", 1024,
                        [[SPARSE, SWA, SWA, SWA]])
    if wid == 4:
        perm = _randperm(4, 0)[:3].tolist()
        kinds = [SPARSE if h in perm else SWA for h in range(4)]
        return Workload(4, "decode-8x256k", 8, 1, 32, 4, 1, 8192, 128, 32, 4, "lowfreq", 0, [kinds],
                        cache_len=262144, decode=True)
    raise ValueError(f"unknown workload {wid}")


def seed_of(wid: int, layer: int, tensor_id: int) -> int:
    return 1000 * wid + 10 * layer + tensor_id


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def rope_tables(n: int, device, d: int = HEAD_DIM, base: float = ROPE_BASE, start: int = 0):
    """cos/sin tables [n, d/2] in fp32 (angles formed in fp64)."""
    half = d // 2
    inv = base ** (-2.0 * torch.arange(half, dtype=torch.float64, device=device) / d)
    pos = torch.arange(start, start + n, dtype=torch.float64, device=device)
    ang = pos[:, None] * inv[None, :]
    return torch.cos(ang).float(), torch.sin(ang).float()


def apply_rope_fp32(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """Rotate-half rotary encoding of x [n, d] fp32."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def _rotary_heads(n_heads: int, n: int, seed: int, device, rotate: bool, cos=None, sin=None) -> torch.Tensor:
    """[n_heads, n, 128] bf16: N(0,1) fp32 draws, optionally rotated, rounded once."""
    g = _gen(seed, device)
    out = torch.empty(n_heads, n, HEAD_DIM, dtype=torch.bfloat16, device=device)
    for h in range(n_heads):
        x = torch.randn(n, HEAD_DIM, generator=g, device=device, dtype=torch.float32)
        if rotate:
            x = apply_rope_fp32(x, cos, sin)
        out[h] = x.to(torch.bfloat16)
    return out


def lowfreq_projector(device="cpu") -> torch.Tensor:
    """[128, 16] fp32 selecting dims 56..63 and 120..127 (the 8 slowest rotary pairs)."""
    p = torch.zeros(HEAD_DIM, RANK, dtype=torch.float32, device=device)
    dims = list(range(56, 64)) + list(range(120, 128))
    for c, d in enumerate(dims):
        p[d, c] = 1.0
    return p


def random_projector(seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, "cpu")
    p = torch.randn(HEAD_DIM, RANK, generator=g, dtype=torch.float32) / math.sqrt(HEAD_DIM)
    return p.to(device)


def projector_for(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    if w.projector == "random":
        return random_projector(seed_of(w.wid, layer, 3), device)
    return lowfreq_projector(device)


def plant_needles(w: Workload, layer: int, q: torch.Tensor, k: torch.Tensor, kinds: list) -> list:
    """Overwrite needle keys in every retrieval head of one layer, in place.

    For each needle: a target query position tq uniform in [(L+2)B, N), a
    query head of the group, and a key position j uniform in
    [B, B*(tq//B - L)) (outside the sink and local blocks of tq's block);
    k[j] := 4 * q[h, tq] / ||q[h, tq]|| (fp32, rounded to bf16).  Later
    needles overwrite earlier ones.  Returns (kv_head, q_head, tq, j) tuples.
    """
    if w.needles == 0:
        return []
    g = _gen(seed_of(w.wid, layer, 4), "cpu")
    B, L, N, G = w.block, w.n_local, w.seq, w.group
    planted = []
    for kvh, kind in enumerate(kinds):
        if kind != SPARSE:
            continue
        lo = (L + 2) * B
        tq = torch.randint(lo, N, (w.needles,), generator=g)
        hh = torch.randint(0, G, (w.needles,), generator=g)
        u = torch.rand(w.needles, generator=g, dtype=torch.float64)
        for n in range(w.needles):
            t = int(tq[n])
            hi = B * (t // B - L)
            j = B + int(u[n].item() * (hi - B))
            j = min(max(j, B), hi - 1)
            qh = kvh * G + int(hh[n])
            qv = q[0, qh, t].float()
            k[0, kvh, j] = (4.0 * qv / qv.norm()).to(torch.bfloat16)
            planted.append((kvh, qh, t, j))
    return planted


def prefill_layer(w: Workload, layer: int, device) -> dict:
    """Q, K, V [1, H, N, 128] bf16 (rotated Q/K), projector, kinds, needles."""
    assert not w.decode
    cos, sin = rope_tables(w.seq, device)
    q = _rotary_heads(w.n_q_heads, w.seq, seed_of(w.wid, layer, 0), device, True, cos, sin).unsqueeze(0)
    k = _rotary_heads(w.n_kv_heads, w.seq, seed_of(w.wid, layer, 1), device, True, cos, sin).unsqueeze(0)
    v = _rotary_heads(w.n_kv_heads, w.seq, seed_of(w.wid, layer, 2), device, False).unsqueeze(0)
    del cos, sin
    kinds = list(w.kinds[layer])
    needles = plant_needles(w, layer, q, k, kinds)
    return dict(q=q, k=k, v=v, proj=projector_for(w, layer, device), kinds=kinds, needles=needles)


def small_prefill(seq: int, hq: int, hkv: int, kinds: list, seed: int, device="cpu", rotate: bool = True) -> dict:
    """An arbitrary small seeded layer (test shapes: ragged tails, edge cases)."""
    cos, sin = rope_tables(seq, device)
    q = _rotary_heads(hq, seq, seed, device, rotate, cos, sin).unsqueeze(0)
    k = _rotary_heads(hkv, seq, seed + 1, device, rotate, cos, sin).unsqueeze(0)
    v = _rotary_heads(hkv, seq, seed + 2, device, False).unsqueeze(0)
    return dict(q=q, k=k, v=v, proj=lowfreq_projector(device), kinds=list(kinds), needles=[])


def decode_step(w: Workload, device, cache_len: int | None = None, batch: int | None = None) -> dict:
    """q [Bt, Hq, 1, 128], K/V caches [Bt, Hkv, Lc, 128] bf16 (rotated q/k).

    The new token is the last cache entry (position Lc-1), so q is rotated
    at that position.
    """
    assert w.decode
    Lc = cache_len or w.cache_len
    Bt = batch or w.batch
    cos, sin = rope_tables(Lc, device)
    kc = torch.empty(Bt, w.n_kv_heads, Lc, HEAD_DIM, dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    q = torch.empty(Bt, w.n_q_heads, 1, HEAD_DIM, dtype=torch.bfloat16, device=device)
    for b in range(Bt):
        kc[b] = _rotary_heads(w.n_kv_heads, Lc, seed_of(w.wid, b, 1), device, True, cos, sin)
        vc[b] = _rotary_heads(w.n_kv_heads, Lc, seed_of(w.wid, b, 2), device, False)
        g = _gen(seed_of(w.wid, b, 0), device)
        x = torch.randn(w.n_q_heads, HEAD_DIM, generator=g, device=device, dtype=torch.float32)
        q[b, :, 0] = apply_rope_fp32(x, cos[Lc - 1:Lc], sin[Lc - 1:Lc]).to(torch.bfloat16)
    return dict(q=q, kcache=kc, vcache=vc, proj=projector_for(w, 0, device), kinds=list(w.kinds[0]),
                cache_len=Lc)
