"""Seeded k-means inputs shared by the tensor-core / exact-path comparison
(tests/test_gpu_kmeans.py runs them in this process and, with
RTP_KMEANS_EXACT_ASSIGN=1, in a child process through `python
kmeans_cases.py <out>`)."""

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# (name, batch, heads, kinds, cache capacity, clu_end, block, n_clusters, iters, seed, kind of keys)
CASES = [
    ("nc24", 2, 3, [2, 0, 2], 4096, 2944, 128, 24, 4, 11, "randn"),
    ("nc100-block64", 1, 2, [2, 2], 4096, 3008, 64, 100, 3, 12, "randn"),
    ("nc1", 1, 1, [2], 1024, 896, 128, 1, 2, 13, "randn"),
    ("nc2048", 1, 1, [2], 8320, 8192, 128, 2048, 3, 14, "randn"),
    ("ties", 1, 1, [2], 4224, 4096, 128, 2048, 3, 15, "dup"),      # every key twice, seeds on both copies:
                                                                    # equal centroids, exact distance ties
    ("huge", 1, 1, [2], 2176, 2048, 128, 32, 2, 16, "huge"),       # beyond fp16's safe range
]


def make_cache(B, H, cap, seed, kind, device):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, H, cap, 128, generator=g)
    if kind == "dup":
        k[:, :, 1::2] = k[:, :, 0::2]
    if kind == "huge":
        k = k * 3.0e4
    v = torch.randn(B, H, cap, 128, generator=g)
    return k.to(torch.bfloat16).to(device), v.to(torch.bfloat16).to(device)


def run_all(rtp, device):
    from swa_hybrid_attention_b200 import inputs

    out = {}
    for name, B, H, kinds, cap, clu_end, block, nc, iters, seed, kind in CASES:
        k, v = make_cache(B, H, cap, seed, kind, device)
        proj = inputs.random_projector(5, device)
        cl = rtp.cluster_cache(k, v, proj, kinds, clu_end=clu_end, n_clusters=nc, iters=iters, block=block)
        torch.cuda.synchronize()
        out[name] = {f: getattr(cl, f).cpu() for f in ("centroids", "members", "offsets", "n_chunks", "chunk_start",
                                                      "chunk_len", "chunk_centroids")}
        out[name]["status"] = int(rtp.rtp_last_device_status())
    return out


def run_full(rtp, device):
    """The decode workload's whole cache (8 sequences x 262,144 rows, 3 of 4
    heads clustered), 2048 clusters, 8 rounds: the bench's clustering."""
    from swa_hybrid_attention_b200 import inputs

    w = inputs.workload(4)
    d = inputs.decode_step(w, device)
    Lc = d["cache_len"]
    clu_end = (Lc // w.block - w.n_local) * w.block
    cl = rtp.cluster_cache(d["kcache"], d["vcache"], d["proj"], d["kinds"], clu_end=clu_end, n_clusters=2048,
                           iters=8, block=w.block, in_place=True)
    torch.cuda.synchronize()
    out = {f: getattr(cl, f).cpu() for f in ("centroids", "members", "offsets", "n_chunks", "chunk_start",
                                             "chunk_len", "chunk_centroids")}
    out["status"] = int(rtp.rtp_last_device_status())
    return {"full": out}


if __name__ == "__main__":
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    run = run_full if "--full" in sys.argv[2:] else run_all
    torch.save(run(mod, torch.device("cuda:0")), sys.argv[1])
