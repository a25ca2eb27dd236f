"""The allocation-free decode entry point, checked against the regular one.

rtp_sparse_decode_noalloc exists for callers that must not allocate device
memory while they run: latency-critical serving loops that cannot afford the
device-wide synchronisation cudaMalloc implies, and hosts whose device memory
is owned by another runtime's pool.  It keeps its split-K scratch in a fixed
array inside the library instead of a caller-supplied workspace.

This file is collected last on purpose (test_zz_*), so that a failure here
is reported only after every other test has run.  It passes both on its own
in a fresh process and after the rest of the suite: the first call on a
device performs the one-time address lookup of the array.
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import O_MAX_ABS, O_MEAN_ABS
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu

KINDS = [2, 2, 0, 2]
WINDOW, BLOCK, TOPK, N_LOCAL = 1024, 128, 6, 2


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def make_case(seed, device):
    w = inputs.Workload(40 + seed, "noalloc", 2, 1, 16, 4, 1, WINDOW, BLOCK, TOPK, N_LOCAL, "lowfreq", 0, [KINDS],
                        cache_len=4096, decode=True)
    d = inputs.decode_step(w, "cpu")
    C = torch.zeros(2, 4, 4096 // BLOCK, 16)
    for b in range(2):
        for h, kind in enumerate(KINDS):
            if kind == 2:
                C[b, h] = torch.from_numpy(oracle.centroids(d["kcache"][b, h], BLOCK, d["proj"]).astype(np.float32))
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in d.items()} | {"C": C.to(device)}


def test_noalloc_matches_workspace_path_on_two_calls(rtp, cuda_device):
    cfg = rtp.AttnConfig(2, 1, 16, 4, WINDOW, BLOCK, TOPK, N_LOCAL)
    cases = [make_case(s, cuda_device) for s in (1, 2)]
    results = []
    for d in cases:  # two calls in a row, different inputs
        o = torch.empty_like(d["q"])
        sel = torch.full((2, 4, cfg.kmax), -1, dtype=torch.int32, device=cuda_device)
        cnt = torch.zeros(2, 4, dtype=torch.int32, device=cuda_device)
        rtp.rtp_sparse_decode_noalloc(cfg, KINDS, 4096, d["q"], d["kcache"], d["vcache"], d["C"], d["proj"], o,
                                      sel, cnt)
        results.append((o, sel, cnt))
    torch.cuda.synchronize()
    for d, (o, sel, cnt) in zip(cases, results):
        ref_o, ref_sel, ref_cnt = rtp.sparse_decode_step(d["q"], d["kcache"], d["vcache"], d["C"], d["proj"], KINDS,
                                                         window=WINDOW, block=BLOCK, topk=TOPK, n_local=N_LOCAL,
                                                         return_selection=True)
        torch.cuda.synchronize()
        err = (o.double() - ref_o.double()).abs()
        assert float(err.max()) <= O_MAX_ABS and float(err.mean()) <= O_MEAN_ABS
        for b in range(2):
            for h, kind in enumerate(KINDS):
                if kind == 2:
                    n = int(cnt[b, h])
                    assert n == int(ref_cnt[b, h])
                    assert torch.equal(sel[b, h, :n], ref_sel[b, h, :n])
    assert rtp.rtp_last_device_status() == rtp.RTP_OK


def test_noalloc_calls_and_status_read_change_no_free_memory(rtp, cuda_device):
    """Once the first call on the device has looked up the array's address,
    further calls, and reading the status words back, leave the device's free
    memory exactly as it was: nothing is allocated or freed."""
    cfg = rtp.AttnConfig(2, 1, 16, 4, WINDOW, BLOCK, TOPK, N_LOCAL)
    d = make_case(5, cuda_device)
    o = torch.empty_like(d["q"])

    def call():
        rtp.rtp_sparse_decode_noalloc(cfg, KINDS, 4096, d["q"], d["kcache"], d["vcache"], d["C"], d["proj"], o)

    call()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        call()
    status = rtp.rtp_last_device_status()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert status == rtp.RTP_OK


def test_noalloc_rejects_shapes_beyond_its_scratch(rtp, cuda_device):
    # 64 sequences x 4 heads x 64 splits x 8 heads of partials is ~35 MB > 16 MiB
    cfg = rtp.AttnConfig(64, 1, 32, 4, 8192, 128, 32, 4)
    assert rtp.rtp_decode_workspace_bytes(cfg, KINDS, 262144) > 16 << 20
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_sparse_decode_noalloc(cfg, KINDS, 262144, 16, 16, 16, 16, 16, 16)
    assert e.value.status == rtp.RTP_ERR_INVALID_ARG
