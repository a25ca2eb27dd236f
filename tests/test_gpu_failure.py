"""Failure detection on the GPU without faulting it: a wait that can never
complete gives up after its limit, reports RTP_ERR_TIMEOUT through the
device status word, and the context stays usable for the next call."""

import time

import numpy as np
import pytest
import torch

import oracle
from swa_hybrid_attention_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rtp(cuda_device):
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def test_bounded_wait_times_out_and_context_survives(rtp, cuda_device):
    t0 = time.perf_counter()
    st = rtp.rtp_selftest_bounded_wait(200)
    dt = time.perf_counter() - t0
    assert st == rtp.RTP_ERR_TIMEOUT, rtp.status_str(st)
    assert 0.19 <= dt < 5.0, dt
    # the status word was read and cleared; the next call is clean
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    # and the context still runs the attention path correctly
    d = inputs.small_prefill(256, 2, 1, [oracle.FULL], seed=3)
    o, _ = rtp.hybrid_prefill_layer(d["q"].to(cuda_device), d["k"].to(cuda_device), d["v"].to(cuda_device),
                                    d["kinds"], window=64)
    torch.cuda.synchronize()
    assert rtp.rtp_last_device_status() == rtp.RTP_OK
    ref = oracle.attention_rows(d["q"][0, 0], np.arange(256), d["k"][0, 0], d["v"][0, 0], oracle.FULL)
    got = o[0, 0].double().cpu().numpy()
    assert np.max(np.abs(got - oracle.round_bf16(ref))) <= 2e-2


def test_selftest_rejects_bad_limit(rtp, cuda_device):
    assert rtp.rtp_selftest_bounded_wait(0) == rtp.RTP_ERR_INVALID_ARG
    assert rtp.rtp_selftest_bounded_wait(20000) == rtp.RTP_ERR_INVALID_ARG
