"""Failure detection of the tensor-core kernel: every mbarrier wait is bounded.

A test-only hook (SOL_ATTN_TEST_STALL) makes the first S of every CTA go
unsignalled, so the waits on it cannot complete.  With a short limit
(SOL_ATTN_WAIT_LIMIT_NS) they run out, the kernel takes its abort path (waits
for its own copies and MMAs, frees tensor memory, records the wait id) and
sol_attn_device_status reports SOL_ERR_DEVICE_TIMEOUT.  Nothing faults, traps
or hangs: the same context then computes the same output as before."""

import pytest
import torch

from video_diffusion_b200 import api, build
from video_diffusion_b200 import inputs as I

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_stays_usable(cuda_device, monkeypatch):
    build.build()
    api.lib()
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=21, device="cuda")  # 16 query blocks
    ref = api.forward(Q, K, V, 1.04)
    assert api.device_status() == 0

    monkeypatch.setenv("SOL_ATTN_WAIT_LIMIT_NS", "20000000")  # 20 ms
    monkeypatch.setenv("SOL_ATTN_TEST_STALL", "1")
    api.forward(Q, K, V, 1.04)  # enqueued normally; the kernel gives up inside
    word = api.device_status()
    assert word & 0x1000, hex(word)  # a wait of the attention kernel expired
    assert api.status_string(api.lib().sol_attn_device_status(None, None)) == "SOL_OK"  # the word was cleared

    monkeypatch.delenv("SOL_ATTN_TEST_STALL")
    monkeypatch.delenv("SOL_ATTN_WAIT_LIMIT_NS")
    again = api.forward(Q, K, V, 1.04)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(again, ref)
