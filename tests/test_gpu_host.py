"""sol_attn_forward_host: the forward with q, k, v and out in host memory.

The call pipelines groups of (batch, head) slices through device staging
buffers, so its output must equal, bit for bit, that of sol_attn_forward(_ex)
on device copies of the same tensors, for every grouping (one slice per
group, a ragged last group, one group for everything, more slices per group
than there are), both dtypes and every flag, with page-locked or pageable
host memory."""

import pytest
import torch

from video_diffusion_b200 import api
from video_diffusion_b200 import inputs as I


def _host(t, pinned):
    h = t.cpu()
    return h.pin_memory() if pinned else h


@pytest.mark.gpu
@pytest.mark.parametrize("slices", [0, 1, 4, 6, 11])
def test_host_forward_equals_device_forward_for_every_grouping(cuda_device, slices):
    # batch 2 x 3 heads = 6 slices, L = 1800 (ragged last block)
    Q, K, V = I.make_qkv((5, 9, 40), heads=3, d=128, seed=31, batch=2, device=cuda_device)
    ref = api.forward(Q, K, V, 1.04, 128).cpu()
    hq, hk, hv = (_host(t, True) for t in (Q, K, V))
    out = torch.full_like(hq, float("nan")).pin_memory()
    api.forward_host(hq, hk, hv, 1.04, 128, out=out, slices_per_step=slices)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(out, ref)
    assert api.device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("kw", [dict(keep_or_drop=True), dict(diagonal_sigma=True), dict(route_in_kernel=True)])
def test_host_forward_flags(cuda_device, kw):
    Q, K, V = I.make_qkv((4, 16, 24), heads=5, d=128, seed=32, device=cuda_device)  # L = 1536
    ref = api.forward_ex(Q, K, V, 0.5, 128, **kw).cpu()
    out = api.forward_host(*(_host(t, True) for t in (Q, K, V)), 0.5, 128, slices_per_step=2, **kw)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(out, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("d,block,dtype", [(64, 128, torch.bfloat16), (128, (128, 64), torch.bfloat16),
                                           (64, 64, torch.float32)])
def test_host_forward_other_paths_and_pageable_memory(cuda_device, d, block, dtype):
    """d = 64, 64-token key blocks and the fp32 (CUDA-core) kernel, from
    pageable host memory (copies that block the host, same results)."""
    Q, K, V = I.make_qkv((3, 10, 33), heads=4, d=d, seed=33, dtype=dtype, device=cuda_device)  # L = 990
    ref = api.forward(Q, K, V, 1.04, block).cpu()
    out = api.forward_host(Q.cpu(), K.cpu(), V.cpu(), 1.04, block, slices_per_step=3)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(out, ref)


@pytest.mark.gpu
def test_host_forward_on_a_side_stream_back_to_back(cuda_device):
    """Two calls on a caller-owned stream, the second reading the host output
    of the first as its value tensor: stream order must hold across them."""
    Q, K, V = I.make_qkv((4, 8, 16), heads=3, d=128, seed=34, device=cuda_device)  # L = 512
    ref1 = api.forward(Q, K, V, 1.04, 128)
    ref2 = api.forward(Q, K, ref1, 1.04, 128).cpu()
    hq, hk, hv = (_host(t, True) for t in (Q, K, V))
    o1 = torch.empty_like(hq).pin_memory()
    o2 = torch.empty_like(hq).pin_memory()
    s = torch.cuda.Stream()
    api.forward_host(hq, hk, hv, 1.04, 128, out=o1, slices_per_step=1, stream=s)
    # o1 is written by the first call's copies back; the second call's copies in
    # are ordered after them on the same stream
    api.forward_host(hq, hk, o1, 1.04, 128, out=o2, slices_per_step=2, stream=s)
    s.synchronize()
    assert torch.equal(o1, ref1.cpu())
    assert torch.equal(o2, ref2)
