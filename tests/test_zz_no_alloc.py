"""sol_attn_forward_noalloc: the forward for callers that may not allocate
device memory (plugin hosts that own all device memory, serving loops that
reserve everything up front).  It takes its scratch from a fixed array in the
library, so it must give the same results as sol_attn_forward call after
call, even though the array keeps the previous call's contents.

This file is collected last on purpose: it runs after every other GPU test
in a full run, and also passes alone in a fresh process."""

import ctypes

import numpy as np
import pytest
import torch

from tests import parity_helpers as P
from video_diffusion_b200 import api, build
from video_diffusion_b200 import inputs as I


def _fn():
    build.build()
    f = api.lib().sol_attn_forward_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.c_float, vp]
    f.restype = ctypes.c_int
    return f


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_device):
    f = _fn()
    stream = torch.cuda.current_stream()
    # two different inputs back to back: the second call must not see the
    # first call's leftovers in the shared scratch
    cases = [((8, 16, 24), 4, 21, 1.04), ((5, 9, 40), 3, 22, 0.5)]  # L = 3072 and 1800 (ragged)
    for grid, heads, seed, beta in cases:
        Q, K, V = I.make_qkv(grid, heads=heads, d=128, seed=seed, device=cuda_device)
        ref = api.forward(Q, K, V, beta, 128)
        out = torch.full_like(Q, float("nan"))
        b, h, L, d = Q.shape
        rc = f(Q.data_ptr(), K.data_ptr(), V.data_ptr(), out.data_ptr(), b, h, L, d, 128, 128, beta,
               stream.cuda_stream)
        assert rc == 0, api.status_string(rc)
        torch.cuda.synchronize()
        assert not torch.isnan(out).any()
        P.check_close(out.double().cpu().numpy(), ref.double().cpu().numpy(), torch.bfloat16, "noalloc vs forward")
    assert api.device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("d,bk", [(128, 64), (64, 128)])
def test_noalloc_other_shapes_match_forward(cuda_device, d, bk):
    """64-token key blocks (two per tensor-core tile) and 64-wide heads take
    the same kernels through the fixed scratch."""
    f = _fn()
    stream = torch.cuda.current_stream()
    Q, K, V = I.make_qkv((5, 9, 40), heads=3, d=d, seed=23, device=cuda_device)  # L = 1800 (ragged)
    ref = api.forward(Q, K, V, 1.04, (128, bk))
    for _ in range(2):
        out = torch.full_like(Q, float("nan"))
        b, h, L, dd = Q.shape
        rc = f(Q.data_ptr(), K.data_ptr(), V.data_ptr(), out.data_ptr(), b, h, L, dd, 128, bk, 1.04,
               stream.cuda_stream)
        assert rc == 0, api.status_string(rc)
        torch.cuda.synchronize()
        assert not torch.isnan(out).any()
        P.check_close(out.double().cpu().numpy(), ref.double().cpu().numpy(), torch.bfloat16, "noalloc vs forward")
    assert api.device_status() == 0


def test_noalloc_rejects_calls_larger_than_its_scratch():
    f = _fn()
    fake = 0x10000  # never dereferenced: the size check comes before any CUDA call
    # 400 heads of L = 75600 need about 384 MiB of scratch, more than the fixed 48 MiB
    rc = f(fake, fake, fake, fake, 1, 400, 75600, 128, 128, 128, 1.04, None)
    assert rc == -4 and api.status_string(rc) == "SOL_ERR_NO_MEMORY"
    # argument errors are reported as for sol_attn_forward
    assert f(0, fake, fake, fake, 1, 1, 256, 128, 128, 128, 1.0, None) == -1
