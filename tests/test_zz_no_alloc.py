"""sol_attn_forward_noalloc: the forward for callers that may not allocate
device memory (plugin hosts that own all device memory, serving loops that
reserve everything up front).  It takes its scratch from a fixed array in the
library, so it must give the same results as sol_attn_forward call after
call, even though the array keeps the previous call's contents.  Both entry
points run the same deterministic kernels on the same inputs, so the outputs
must be equal bit for bit: a tolerance would hide stale scratch that shifts a
few pooled values.

This file is collected last on purpose: it runs after every other GPU test
in a full run, and also passes alone in a fresh process."""

import ctypes

import pytest
import torch

from video_diffusion_b200 import api, build
from video_diffusion_b200 import inputs as I


def _fn():
    build.build()
    f = api.lib().sol_attn_forward_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.c_float, vp]
    f.restype = ctypes.c_int
    return f


def _noalloc(f, Q, K, V, bq, bk, beta):
    stream = torch.cuda.current_stream()
    out = torch.full_like(Q, float("nan"))
    b, h, L, d = Q.shape
    rc = f(Q.data_ptr(), K.data_ptr(), V.data_ptr(), out.data_ptr(), b, h, L, d, bq, bk, beta, stream.cuda_stream)
    assert rc == 0, api.status_string(rc)
    torch.cuda.synchronize()
    return out


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_device):
    f = _fn()
    # two different inputs back to back: the second call must not see the
    # first call's leftovers in the shared scratch
    cases = [((8, 16, 24), 4, 21, 1.04), ((5, 9, 40), 3, 22, 0.5)]  # L = 3072 and 1800 (ragged)
    for grid, heads, seed, beta in cases:
        Q, K, V = I.make_qkv(grid, heads=heads, d=128, seed=seed, device=cuda_device)
        ref = api.forward(Q, K, V, beta, 128)
        out = _noalloc(f, Q, K, V, 128, 128, beta)
        assert torch.equal(out, ref)
    assert api.device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("d,bk", [(128, 64), (64, 128)])
def test_noalloc_other_shapes_match_forward(cuda_device, d, bk):
    """64-token key blocks (two per tensor-core tile) and 64-wide heads take
    the same kernels through the fixed scratch."""
    f = _fn()
    Q, K, V = I.make_qkv((5, 9, 40), heads=3, d=d, seed=23, device=cuda_device)  # L = 1800 (ragged)
    ref = api.forward(Q, K, V, 1.04, (128, bk))
    for _ in range(2):
        assert torch.equal(_noalloc(f, Q, K, V, 128, bk, 1.04), ref)
    assert api.device_status() == 0


@pytest.mark.gpu
def test_noalloc_cuda_core_path_after_a_larger_call(cuda_device):
    """A bf16 call with 64-token query blocks runs the CUDA-core kernel on
    fp32 pooled operands.  Made right after a larger tensor-core call, it
    would read that call's pooled rows and selection words if it skipped a
    reset of anything it reads."""
    f = _fn()
    Qa, Ka, Va = I.make_qkv((6, 16, 32), heads=4, d=128, seed=31, device=cuda_device)  # L = 3072
    assert torch.equal(_noalloc(f, Qa, Ka, Va, 128, 128, 0.5), api.forward(Qa, Ka, Va, 0.5, 128))
    Q, K, V = I.make_qkv((3, 7, 30), heads=2, d=128, seed=32, device=cuda_device)  # L = 630 (ragged)
    ref = api.forward(Q, K, V, 1.04, (64, 64))
    assert torch.equal(_noalloc(f, Q, K, V, 64, 64, 1.04), ref)
    assert api.device_status() == 0


def test_noalloc_rejects_calls_larger_than_its_scratch():
    f = _fn()
    fake = 0x10000  # never dereferenced: the size check comes before any CUDA call
    # 400 heads of L = 75600 need about 384 MiB of scratch, more than the fixed 48 MiB
    rc = f(fake, fake, fake, fake, 1, 400, 75600, 128, 128, 128, 1.04, None)
    assert rc == -4 and api.status_string(rc) == "SOL_ERR_NO_MEMORY"
    # the Wan2.1 720p call fits with 128-token key blocks (about 37 MiB) but
    # not with 64-token key blocks (about 61 MiB); the 128 case is not run
    # here (it would launch), only the refusal is
    rc = f(fake, fake, fake, fake, 1, 40, 75600, 128, 128, 64, 1.04, None)
    assert rc == -4
    rc = f(fake, fake, fake, fake, 1, 24, 119056, 128, 128, 64, 1.04, None)
    assert rc == -4
    # argument errors are reported as for sol_attn_forward
    assert f(0, fake, fake, fake, 1, 1, 256, 128, 128, 128, 1.0, None) == -1
