"""The debug build (-DSOL_ATTN_DEBUG_CHECKS) of the tensor-core kernel checks,
on every tile, that the item's tile count matches its selection, that tile
and block indices are in range, that each half's valid-column count is in
[0, 64] and that every row sum is positive; a failed check is recorded in
the device status word instead of trapping.  Here it runs the shapes the
kernel branches on and must report nothing and give the release build's
bits."""

import ctypes
import math

import pytest
import torch

from video_diffusion_b200 import api, build
from video_diffusion_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg(cuda_device):
    L = ctypes.CDLL(build.build(debug=True))
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    L.sol_attn_forward_ex.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                      ctypes.c_uint, vp, vp]
    L.sol_attn_forward_ex.restype = ctypes.c_int
    L.sol_attn_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    L.sol_attn_device_status.restype = ctypes.c_int
    build.build()
    api.lib()
    return L


CASES = [  # (grid, heads, d, (Bq, Bk), beta, flags)
    ((10, 10, 10), 2, 128, (128, 128), 1.04, 0),
    ((10, 10, 10), 2, 128, (128, 128), -math.inf, 0),
    ((10, 10, 10), 2, 128, (128, 128), math.inf, 0),
    ((10, 10, 10), 2, 128, (128, 64), 1.04, 0),
    ((10, 10, 10), 2, 64, (128, 128), 0.5, 0),
    ((10, 10, 10), 2, 128, (128, 128), 1.04, api.FLAG_KEEP_OR_DROP),
    ((10, 10, 10), 2, 128, (128, 64), 1.04, api.FLAG_ROUTE_IN_KERNEL | api.FLAG_DIAGONAL_SIGMA),
    ((21, 30, 52), 4, 128, (128, 128), 1.04, api.FLAG_ROUTE_IN_KERNEL),
    ((10, 10, 10), 2, 128, (64, 128), 1.04, 0),   # 64-token query blocks, two per tile
    ((3, 10, 31), 2, 64, (64, 64), 0.5, 0),       # L = 930: odd query-block count
    ((10, 10, 10), 2, 128, (64, 128), 2.0, api.FLAG_KEEP_OR_DROP),
]


@pytest.mark.parametrize("grid,heads,d,block,beta,flags", CASES)
def test_debug_checks_pass_and_match_release(dbg, grid, heads, d, block, beta, flags):
    Q, K, V = I.make_qkv(grid, heads=heads, d=d, seed=31, device="cuda")
    b, h, L, dd = Q.shape
    ref = api.forward_ex(Q, K, V, beta, block, keep_or_drop=bool(flags & api.FLAG_KEEP_OR_DROP),
                         diagonal_sigma=bool(flags & api.FLAG_DIAGONAL_SIGMA),
                         route_in_kernel=bool(flags & api.FLAG_ROUTE_IN_KERNEL))
    out = torch.full_like(Q, float("nan"))
    rc = dbg.sol_attn_forward_ex(Q.data_ptr(), K.data_ptr(), V.data_ptr(), out.data_ptr(), api.DTYPE_BF16, b, h,
                                 L, dd, block[0], block[1], beta, flags, None,
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    word = ctypes.c_int32(0)
    dbg.sol_attn_device_status(torch.cuda.current_stream().cuda_stream, ctypes.byref(word))
    assert word.value == 0, hex(word.value)
    assert torch.equal(out, ref)
