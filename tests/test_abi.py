"""Host checks of the C ABI: the library loads, exports every declared entry
point, and rejects bad arguments before touching the GPU."""

import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from video_diffusion_b200 import build, api
    build.build()
    return api.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "sol_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sol_attn_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "sol_attn_forward" in names and "sol_attn_stats" in names
    for n in names:
        assert hasattr(L, n), n
    from video_diffusion_b200 import api
    assert set(api.EXPORTS) <= set(names)


def test_status_strings_and_version(L):
    from video_diffusion_b200 import api
    assert api.status_string(0) == "SOL_OK"
    assert api.status_string(-1) == "SOL_ERR_INVALID_ARG"
    assert api.status_string(-5) == "SOL_ERR_DEVICE_TIMEOUT"
    assert api.status_string(7) == "SOL_ERR_UNKNOWN"
    assert api.version() == 105


# Argument checks run on the host before any CUDA call, so fake device
# addresses are never dereferenced.
FAKE = 0x10000


def call_fwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, b=1, h=1, n=256, d=128, bq=128, bk=128, beta=1.0):
    return L.sol_attn_forward(q, k, v, o, b, h, n, d, bq, bk, ctypes.c_float(beta), None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(k=0), -1), (dict(v=0), -1), (dict(o=0), -1),
    (dict(q=FAKE + 8), -1), (dict(o=FAKE + 2), -1),
    (dict(b=0), -1), (dict(h=0), -1), (dict(n=0), -1), (dict(d=0), -1),
    (dict(beta=float("nan")), -1),
    (dict(d=96), -2), (dict(d=256), -2), (dict(bq=96, bk=128), -2), (dict(bq=128, bk=32), -2),
    (dict(bq=32, bk=32), -2), (dict(bq=256, bk=256), -2), (dict(bq=128, bk=256), -2),
    (dict(n=64 * 6145, bk=64), -2), (dict(n=128 * 6145), -2),
    # batch * heads is a grid dimension of the prologue kernels (at most 65535)
    (dict(b=2, h=32768, n=4), -2), (dict(b=1, h=65536, n=4), -2),
])
def test_forward_rejects_bad_arguments(L, kw, code):
    assert call_fwd(L, **kw) == code


def test_stats_and_ex_reject_bad_arguments(L):
    f = ctypes.c_float
    assert L.sol_attn_stats(FAKE, FAKE, None, None, 1, 1, 256, 128, 128, 128, f(1.0), 0, None) == -1
    assert L.sol_attn_stats(FAKE, FAKE, FAKE, None, 1, 1, 256, 128, 128, 128, f(1.0), 9, None) == -1
    assert L.sol_attn_stats(FAKE, FAKE, FAKE, None, 1, 1, 256, 100, 128, 128, f(1.0), 0, None) == -2
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 5, 1, 1, 256, 128, 128, 128, f(1.0), 0, None, None) == -1
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 256, 128, 128, 128, f(1.0), 9, None, None) == -1
    assert L.sol_attn_forward_f32(FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 64, 64, 64, f(math.nan), None) == -1
    # stats_ex takes SOL_FLAG_DIAGONAL_SIGMA only; forward_ex both flags, no other bit
    assert L.sol_attn_stats_ex(FAKE, FAKE, FAKE, None, 1, 1, 256, 128, 128, 128, f(1.0), 0, 1, None) == -1
    assert L.sol_attn_stats_ex(FAKE, FAKE, FAKE, None, 1, 1, 256, 128, 128, 128, f(1.0), 0, 4, None) == -1
    assert L.sol_attn_stats_ex(FAKE, FAKE, None, None, 1, 1, 256, 128, 128, 128, f(1.0), 0, 2, None) == -1
    assert L.sol_attn_stats_ex(FAKE, FAKE, FAKE, None, 1, 1, 256, 128, 128, 96, f(1.0), 0, 2, None) == -2
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 256, 128, 128, 128, f(1.0), 8, None, None) == -1
    # in-kernel routing: tensor-core calls only, at most 2048 key blocks
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 256, 128, 128, 128, f(1.0), 4, None, None) == -2
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 256, 128, 64, 64, f(1.0), 4, None, None) == -2
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 64 * 2049, 128, 128, 64, f(1.0), 4, None,
                                 None) == -2
    assert L.sol_attn_forward_ex(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 256, 96, 128, 64, f(1.0), 3, None, None) == -2


def test_near_ties_rejects_bad_arguments(L):
    f = ctypes.c_float

    def call(q=FAKE, k=FAKE, out=FAKE, margin=1e-3, b=1, h=1, n=256, d=128, bq=128, bk=128, beta=1.0, dtype=0,
             flags=0):
        return L.sol_attn_near_ties(q, k, out, f(margin), b, h, n, d, bq, bk, f(beta), dtype, flags, None)

    assert call(out=0) == -1 and call(q=0) == -1
    assert call(margin=-1e-3) == -1 and call(margin=math.nan) == -1 and call(margin=math.inf) == -1
    assert call(beta=math.nan) == -1 and call(dtype=7) == -1 and call(flags=1) == -1
    assert call(d=96) == -2 and call(bk=32) == -2


def test_cta_times_arguments_and_load_balance_summary(L):
    import numpy as np
    from video_diffusion_b200 import api
    assert L.sol_attn_cta_times(None, None, 4) == -1
    buf = np.zeros((4, 4), dtype=np.uint64)
    assert L.sol_attn_cta_times(None, buf.ctypes.data, -1) == -1
    assert L.sol_attn_cta_times(None, buf.ctypes.data, 4) == 0  # no attention launch in this process
    # three CTAs over [0, 100] ns: busy 100, 70, 95; idle tails 0, 20, 0
    rows = np.array([[0, 100, 3, 30], [10, 80, 2, 25], [5, 100, 3, 31]])
    lb = api.load_balance(rows)
    assert lb["ctas"] == 3 and abs(lb["span_ms"] - 1e-4) < 1e-12
    assert abs(lb["busy_max_over_mean"] - 100 / (265 / 3)) < 1e-12
    assert abs(lb["tail_idle_fraction"] - 20 / 300) < 1e-12
    assert abs(lb["tiles_max_over_mean"] - 31 / (86 / 3)) < 1e-12
    assert api.load_balance(np.zeros((0, 4))) == {}


def test_forward_host_rejects_bad_arguments(L):
    """The host-buffer entry point checks everything before its first CUDA call."""
    f = ctypes.c_float

    def call(q=FAKE, k=FAKE, v=FAKE, o=FAKE, dtype=0, b=1, h=2, n=256, d=128, bq=128, bk=128, beta=1.0,
             flags=0, g=0):
        return L.sol_attn_forward_host(q, k, v, o, dtype, b, h, n, d, bq, bk, f(beta), flags, g, None)

    assert call(q=0) == -1 and call(v=0) == -1 and call(o=0) == -1
    assert call(k=FAKE + 4) == -1
    assert call(dtype=3) == -1
    assert call(flags=8) == -1
    assert call(g=-1) == -1
    assert call(beta=math.nan) == -1
    assert call(h=0) == -1
    assert call(d=80) == -2
    assert call(bq=128, bk=32) == -2
    assert call(dtype=1, flags=4) == -2  # in-kernel routing needs the tensor-core path


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from video_diffusion_b200 import api
    monkeypatch.setattr(api, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(api, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        api.lib()


def test_binding_rejects_bad_tensors_before_calling_the_library():
    """The Python binding checks layout, device and dtype itself (ValueError)
    before anything reaches the C ABI."""
    import torch
    from video_diffusion_b200 import api
    q = torch.zeros(1, 2, 256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        api.forward(q, q, q, 1.0)  # host tensors to the device entry point
    with pytest.raises(ValueError, match="batch, heads, L, d"):
        api.forward(q[0], q[0], q[0], 1.0)
    with pytest.raises(ValueError, match="share"):
        api.forward_host(q, q, q[:, :, :128], 1.0)
    with pytest.raises(ValueError, match="contiguous"):
        api.forward_host(q.transpose(2, 3), q.transpose(2, 3), q.transpose(2, 3), 1.0)
    with pytest.raises(ValueError, match="out"):
        api.forward_host(q, q, q, 1.0, out=torch.zeros(1, 2, 256, 128, dtype=torch.float32))
    assert api.blocks(128) == (128, 128) and api.blocks((128, 64)) == (128, 64)
    # a caller's output tensor must match q exactly: the kernels write every
    # row with 16- or 32-byte stores, so a smaller, wider-typed or strided
    # `out` would be written past its end
    with pytest.raises(ValueError, match="out must match q"):
        api._out_like(q, torch.zeros(1, 2, 128, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must match q"):
        api._out_like(q, torch.zeros(1, 2, 256, 128, dtype=torch.float32))
    with pytest.raises(ValueError, match="out must match q"):
        api._out_like(q, torch.zeros(1, 2, 256, 128, dtype=torch.bfloat16, device="meta"))
    with pytest.raises(ValueError, match="contiguous CUDA"):
        api._out_like(q, torch.zeros(1, 2, 128, 256, dtype=torch.bfloat16).transpose(2, 3))
    with pytest.raises(ValueError, match="torch.Tensor"):
        api._out_like(q, [0.0])
    words = torch.tensor([[0b101, 1 << 31]], dtype=torch.int64).to(torch.int32)
    bits = api.unpack_mask(words, 40)
    assert bits.shape == (1, 40)
    assert bits[0, 0] and not bits[0, 1] and bits[0, 2] and not bits[0, 31] and not bits[0, 39]
    words = torch.tensor([[0, -2147483648]], dtype=torch.int32)  # bit 31 of word 1 = block 63
    assert api.unpack_mask(words, 64)[0, 63] and api.unpack_mask(words, 64).sum() == 1
