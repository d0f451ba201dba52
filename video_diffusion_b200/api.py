"""Python binding of libsolattn (the C ABI in include/sol_attn.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
compiled library is missing the first call raises; there is no fallback.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn.so")
_lib = None

SOL_OK = 0
STATUS = {0: "SOL_OK", -1: "SOL_ERR_INVALID_ARG", -2: "SOL_ERR_UNSUPPORTED", -3: "SOL_ERR_CUDA",
          -4: "SOL_ERR_NO_MEMORY", -5: "SOL_ERR_DEVICE_TIMEOUT"}
DTYPE_BF16, DTYPE_F32 = 0, 1
FLAG_KEEP_OR_DROP = 1  # correction off: unselected blocks contribute nothing
FLAG_DIAGONAL_SIGMA = 2  # sigma_i from the diagonal moment estimator
FLAG_ROUTE_IN_KERNEL = 4  # Eq. 4 decided inside the attention kernel (no selection mask)

EXPORTS = ("sol_attn_forward", "sol_attn_forward_f32", "sol_attn_forward_ex", "sol_attn_forward_host",
           "sol_attn_stats", "sol_attn_stats_ex", "sol_attn_near_ties", "sol_attn_cta_times", "sol_attn_device_status",
           "sol_attn_status_string", "sol_attn_version")


class SolAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Loads libsolattn.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m video_diffusion_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.sol_attn_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.sol_attn_forward_f32.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.sol_attn_forward_ex.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, ctypes.c_uint,
                                          vp, vp]
        L.sol_attn_forward_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.sol_attn_forward_host.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, ctypes.c_uint,
                                            i32, vp]
        L.sol_attn_stats.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp]
        L.sol_attn_stats_ex.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, ctypes.c_uint,
                                        vp]
        L.sol_attn_near_ties.argtypes = [vp, vp, vp, f32, i32, i32, i32, i32, i32, i32, f32, i32, ctypes.c_uint,
                                         vp]
        L.sol_attn_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        L.sol_attn_cta_times.argtypes = [vp, vp, i32]
        L.sol_attn_status_string.argtypes = [i32]
        L.sol_attn_status_string.restype = ctypes.c_char_p
        L.sol_attn_version.argtypes = []
        for name in ("sol_attn_forward", "sol_attn_forward_f32", "sol_attn_forward_ex", "sol_attn_stats",
                     "sol_attn_stats_ex", "sol_attn_device_status", "sol_attn_version",
                     "sol_attn_forward_noalloc", "sol_attn_forward_host", "sol_attn_near_ties",
                     "sol_attn_cta_times"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(fn: str, rc: int):
    if rc != SOL_OK:
        raise SolAttnError(fn, rc)


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _shape(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor | None = None):
    if q.dim() != 4:
        raise ValueError("expected [batch, heads, L, d] tensors")
    for t in (q, k) + ((v,) if v is not None else ()):
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v must share shape, dtype and device")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    return q.shape


def _out_like(q: torch.Tensor, out: torch.Tensor | None) -> torch.Tensor:
    """The output tensor: a new one like q, or the caller's after checking
    that the kernels' row stores stay inside it (same shape, dtype and device
    as q, contiguous CUDA memory)."""
    if out is None:
        return torch.empty_like(q)
    if not isinstance(out, torch.Tensor):
        raise ValueError("out must be a torch.Tensor")
    if out.shape != q.shape or out.dtype != q.dtype or out.device != q.device:
        raise ValueError(f"out must match q: shape {tuple(q.shape)}, dtype {q.dtype}, device {q.device} "
                         f"(got {tuple(out.shape)}, {out.dtype}, {out.device})")
    if not out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous CUDA tensor")
    return out


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def blocks(block) -> tuple[int, int]:
    """(Bq, Bk) from a block size or a (query, key) pair."""
    if isinstance(block, (tuple, list)):
        bq, bk = block
        return int(bq), int(bk)
    return int(block), int(block)


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: float, block=128,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Sol-Attn forward of [batch, heads, L, d] bf16 or fp32 tensors; block is
    one size for query and key blocks or a (Bq, Bk) pair."""
    b, h, L, d = _shape(q, k, v)
    bq, bk = blocks(block)
    out = _out_like(q, out)
    fn = lib().sol_attn_forward if q.dtype == torch.bfloat16 else lib().sol_attn_forward_f32
    _dtype_code(q)
    rc = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b, h, L, d, bq, bk,
            float(beta), _stream_handle(stream))
    _check("sol_attn_forward", rc)
    return out


def forward_ex(q, k, v, beta: float, block=128, out=None, events=None, stream=None,
               keep_or_drop: bool = False, diagonal_sigma: bool = False,
               route_in_kernel: bool = False) -> torch.Tensor:
    """forward() that also records up to four torch.cuda.Event objects: before
    pooling, after pooling, after routing, after the attention kernel.  The
    events must exist already (torch creates them on their first record()).
    keep_or_drop=True switches the correction off (unselected blocks
    contribute nothing; rows with no selected block give 0); diagonal_sigma=True
    takes sigma_i from the diagonal moment estimator; route_in_kernel=True has
    the attention kernel decide the selection itself (same results)."""
    b, h, L, d = _shape(q, k, v)
    bq, bk = blocks(block)
    out = _out_like(q, out)
    ev = None
    if events is not None:
        arr = (ctypes.c_void_p * 4)()
        for i, e in enumerate(events):
            arr[i] = int(e.cuda_event) if e is not None else 0
            if e is not None and arr[i] is None:
                raise ValueError("event not created yet: record it once before passing it")
        ev = ctypes.cast(arr, ctypes.c_void_p)
    rc = lib().sol_attn_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dtype_code(q),
                                   b, h, L, d, bq, bk, float(beta),
                                   _flags(keep_or_drop, diagonal_sigma, route_in_kernel), ev, _stream_handle(stream))
    _check("sol_attn_forward_ex", rc)
    return out


def _flags(keep_or_drop: bool, diagonal_sigma: bool, route_in_kernel: bool) -> int:
    return ((FLAG_KEEP_OR_DROP if keep_or_drop else 0) | (FLAG_DIAGONAL_SIGMA if diagonal_sigma else 0)
            | (FLAG_ROUTE_IN_KERNEL if route_in_kernel else 0))


def forward_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: float, block=128,
                 out: torch.Tensor | None = None, slices_per_step: int = 0, stream=None,
                 keep_or_drop: bool = False, diagonal_sigma: bool = False,
                 route_in_kernel: bool = False) -> torch.Tensor:
    """forward() of [batch, heads, L, d] tensors in host memory (pin them for
    overlapped copies): the library streams groups of (batch, head) slices
    through device staging buffers on the current CUDA device, copying the
    next group in and the previous group out while it computes.  `out` (a
    host tensor) is complete once `stream` has reached this call; synchronise
    it before reading."""
    if q.dim() != 4:
        raise ValueError("expected [batch, heads, L, d] tensors")
    for t in (q, k, v):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v must share shape and dtype")
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous host tensors")
    b, h, L, d = q.shape
    bq, bk = blocks(block)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    if out.shape != q.shape or out.dtype != q.dtype or out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor like q")
    rc = lib().sol_attn_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dtype_code(q),
                                     b, h, L, d, bq, bk, float(beta),
                                     _flags(keep_or_drop, diagonal_sigma, route_in_kernel), int(slices_per_step),
                                     _stream_handle(stream))
    _check("sol_attn_forward_host", rc)
    return out


def stats(q: torch.Tensor, k: torch.Tensor, beta: float, block=128, with_mask: bool = False,
          stream=None, diagonal_sigma: bool = False):
    """Selected-block counts [batch, heads, Nq] (int32) and, if asked, the
    selection as a bool tensor [batch, heads, Nq, Nk] unpacked from the
    library's 1-bit mask."""
    b, h, L, d = _shape(q, k)
    bq, bk = blocks(block)
    Nq, Nk = -(-L // bq), -(-L // bk)
    W = -(-Nk // 32)
    counts = torch.empty(b, h, Nq, dtype=torch.int32, device=q.device)
    mask = torch.empty(b, h, Nq, W, dtype=torch.int32, device=q.device) if with_mask else None
    rc = lib().sol_attn_stats_ex(q.data_ptr(), k.data_ptr(), counts.data_ptr(),
                                 mask.data_ptr() if mask is not None else None, b, h, L, d, bq, bk,
                                 float(beta), _dtype_code(q), FLAG_DIAGONAL_SIGMA if diagonal_sigma else 0,
                                 _stream_handle(stream))
    _check("sol_attn_stats_ex", rc)
    if mask is None:
        return counts
    return counts, unpack_mask(mask, Nk)


def near_ties(q: torch.Tensor, k: torch.Tensor, beta: float, block=128, margin: float = 1e-3, stream=None,
              diagonal_sigma: bool = False) -> torch.Tensor:
    """Per query block, the number of key blocks whose proxy score lies within
    `margin` of the block's threshold tau_i ([batch, heads, Nq] int32)."""
    b, h, L, d = _shape(q, k)
    bq, bk = blocks(block)
    near = torch.empty(b, h, -(-L // bq), dtype=torch.int32, device=q.device)
    rc = lib().sol_attn_near_ties(q.data_ptr(), k.data_ptr(), near.data_ptr(), float(margin), b, h, L, d, bq, bk,
                                  float(beta), _dtype_code(q), FLAG_DIAGONAL_SIGMA if diagonal_sigma else 0,
                                  _stream_handle(stream))
    _check("sol_attn_near_ties", rc)
    return near


def unpack_mask(words: torch.Tensor, N: int) -> torch.Tensor:
    """[..., W] int32 words -> [..., N] bool, bit j % 32 of word j // 32."""
    shifts = torch.arange(32, device=words.device, dtype=torch.int64)
    bits = (words.to(torch.int64).unsqueeze(-1) >> shifts) & 1
    return bits.reshape(*words.shape[:-1], words.shape[-1] * 32)[..., :N].bool()


def cta_times(stream=None, max_rows: int = 1024):
    """Per-CTA record of the last tensor-core attention launch: an int64
    array [ctas, 4] of start ns, end ns, work items, tiles (synchronises)."""
    import numpy as np
    buf = np.zeros((max_rows, 4), dtype=np.uint64)
    n = lib().sol_attn_cta_times(_stream_handle(stream), buf.ctypes.data, int(max_rows))
    if n < 0:
        _check("sol_attn_cta_times", n)
    return buf[:n].astype(np.int64)


def load_balance(rows) -> dict:
    """Busy spread of one launch from cta_times(): per-CTA busy time
    (end - start), its max / mean, and the tail-idle fraction = CTA time left
    idle between each CTA's end and the last CTA's end, over all CTAs' span."""
    import numpy as np
    rows = np.asarray(rows, dtype=np.int64)
    if len(rows) == 0:
        return {}
    t0, t1 = rows[:, 0].min(), rows[:, 1].max()
    busy = (rows[:, 1] - rows[:, 0]).astype(np.float64)
    span = float(t1 - t0)
    return {"ctas": int(len(rows)), "span_ms": span * 1e-6, "busy_max_over_mean": float(busy.max() / busy.mean()),
            "busy_min_over_mean": float(busy.min() / busy.mean()),
            "tail_idle_fraction": float((t1 - rows[:, 1]).sum() / (span * len(rows))) if span > 0 else 0.0,
            "start_skew_ms": float(rows[:, 0].max() - t0) * 1e-6,
            "items_max_over_mean": float(rows[:, 2].max() / max(rows[:, 2].mean(), 1e-9)),
            "tiles_max_over_mean": float(rows[:, 3].max() / max(rows[:, 3].mean(), 1e-9))}


def device_status(stream=None) -> int:
    """Synchronises the stream, reads and clears the device status word."""
    w = ctypes.c_int32(0)
    rc = lib().sol_attn_device_status(_stream_handle(stream), ctypes.byref(w))
    if rc not in (SOL_OK, -5):
        _check("sol_attn_device_status", rc)
    return int(w.value)


def status_string(code: int) -> str:
    return lib().sol_attn_status_string(int(code)).decode()


def version() -> int:
    return int(lib().sol_attn_version())


def n_blocks(L: int, block: int) -> int:
    return -(-L // block)


def beta_is_dense(beta: float) -> bool:
    return beta == -math.inf
