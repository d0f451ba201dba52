"""Helpers for GPU-vs-oracle parity: selection comparison with the near-tie
rule, oracle outputs on sampled query blocks, error metrics."""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import sol_attn as O

# bf16 operands: max-abs 2e-2 and relative L2 1e-2; fp32: relative L2 1e-4.
TOL = {torch.bfloat16: dict(max_abs=2e-2, rel_l2=1e-2), torch.float32: dict(max_abs=1e-3, rel_l2=1e-4)}


def head_np(t: torch.Tensor, b: int, h: int) -> np.ndarray:
    return t[b, h].detach().to("cpu", torch.float64).numpy()


def compare_selection(route: dict, gpu_sel: np.ndarray, gpu_counts: np.ndarray) -> dict:
    """Asserts the GPU's selection equals the oracle's except on near-ties
    (|s_ij - tau_i| < NEAR_TIE); returns mismatch statistics."""
    osel = route["sel"]
    assert gpu_sel.shape == osel.shape, (gpu_sel.shape, osel.shape)
    np.testing.assert_array_equal(gpu_counts, gpu_sel.sum(axis=1))
    diff = gpu_sel != osel
    n_diff = int(diff.sum())
    if n_diff:
        gap = np.abs(route["s"] - route["tau"][:, None])[diff]
        assert np.all(gap < O.NEAR_TIE), f"{n_diff} selection mismatches, max gap {gap.max():.3g}"
    return dict(mismatches=n_diff, pairs=int(osel.size), selected=int(osel.sum()))


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def check_close(gpu: np.ndarray, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    tol = TOL[dtype]
    assert np.isfinite(gpu).all(), f"{what}: non-finite GPU output"
    err = float(np.abs(gpu - ref).max())
    rl = rel_l2(gpu, ref)
    assert rl <= tol["rel_l2"], f"{what}: rel-L2 {rl:.3g} > {tol['rel_l2']}"
    if dtype == torch.bfloat16:
        assert err <= tol["max_abs"], f"{what}: max-abs {err:.3g} > {tol['max_abs']}"
    return dict(max_abs=err, rel_l2=rl)


def sample_blocks(N: int, counts_row: np.ndarray, k: int, rng: np.random.Generator, extra=()) -> list[int]:
    """First, last, max-count and min-count blocks plus `extra` and random ones."""
    pick = {0, N - 1, int(np.argmax(counts_row)), int(np.argmin(counts_row)), *extra}
    while len(pick) < min(k, N):
        pick.add(int(rng.integers(0, N)))
    return sorted(pick)


def pair(block) -> tuple[int, int]:
    """(Bq, Bk) from one block size or a (query, key) pair."""
    if isinstance(block, (tuple, list)):
        return int(block[0]), int(block[1])
    return int(block), int(block)


def oracle_rows(Q, K, V, b, h, block, beta, sel, blocks, moments="eq5", correction=True):
    """Oracle output rows of the given query blocks of head (b, h), using the
    selection `sel` (the GPU's, checked against the oracle's beforehand)."""
    bq, bk = pair(block)
    out, _ = O.forward_head(head_np(Q, b, h), head_np(K, b, h), head_np(V, b, h), bq, bk, beta,
                            sel=sel, query_blocks=blocks, moments=moments, correction=correction)
    return out


def rows_of(blocks, block, L):
    """Token rows of the given query blocks (block: Bq or a (Bq, Bk) pair)."""
    bq = pair(block)[0]
    idx = []
    for i in blocks:
        idx.extend(range(i * bq, min(L, i * bq + bq)))
    return np.asarray(idx, dtype=np.int64)
