"""Float64 CPU oracle of the Sol-Attn single-pass sparse attention forward.

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Nothing in the CUDA
library imports this file; it is slow on purpose and written so that each step
can be checked against the formula it restates.

Method (Sol-Attn visual explainer, "The complete idea in one pass"):
  1. pool Q and K into per-block means and V into per-block sums;
  2. score each query block against each key block through the pooled vectors;
  3. threshold each score row at tau_i = mu_i + beta * sigma_i (Eq. 4, Eq. 5);
  4. selected key blocks are attended exactly, token by token;
  5. every unselected block is folded in through its pooled key and summed
     value (Eq. 9 denominator, Eq. 10 numerator), in the same softmax.

Readings taken where the pages are silent (the CUDA path takes the same ones):
  * logits carry the usual 1/sqrt(d) scale (standard attention definition in
    the papers.ananclaw.com explainer, "解决什么真问题"); Eqs. 9-11 print the
    exponent without it.  The threshold decision is unchanged by any positive
    scale.
  * blocks are contiguous runs of B tokens in the given order; the last block
    may be partial.  Its weight in Eq. 9 is its real token count n_j (the
    legend of Eq. 9 defines B as "tokens per block"), and it counts once in
    the moments of Eq. 5 (N = number of key blocks).
  * sigma is the population standard deviation (1/N, Eq. 5).
  * selection is strict: s_ij > tau_i (Eq. 4).  beta = -inf selects every
    block, beta = +inf selects none (handled without forming inf * 0).
  * no causal mask and no forced diagonal blocks (none is named anywhere).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Pairs with |s_ij - tau_i| below this (scaled-logit units) may be decided
# either way by an implementation that rounds differently.
NEAR_TIE = 1e-3


@dataclass(frozen=True)
class BlockGeometry:
    """Contiguous token blocks: block b covers [starts[b], starts[b] + counts[b])."""

    L: int
    B: int
    starts: np.ndarray
    counts: np.ndarray

    @property
    def n(self) -> int:
        return int(self.counts.shape[0])


def block_geometry(L: int, B: int) -> BlockGeometry:
    """Tokens grouped into hardware-sized blocks of B tokens (Sol-Attn visual
    explainer, glossary "Block / tile"); the tail block holds the remainder."""
    if L < 1 or B < 1:
        raise ValueError("L and B must be >= 1")
    starts = np.arange(0, L, B, dtype=np.int64)
    counts = np.minimum(B, L - starts)
    return BlockGeometry(L, B, starts, counts)


def pool_blocks(X: np.ndarray, geom: BlockGeometry, reduce: str) -> np.ndarray:
    """Per-block representative of the rows of X [L, d].

    reduce="mean" gives the pooled query / key (Q-bar_i, K-bar_j: "mean query
    vector in block i", "mean key vector in block j", legend of Eq. 5);
    reduce="sum" gives the summed value V-hat_j (legend of Eq. 10: "summed and
    original values").
    """
    X = np.asarray(X, dtype=np.float64)
    out = np.empty((geom.n, X.shape[1]), dtype=np.float64)
    for b in range(geom.n):
        s, n = int(geom.starts[b]), int(geom.counts[b])
        rows = X[s:s + n]
        total = rows.sum(axis=0)
        if reduce == "sum":
            out[b] = total
        elif reduce == "mean":
            out[b] = total / n
        else:
            raise ValueError(reduce)
    return out


def proxy_scores(Qbar: np.ndarray, Kbar: np.ndarray, scale: float) -> np.ndarray:
    """s-hat_ij = Q-bar_i K-bar_j^T ("pooled block proxy score", legend of
    Eq. 4), in scaled-logit units.  Returns the full [Nq, Nk] map -- fine on
    the host; the method's point is that the GPU never stores it."""
    return scale * (np.asarray(Qbar, np.float64) @ np.asarray(Kbar, np.float64).T)


def row_moments(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Mean and population standard deviation of every proxy-score row, two
    passes over the row (the quantities Eq. 5 computes without the row)."""
    s = np.asarray(s, np.float64)
    mu = s.mean(axis=1)
    var = ((s - mu[:, None]) ** 2).mean(axis=1)
    return mu, np.sqrt(var)


def eq5_moments(Qbar: np.ndarray, Kbar: np.ndarray, scale: float) -> tuple[np.ndarray, np.ndarray]:
    """Eq. 5 as printed: mu_i = Q-bar_i ((1/N) sum_j K-bar_j)^T and
    sigma_i^2 = Q-bar_i ((1/N) sum_j K-bar_j^T K-bar_j) Q-bar_i^T - mu_i^2,
    both times the logit scale (sigma^2 times its square)."""
    Qbar = np.asarray(Qbar, np.float64)
    Kbar = np.asarray(Kbar, np.float64)
    N = Kbar.shape[0]
    kmean = Kbar.sum(axis=0) / N
    second = (Kbar.T @ Kbar) / N  # (1/N) sum_j K-bar_j^T K-bar_j, d x d
    mu = scale * (Qbar @ kmean)
    var = scale * scale * np.einsum("id,de,ie->i", Qbar, second, Qbar) - mu * mu
    return mu, np.sqrt(np.maximum(var, 0.0))


def diagonal_sigma(Qbar: np.ndarray, Kbar: np.ndarray, scale: float) -> np.ndarray:
    """The cheaper "diagonal estimator" of sigma_i that the Sol-Attn visual
    explainer names beside Eq. 5 (its formula is not printed there).  Reading:
    the d x d centred second moment of the pooled keys,
    C = (1/N) sum_j (K-bar_j - k)^T (K-bar_j - k) with k the mean pooled key,
    is replaced by its diagonal, so that

        sigma_i^2 ~ scale^2 sum_c Q-bar_{i,c}^2 Var_j(K-bar_{j,c})

    (population variance over the N key blocks).  It equals the Eq. 5 sigma
    whenever the pooled-key channels are uncorrelated over the blocks, and
    always when Q-bar_i has one non-zero channel."""
    Qbar = np.asarray(Qbar, np.float64)
    Kbar = np.asarray(Kbar, np.float64)
    N = Kbar.shape[0]
    kmean = Kbar.sum(axis=0) / N
    var_c = ((Kbar - kmean[None, :]) ** 2).sum(axis=0) / N    # Var_j(K-bar_{j,c}), one per channel
    return scale * np.sqrt((Qbar * Qbar) @ var_c)


MOMENTS = ("eq5", "diagonal")


def threshold(mu: np.ndarray, sigma: np.ndarray, beta: float) -> np.ndarray:
    """tau_i = mu_i + beta sigma_i (Eq. 4).  beta = -inf gives tau = -inf and
    beta = +inf gives tau = +inf for every row, also where sigma_i = 0."""
    mu = np.asarray(mu, np.float64)
    if math.isnan(beta):
        raise ValueError("beta is NaN")
    if beta == -math.inf:
        return np.full_like(mu, -math.inf)
    if beta == math.inf:
        return np.full_like(mu, math.inf)
    return mu + beta * np.asarray(sigma, np.float64)


def select_blocks(s: np.ndarray, tau: np.ndarray) -> np.ndarray:
    """S_i = {j : s-hat_ij > tau_i} (Eq. 4, strict).  Boolean [Nq, Nk]."""
    return np.asarray(s, np.float64) > np.asarray(tau, np.float64)[:, None]


def route_head(Qh, Kh, Bq: int, Bk: int, beta: float, moments: str = "eq5") -> dict:
    """Steps 1-3 for one (batch, head): pooling, proxy scores, Eq. 4 routing.

    moments="eq5": mu_i and sigma_i of the score row (Eq. 5).
    moments="diagonal": the same mu_i, sigma_i from ``diagonal_sigma``."""
    if moments not in MOMENTS:
        raise ValueError(moments)
    Qh = np.asarray(Qh, np.float64)
    Kh = np.asarray(Kh, np.float64)
    L, d = Qh.shape
    scale = 1.0 / math.sqrt(d)
    qg, kg = block_geometry(L, Bq), block_geometry(L, Bk)
    Qbar = pool_blocks(Qh, qg, "mean")
    Kbar = pool_blocks(Kh, kg, "mean")
    s = proxy_scores(Qbar, Kbar, scale)
    mu, sigma = row_moments(s)
    if moments == "diagonal":
        sigma = diagonal_sigma(Qbar, Kbar, scale)
    tau = threshold(mu, sigma, beta)
    sel = select_blocks(s, tau)
    return dict(qgeom=qg, kgeom=kg, Qbar=Qbar, Kbar=Kbar, s=s, mu=mu, sigma=sigma, tau=tau, sel=sel)


def attend_query_block(Qi, Kh, Vh, kgeom: BlockGeometry, Kbar, Vhat, sel_row, scale: float,
                       correction: bool = True) -> np.ndarray:
    """Output rows of one query block, Eqs. 9 and 10 as printed.

    D_i = sum_{j in U_i} n_j exp(Q_i K-bar_j^T) + sum_{j in S_i} RowSum(exp(Q_i K_j^T))
    N_i = sum_{j in U_i} exp(Q_i K-bar_j^T) V-hat_j + sum_{j in S_i} exp(Q_i K_j^T) V_j
    out = N_i / D_i (the online-softmax state after the last block).

    Every exponent is shifted by the row maximum m of all exponents taken; the
    shift multiplies D and N by the same factor and cancels in N / D.

    correction=False is the keep-or-drop baseline the pages contrast Sol-Attn
    with (visual explainer, "Ordinary block sparse": every unselected block
    contributes zero): only the "Exact" terms remain.  With no block selected
    D = N = 0; that row's output is read as 0.
    """
    Qi = np.asarray(Qi, np.float64)
    sel_row = np.asarray(sel_row, bool)
    approx = np.nonzero(~sel_row)[0] if correction else np.zeros(0, dtype=np.int64)
    exact = np.nonzero(sel_row)[0]

    # Approximate terms: one pooled logit per unselected block and row.
    a = scale * (Qi @ Kbar[approx].T) if approx.size else np.zeros((Qi.shape[0], 0))
    # Exact terms: token logits of every selected block.
    xs = []
    vs = []
    for j in exact:
        s0, n = int(kgeom.starts[j]), int(kgeom.counts[j])
        xs.append(scale * (Qi @ Kh[s0:s0 + n].T))
        vs.append(Vh[s0:s0 + n])
    x = np.concatenate(xs, axis=1) if xs else np.zeros((Qi.shape[0], 0))
    vx = np.concatenate(vs, axis=0) if vs else np.zeros((0, Vh.shape[1]))

    if a.shape[1] + x.shape[1] == 0:
        return np.zeros((Qi.shape[0], Vh.shape[1]))
    m = np.max(np.concatenate([a, x], axis=1), axis=1, keepdims=True)
    ea = np.exp(a - m)
    ex = np.exp(x - m)
    n_approx = kgeom.counts[approx].astype(np.float64)
    D = (ea * n_approx[None, :]).sum(axis=1) + ex.sum(axis=1)       # Eq. 9
    N = ea @ Vhat[approx] + ex @ vx                                  # Eq. 10
    return N / D[:, None]


def forward_head(Qh, Kh, Vh, Bq: int, Bk: int, beta: float, sel=None, query_blocks=None,
                 correction: bool = True, moments: str = "eq5"):
    """One (batch, head): route (or take ``sel`` as given) and attend.

    Returns (out [L, d] with NaN in rows of blocks not requested, route dict).
    ``sel`` lets a caller substitute another implementation's decisions on
    near-tie pairs; ``query_blocks`` restricts the (expensive) attention step
    to a sample of query blocks.
    """
    Qh = np.asarray(Qh, np.float64)
    Kh = np.asarray(Kh, np.float64)
    Vh = np.asarray(Vh, np.float64)
    L, d = Qh.shape
    scale = 1.0 / math.sqrt(d)
    r = route_head(Qh, Kh, Bq, Bk, beta, moments)
    if sel is not None:
        sel = np.asarray(sel, bool)
        assert sel.shape == r["sel"].shape
        r["sel_used"] = sel
    else:
        r["sel_used"] = r["sel"]
    kg, qg = r["kgeom"], r["qgeom"]
    Vhat = pool_blocks(Vh, kg, "sum")
    out = np.full((L, Vh.shape[1]), np.nan)
    blocks = range(qg.n) if query_blocks is None else query_blocks
    for i in blocks:
        s0, n = int(qg.starts[i]), int(qg.counts[i])
        out[s0:s0 + n] = attend_query_block(Qh[s0:s0 + n], Kh, Vh, kg, r["Kbar"], Vhat, r["sel_used"][i], scale,
                                            correction)
    return out, r


def forward(Q, K, V, Bq: int, Bk: int, beta: float, correction: bool = True, moments: str = "eq5") -> np.ndarray:
    """Full forward over [batch, heads, L, d] inputs; float64 output
    (correction=False: the keep-or-drop baseline; moments: see route_head)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    out = np.empty_like(Q)
    for b in range(Q.shape[0]):
        for h in range(Q.shape[1]):
            out[b, h], _ = forward_head(Q[b, h], K[b, h], V[b, h], Bq, Bk, beta, correction=correction,
                                        moments=moments)
    return out


def stats(Q, K, Bq: int, Bk: int, beta: float, moments: str = "eq5"):
    """Selected-block counts |S_i| [b, H, Nq] and the selection [b, H, Nq, Nk]."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    counts = []
    sels = []
    for b in range(Q.shape[0]):
        cb, sb = [], []
        for h in range(Q.shape[1]):
            r = route_head(Q[b, h], K[b, h], Bq, Bk, beta, moments)
            cb.append(r["sel"].sum(axis=1))
            sb.append(r["sel"])
        counts.append(cb)
        sels.append(sb)
    return np.asarray(counts, np.int64), np.asarray(sels, bool)


def dense_attention(Q, K, V) -> np.ndarray:
    """Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V, the textbook
    definition quoted in the papers.ananclaw.com explainer; rows are shifted
    by their maximum before exponentiation.  Works on [..., L, d]."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    d = Q.shape[-1]
    logits = (Q @ np.swapaxes(K, -1, -2)) / math.sqrt(d)
    logits -= logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    return (w @ V) / w.sum(axis=-1, keepdims=True)
