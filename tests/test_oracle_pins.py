"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test checks an oracle function against a closed form, a library routine,
an invariant the pages state, a brute-force restatement in another form, or a
value the pages print.  A plausible slip in the oracle (dropped 1/sqrt(d),
dropped block weight n_j, mean instead of sum of V, sample instead of
population sigma, >= instead of >, transposed operand) fails at least one.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import sol_attn as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BETAS = (-math.inf, -0.5, 0.0, 0.5, 1.04, 2.0, math.inf)


def rng_qkv(seed, L, d, H=1, b=1):
    g = np.random.default_rng(seed)
    return (g.standard_normal((b, H, L, d)), g.standard_normal((b, H, L, d)), g.standard_normal((b, H, L, d)))


# ---------------------------------------------------------------- geometry / pooling

def test_block_geometry_ragged():
    g = O.block_geometry(1000, 128)
    assert g.n == 8
    assert list(g.counts) == [128] * 7 + [104]
    assert int(g.counts.sum()) == 1000
    g1 = O.block_geometry(1, 64)
    assert g1.n == 1 and int(g1.counts[0]) == 1


def test_pool_invariants():
    X = np.random.default_rng(0).standard_normal((37, 5))
    g = O.block_geometry(37, 8)
    mean = O.pool_blocks(X, g, "mean")
    total = O.pool_blocks(X, g, "sum")
    # count-weighted means and the block sums both give the column totals
    np.testing.assert_allclose((mean * g.counts[:, None]).sum(0), X.sum(0), rtol=1e-13)
    np.testing.assert_allclose(total.sum(0), X.sum(0), rtol=1e-13)
    # a block of identical rows pools to that row (mean) and n times it (sum)
    Y = np.repeat(np.arange(5.0)[None, :], 8, axis=0)
    gy = O.block_geometry(8, 8)
    np.testing.assert_array_equal(O.pool_blocks(Y, gy, "mean")[0], np.arange(5.0))
    np.testing.assert_array_equal(O.pool_blocks(Y, gy, "sum")[0], 8 * np.arange(5.0))


# ---------------------------------------------------------------- proxy scores, moments, threshold

def test_eq11_column_mean_of_token_tile_is_proxy_score():
    """Eq. 11: Mean over query tokens of Q_i K-bar^T equals Q-bar_i K-bar^T."""
    Q, K, _ = rng_qkv(1, 200, 16)
    Qh, Kh = Q[0, 0], K[0, 0]
    r = O.route_head(Qh, Kh, 32, 32, 1.0)
    scale = 1 / 4.0
    for i in range(r["qgeom"].n):
        s0, n = int(r["qgeom"].starts[i]), int(r["qgeom"].counts[i])
        tile = scale * Qh[s0:s0 + n] @ r["Kbar"].T
        np.testing.assert_allclose(tile.mean(axis=0), r["s"][i], rtol=1e-12, atol=1e-14)


def test_eq5_moments_match_two_pass_and_numpy():
    Q, K, _ = rng_qkv(2, 500, 32)
    Qh, Kh = Q[0, 0] + 0.3, K[0, 0] - 0.2  # non-zero means exercise the mu^2 term
    g = O.block_geometry(500, 16)
    Qbar, Kbar = O.pool_blocks(Qh, g, "mean"), O.pool_blocks(Kh, g, "mean")
    scale = 1 / math.sqrt(32)
    s = O.proxy_scores(Qbar, Kbar, scale)
    mu2, sd2 = O.row_moments(s)
    mu5, sd5 = O.eq5_moments(Qbar, Kbar, scale)
    np.testing.assert_allclose(mu5, mu2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sd5, sd2, rtol=1e-10)
    np.testing.assert_allclose(mu2, np.mean(s, axis=1), rtol=1e-13)
    np.testing.assert_allclose(sd2, np.std(s, axis=1, ddof=0), rtol=1e-12)


def test_selection_is_strict_and_uses_population_sigma():
    # [2, 0, 0, 0]: mu = 0.5, population sigma = sqrt(0.75); sample sigma = 1.
    s = np.array([[2.0, 0.0, 0.0, 0.0]])
    mu, sd = O.row_moments(s)
    assert mu[0] == 0.5 and abs(sd[0] - math.sqrt(0.75)) < 1e-15
    # beta = 1.6: tau = 1.886 (population) selects block 0; a sample sigma would not.
    assert O.select_blocks(s, O.threshold(mu, sd, 1.6)).tolist() == [[True, False, False, False]]
    # [1, 1, -1, -1] at beta = 1: tau = 1 exactly -> strict '>' keeps nothing.
    s2 = np.array([[1.0, 1.0, -1.0, -1.0]])
    mu2, sd2 = O.row_moments(s2)
    assert O.select_blocks(s2, O.threshold(mu2, sd2, 1.0)).sum() == 0
    # beta = 0: above-mean blocks only
    assert O.select_blocks(s2, O.threshold(mu2, sd2, 0.0)).tolist() == [[True, True, False, False]]
    # sigma = 0 and finite beta: nothing is strictly above the mean
    s3 = np.full((1, 5), 0.25)
    mu3, sd3 = O.row_moments(s3)
    assert O.select_blocks(s3, O.threshold(mu3, sd3, -3.0)).sum() == 0


def test_threshold_infinite_beta():
    mu = np.array([0.1, -2.0]); sd = np.array([0.0, 1.0])
    assert np.all(O.threshold(mu, sd, -math.inf) == -math.inf)
    assert np.all(O.threshold(mu, sd, math.inf) == math.inf)
    with pytest.raises(ValueError):
        O.threshold(mu, sd, float("nan"))


def test_gaussian_density_matches_printed_figure():
    """Scores of iid Gaussian vectors are near-Gaussian rows; Eq. 4 then keeps
    about 1 - Phi(beta) of each row: 15% at beta = 1.04 as the page prints."""
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))["density_at_beta"]
    g = np.random.default_rng(3)
    Qbar = g.standard_normal((256, 256))
    Kbar = g.standard_normal((1024, 256))
    s = O.proxy_scores(Qbar, Kbar, 1 / 16)
    mu, sd = O.row_moments(s)
    frac = O.select_blocks(s, O.threshold(mu, sd, facts["beta"])).mean()
    assert abs(100 * frac - facts["printed_density_percent"]) < facts["tolerance_percent"] + 0.2
    phi = 0.5 * (1 + math.erf(facts["beta"] / math.sqrt(2)))
    assert abs(frac - (1 - phi)) < 0.005


# ---------------------------------------------------------------- whole method, special cases

def test_dense_attention_matches_naive_loops():
    g = np.random.default_rng(4)
    L, d = 9, 3
    Q, K, V = g.standard_normal((L, d)), g.standard_normal((L, d)), g.standard_normal((L, d))
    out = O.dense_attention(Q, K, V)
    for t in range(L):
        w = [math.exp(sum(Q[t, c] * K[k, c] for c in range(d)) / math.sqrt(d)) for k in range(L)]
        z = sum(w)
        for c in range(d):
            assert abs(out[t, c] - sum(w[k] * V[k, c] for k in range(L)) / z) < 1e-12


def test_beta_minus_inf_is_dense_attention_sdpa():
    Q, K, V = rng_qkv(5, 100, 16, H=2, b=2)
    out = O.forward(Q, K, V, 16, 16, -math.inf)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V)).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(O.dense_attention(Q, K, V), ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("Bq", (16, 8, 32))
@pytest.mark.parametrize("beta", BETAS)
def test_identical_keys_per_block_give_dense_attention(beta, Bq):
    """Eqs. 9/10 replace every key of an unselected block by its mean; when the
    keys of each block are identical that is exact, so every beta gives dense
    attention (Q and V still vary token by token)."""
    g = np.random.default_rng(6)
    L, d, B = 70, 8, 16  # ragged tail of 6 tokens
    geom = O.block_geometry(L, B)
    Kblk = g.standard_normal((geom.n, d)) * 1.5
    K = np.concatenate([np.repeat(Kblk[j][None], geom.counts[j], 0) for j in range(geom.n)])
    Q = g.standard_normal((L, d)) * 1.5
    V = g.standard_normal((L, d))
    out, r = O.forward_head(Q, K, V, Bq, B, beta)
    np.testing.assert_allclose(out, O.dense_attention(Q, K, V), rtol=1e-11, atol=1e-12)


def test_beta_plus_inf_is_attention_over_pooled_keys_with_log_count_bias():
    """No block selected: each query attends to N virtual keys K-bar_j, each
    standing for n_j tokens (bias ln n_j) with value V-hat_j / n_j; computed
    here with the library SDPA and an additive mask."""
    Q, K, V = rng_qkv(7, 90, 16)  # blocks of 32: 32, 32, 26
    Qh, Kh, Vh = Q[0, 0], K[0, 0], V[0, 0]
    geom = O.block_geometry(90, 32)
    Kbar = np.stack([Kh[s:s + n].mean(0) for s, n in zip(geom.starts, geom.counts)])
    Vmean = np.stack([Vh[s:s + n].mean(0) for s, n in zip(geom.starts, geom.counts)])
    bias = np.log(geom.counts.astype(np.float64))[None, :].repeat(90, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Qh)[None], torch.from_numpy(Kbar)[None], torch.from_numpy(Vmean)[None],
        attn_mask=torch.from_numpy(bias)[None]).numpy()[0]
    out, r = O.forward_head(Qh, Kh, Vh, 32, 32, math.inf)
    assert r["sel"].sum() == 0
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("beta", (-1.0, 0.0, 1.04, math.inf))
def test_single_key_block_gives_mean_value(beta):
    """L <= Bk: one key block, sigma = 0, so it is approximate and every
    output row is the block's mean value ('Key consequence' after Eq. 10)."""
    Q, K, V = rng_qkv(8, 50, 8)
    out, r = O.forward_head(Q[0, 0], K[0, 0], V[0, 0], 16, 64, beta)
    assert r["sel"].sum() == 0
    np.testing.assert_allclose(out, np.repeat(V[0, 0].mean(0)[None], 50, 0), rtol=1e-12, atol=1e-13)


def test_key_block_permutation_invariance():
    Q, K, V = rng_qkv(9, 16 * 7 + 5, 8)
    Qh, Kh, Vh = Q[0, 0], K[0, 0], V[0, 0]
    B = 16
    perm = np.random.default_rng(10).permutation(7)  # full blocks only; tail stays last
    idx = np.concatenate([np.arange(p * B, p * B + B) for p in perm] + [np.arange(7 * B, 7 * B + 5)])
    for beta in (0.0, 0.7, 1.04):
        out1, r1 = O.forward_head(Qh, Kh, Vh, B, B, beta)
        out2, r2 = O.forward_head(Qh, Kh[idx], Vh[idx], B, B, beta)
        np.testing.assert_allclose(out1, out2, rtol=1e-11, atol=1e-12)
        full = np.concatenate([perm, [7]])
        np.testing.assert_array_equal(r1["sel"][:, full], r2["sel"])


def _brute_force_key_replacement(Q, K, V, Bq, Bk, beta):
    """Pure-Python restatement in the derivation's own terms: a query block
    keeps the original keys of its selected blocks and sees every key of an
    unselected block replaced by that block's mean key; values are untouched
    ('Limits and open questions': approximation replaces every key in an
    unselected block by its mean)."""
    L, d = len(Q), len(Q[0])
    scale = 1 / math.sqrt(d)
    nb = (L + Bk - 1) // Bk
    blocks = [list(range(b * Bk, min(L, b * Bk + Bk))) for b in range(nb)]
    qblocks = [list(range(b * Bq, min(L, b * Bq + Bq))) for b in range((L + Bq - 1) // Bq)]
    mean = lambda rows, X: [sum(X[r][c] for r in rows) / len(rows) for c in range(d)]
    Qb = [mean(bl, Q) for bl in qblocks]
    Kb = [mean(bl, K) for bl in blocks]
    out = [[0.0] * d for _ in range(L)]
    for i, qb in enumerate(qblocks):
        s = [scale * sum(Qb[i][c] * Kb[j][c] for c in range(d)) for j in range(nb)]
        mu = sum(s) / nb
        sd = math.sqrt(sum((x - mu) ** 2 for x in s) / nb)
        tau = -math.inf if beta == -math.inf else math.inf if beta == math.inf else mu + beta * sd
        keys = []
        for j, bl in enumerate(blocks):
            for k in bl:
                keys.append((K[k] if s[j] > tau else Kb[j], V[k]))
        for t in qb:
            logits = [scale * sum(Q[t][c] * kk[c] for c in range(d)) for kk, _ in keys]
            m = max(logits)
            w = [math.exp(x - m) for x in logits]
            z = sum(w)
            out[t] = [sum(wk * vv[c] for wk, (_, vv) in zip(w, keys)) / z for c in range(d)]
    return out


@pytest.mark.parametrize("Bq,Bk", ((4, 4), (3, 5), (6, 4)))  # key blocks 4,4,4,2 / 5,5,4
@pytest.mark.parametrize("beta", (-math.inf, 0.0, 0.5, 1.04, math.inf))
def test_bruteforce_key_replacement_tiny(beta, Bq, Bk):
    g = np.random.default_rng(11)
    L, d = 14, 3
    Q, K, V = g.standard_normal((L, d)) * 2, g.standard_normal((L, d)) * 2, g.standard_normal((L, d))
    ref = _brute_force_key_replacement(Q.tolist(), K.tolist(), V.tolist(), Bq, Bk, beta)
    out, _ = O.forward_head(Q, K, V, Bq, Bk, beta)
    np.testing.assert_allclose(out, np.array(ref), rtol=1e-12, atol=1e-13)


def test_selection_substitution_and_sampled_blocks():
    """forward_head with an explicit selection equals the default when given
    its own decisions, and a query-block sample reproduces those rows."""
    Q, K, V = rng_qkv(12, 200, 16)
    out, r = O.forward_head(Q[0, 0], K[0, 0], V[0, 0], 32, 32, 0.5)
    out2, _ = O.forward_head(Q[0, 0], K[0, 0], V[0, 0], 32, 32, 0.5, sel=r["sel"], query_blocks=[1, 6])
    np.testing.assert_array_equal(out[32:64], out2[32:64])
    np.testing.assert_array_equal(out[192:200], out2[192:200])
    assert np.isnan(out2[0:32]).all()


def test_stats_counts():
    Q, K, _ = rng_qkv(13, 130, 8, H=3, b=2)
    counts, sel = O.stats(Q, K, 32, 32, 0.3)
    assert counts.shape == (2, 3, 5) and sel.shape == (2, 3, 5, 5)
    np.testing.assert_array_equal(counts, sel.sum(-1))
    c_all, _ = O.stats(Q, K, 32, 32, -math.inf)
    assert np.all(c_all == 5)
    c_none, _ = O.stats(Q, K, 32, 32, math.inf)
    assert np.all(c_none == 0)


# ---------------------------------------------------------------- keep-or-drop baseline (correction off)

def test_keep_or_drop_all_selected_is_dense():
    Q, K, V = rng_qkv(14, 100, 16)
    out, _ = O.forward_head(Q[0, 0], K[0, 0], V[0, 0], 16, 16, -math.inf, correction=False)
    np.testing.assert_allclose(out, O.dense_attention(Q[0, 0], K[0, 0], V[0, 0]), rtol=1e-11, atol=1e-12)


def test_keep_or_drop_is_attention_over_selected_tokens_only():
    """Unselected blocks contribute zero: each query block attends (library
    SDPA) to the tokens of its selected blocks alone; nothing selected -> 0."""
    Q, K, V = rng_qkv(15, 90, 8)  # blocks of 16: 5 full + 10 tokens
    Qh, Kh, Vh = Q[0, 0], K[0, 0], V[0, 0]
    out, r = O.forward_head(Qh, Kh, Vh, 16, 16, 0.8, correction=False)
    geom = r["kgeom"]
    for i in range(r["qgeom"].n):
        s0, n = int(r["qgeom"].starts[i]), int(r["qgeom"].counts[i])
        keys = np.concatenate([np.arange(geom.starts[j], geom.starts[j] + geom.counts[j])
                               for j in np.nonzero(r["sel"][i])[0]] or [np.zeros(0, dtype=np.int64)])
        if keys.size == 0:
            np.testing.assert_array_equal(out[s0:s0 + n], 0.0)
            continue
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Qh[s0:s0 + n])[None], torch.from_numpy(Kh[keys])[None],
            torch.from_numpy(Vh[keys])[None]).numpy()[0]
        np.testing.assert_allclose(out[s0:s0 + n], ref, rtol=1e-11, atol=1e-12)
    out_inf, r_inf = O.forward_head(Qh, Kh, Vh, 16, 16, math.inf, correction=False)
    assert r_inf["sel"].sum() == 0 and np.all(out_inf == 0.0)


# ---------------------------------------------------------------- diagonal moment estimator (reading)

def test_diagonal_sigma_hand_example():
    """Two pooled keys (1, 0) and (3, 2): each channel has population variance 1
    and the channels are perfectly correlated (covariance 1).  Worked by hand:
    Q-bar = (1, 1): scores 1 and 5, row sigma 2; the diagonal drops the 2*1*1*1
    cross term, sigma^2 = 1 + 1 = 2.  Q-bar = (2, -1): scores 2 and 4, row
    sigma 1; diagonal sigma^2 = 4 * 1 + 1 * 1 = 5."""
    Kbar = np.array([[1.0, 0.0], [3.0, 2.0]])
    Qbar = np.array([[1.0, 1.0], [2.0, -1.0]])
    _, sd_row = O.row_moments(O.proxy_scores(Qbar, Kbar, 1.0))
    np.testing.assert_allclose(sd_row, [2.0, 1.0], rtol=1e-15)
    np.testing.assert_allclose(O.diagonal_sigma(Qbar, Kbar, 1.0), [math.sqrt(2.0), math.sqrt(5.0)], rtol=1e-15)
    np.testing.assert_allclose(O.diagonal_sigma(Qbar, Kbar, 0.5), [math.sqrt(2.0) / 2, math.sqrt(5.0) / 2],
                               rtol=1e-15)


def test_diagonal_sigma_equals_row_sigma_for_single_channel_queries():
    g = np.random.default_rng(21)
    Kbar = g.standard_normal((40, 8)) @ g.standard_normal((8, 8)) + 0.7  # correlated channels
    scale = 1 / math.sqrt(8)
    Qbar = np.zeros((8, 8))
    Qbar[np.arange(8), np.arange(8)] = g.standard_normal(8) * 3
    _, sd_row = O.row_moments(O.proxy_scores(Qbar, Kbar, scale))
    np.testing.assert_allclose(O.diagonal_sigma(Qbar, Kbar, scale), sd_row, rtol=1e-12)


def hadamard(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_diagonal_sigma_equals_row_sigma_for_uncorrelated_channels():
    """Columns 1..d of a Sylvester Hadamard matrix sum to zero and are mutually
    orthogonal, so pooled keys built from them have a diagonal covariance."""
    g = np.random.default_rng(22)
    N, d = 32, 12
    Kbar = 0.4 + hadamard(N)[:, 1:d + 1] * g.uniform(0.5, 2.0, d)[None, :]
    Qbar = g.standard_normal((20, d))
    scale = 1 / math.sqrt(d)
    _, sd_row = O.row_moments(O.proxy_scores(Qbar, Kbar, scale))
    np.testing.assert_allclose(O.diagonal_sigma(Qbar, Kbar, scale), sd_row, rtol=1e-12)


def test_diagonal_sigma_misses_exactly_the_off_diagonal_covariance():
    """Row variance - diagonal variance = scale^2 Q-bar (C - diag C) Q-bar^T with
    C the population covariance of the pooled keys (numpy.cov, bias=True)."""
    g = np.random.default_rng(23)
    Kbar = g.standard_normal((50, 6)) @ g.standard_normal((6, 6)) - 0.3
    Qbar = g.standard_normal((15, 6))
    scale = 0.37
    _, sd_row = O.row_moments(O.proxy_scores(Qbar, Kbar, scale))
    C = np.cov(Kbar.T, bias=True)
    off = C - np.diag(np.diag(C))
    gap = scale ** 2 * np.einsum("ic,ce,ie->i", Qbar, off, Qbar)
    np.testing.assert_allclose(sd_row ** 2 - O.diagonal_sigma(Qbar, Kbar, scale) ** 2, gap, atol=1e-12)


def test_diagonal_routing_matches_eq5_routing_when_channels_are_uncorrelated():
    """Keys constant inside each block with Hadamard-structured block means:
    both estimators give the same sigma, hence the same selection; on generic
    keys they differ somewhere."""
    g = np.random.default_rng(24)
    N, B, d = 16, 8, 8
    kb = 0.2 + hadamard(N)[:, 1:d + 1] * g.uniform(0.5, 1.5, d)[None, :]
    K = np.repeat(kb, B, axis=0)[: N * B - 3]   # ragged tail block keeps the same mean
    Q = g.standard_normal((K.shape[0], d))
    for beta in (-math.inf, -0.5, 0.5, 1.04, math.inf):
        a = O.route_head(Q, K, B, B, beta, "eq5")
        b = O.route_head(Q, K, B, B, beta, "diagonal")
        np.testing.assert_allclose(a["sigma"], b["sigma"], rtol=1e-12)
        assert np.all(np.abs(a["s"] - a["tau"][:, None]) > 1e-9) or not np.isfinite(beta)
        assert np.array_equal(a["sel"], b["sel"])
    Kg = g.standard_normal((N * B, d)) @ g.standard_normal((d, d))
    a = O.route_head(Q[: N * B - 3], Kg[: N * B - 3], B, B, 1.04, "eq5")
    b = O.route_head(Q[: N * B - 3], Kg[: N * B - 3], B, B, 1.04, "diagonal")
    assert not np.allclose(a["sigma"], b["sigma"])
    with pytest.raises(ValueError):
        O.route_head(Q, K, B, B, 1.0, "full")
