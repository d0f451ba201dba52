"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle.

Selections must match the oracle's exactly except near-ties; outputs are
compared element by element against the oracle run with the GPU's selection
(which differs from its own only on near-ties).  Small cases are compared on
every row; the full-size video workloads on every selection row and on a
seeded sample of query blocks (first, last, max- and min-count, text blocks).
"""

import math

import numpy as np
import pytest
import torch

from oracle import sol_attn as O
from tests import parity_helpers as P
from video_diffusion_b200 import api, build
from video_diffusion_b200 import inputs as I

pytestmark = pytest.mark.gpu
INF = math.inf


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    api.lib()
    yield
    assert api.device_status() == 0


def gpu_run(Q, K, V, block, beta, diagonal=False):
    out = torch.full_like(Q, float("nan"))
    api.forward_ex(Q, K, V, beta, block, out=out, diagonal_sigma=diagonal)
    counts, sel = api.stats(Q, K, beta, block, with_mask=True, diagonal_sigma=diagonal)
    torch.cuda.synchronize()
    return out, counts.cpu().numpy(), sel.cpu().numpy()


def check_case(Q, K, V, block, beta, sample_k=None, extra_blocks=(), seed=0, heads=None, diagonal=False):
    """Runs the GPU forward + stats and checks them against the oracle."""
    b_, H, L, d = Q.shape
    bq, bk = P.pair(block)
    moments = "diagonal" if diagonal else "eq5"
    out, counts, sel = gpu_run(Q, K, V, block, beta, diagonal)
    rng = np.random.default_rng(seed)
    stats = []
    gpu_rows, ref_rows = [], []
    for b in range(b_):
        for h in range(H) if heads is None else heads:
            r = O.route_head(P.head_np(Q, b, h), P.head_np(K, b, h), bq, bk, beta, moments)
            stats.append(P.compare_selection(r, sel[b, h], counts[b, h]))
            N = r["qgeom"].n
            if sample_k is None:
                blocks = list(range(N))
            else:
                blocks = P.sample_blocks(N, counts[b, h], sample_k, rng, extra_blocks)
            ref = P.oracle_rows(Q, K, V, b, h, block, beta, sel[b, h], blocks, moments)
            rows = P.rows_of(blocks, block, L)
            ref_rows.append(ref[rows])
            gpu_rows.append(out[b, h].double().cpu().numpy()[rows])
    assert not torch.isnan(out).any(), "output rows left unwritten"
    err = P.check_close(np.concatenate(gpu_rows), np.concatenate(ref_rows), Q.dtype, f"beta={beta}")
    return err, stats


# ------------------------------------------------------------------ small cases, every row

@pytest.mark.parametrize("beta", [-INF, -1.0, 0.0, 0.5, 1.04, 2.0, INF])
def test_bf16_ragged_full_rows(beta):
    # L = 1000: 7 full blocks and a 104-token tail; several tiles per query block
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=7, batch=2, device="cuda")
    check_case(Q, K, V, 128, beta)


@pytest.mark.parametrize("beta", [-INF, 0.5, 1.04, INF])
def test_tiny_fp32_workload(beta):
    wl = I.WORKLOADS["tiny-fp32"]
    Q, K, V = I.make_workload(wl, device="cuda")
    err, stats = check_case(Q, K, V, wl.block, beta)
    assert err["rel_l2"] <= 1e-4


@pytest.mark.parametrize("L", [1, 5, 127, 128, 129, 300])
@pytest.mark.parametrize("block", [128, (128, 64), 64, (64, 128)])
@pytest.mark.parametrize("beta", [-INF, 1.04, INF])
def test_short_and_ragged_lengths(L, beta, block):
    # with 64-token query blocks L = 1, 129 and 300 leave an odd block count:
    # the last 128-row tile holds one query block
    Q, K, V = I.make_iid(1, 3, L, 128, seed=L, dtype=torch.bfloat16, device="cuda")
    check_case(Q, K, V, block, beta)


@pytest.mark.parametrize("d,block,dtype", [(128, 128, torch.float32), (64, 64, torch.bfloat16),
                                           (64, 128, torch.bfloat16), (128, 64, torch.bfloat16),
                                           (64, 64, torch.float32)])
def test_other_shapes(d, block, dtype):
    Q, K, V = I.make_qkv((3, 12, 20), heads=2, d=d, seed=11, dtype=dtype, device="cuda")  # L = 720
    for beta in (-INF, 0.7, INF):
        check_case(Q, K, V, block, beta)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bq,bk", [(128, 64), (64, 128)])
@pytest.mark.parametrize("d", [64, 128])
def test_query_and_key_blocks_of_different_sizes(bq, bk, d, dtype):
    # L = 1000: ragged query and key tails of different lengths (104/40 tokens)
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=d, seed=12, dtype=dtype, device="cuda")
    for beta in (-INF, 0.5, 1.04, INF):
        err, _ = check_case(Q, K, V, (bq, bk), beta)
        if dtype == torch.float32:
            assert err["rel_l2"] <= 1e-4


@pytest.mark.parametrize("block", [128, 64, (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_diagonal_sigma(block, dtype):
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=13, dtype=dtype, device="cuda")
    for beta in (-1.0, 0.5, 1.04, 2.0):
        check_case(Q, K, V, block, beta, diagonal=True)


def test_diagonal_sigma_video_workload():
    """Wan2.1 480p shape: every selection row against the oracle's diagonal
    routing; sampled output rows; the selected fraction moves with the
    estimator but stays in the same range."""
    wl = I.WORKLOADS["wan-480p"]
    Q, K, V = I.make_workload(wl, device="cuda")
    out, counts, sel = gpu_run(Q, K, V, wl.block, 1.04, diagonal=True)
    rng = np.random.default_rng(4)
    gpu_rows, ref_rows = [], []
    for h in range(wl.heads):
        r = O.route_head(P.head_np(Q, 0, h), P.head_np(K, 0, h), wl.block, wl.block, 1.04, "diagonal")
        P.compare_selection(r, sel[0, h], counts[0, h])
        if h in (0, wl.heads - 1):
            blocks = P.sample_blocks(wl.n_blocks, counts[0, h], 8, rng)
            ref = P.oracle_rows(Q, K, V, 0, h, wl.block, 1.04, sel[0, h], blocks, "diagonal")
            rows = P.rows_of(blocks, wl.block, wl.L)
            ref_rows.append(ref[rows])
            gpu_rows.append(out[0, h].double().cpu().numpy()[rows])
    P.check_close(np.concatenate(gpu_rows), np.concatenate(ref_rows), Q.dtype, "wan-480p diagonal")
    assert 0.02 < sel.mean() < 0.40


@pytest.mark.parametrize("beta", [-INF, 0.0, 1.04, INF])
def test_identical_keys_per_block_equal_dense(beta):
    """Keys constant inside each block: every beta gives dense attention."""
    Q, K, V = I.make_iid(1, 2, 900, 128, seed=3, dtype=torch.float32, device="cuda")
    N = -(-900 // 128)
    Kb = torch.randn(1, 2, N, 128, device="cuda", generator=torch.Generator("cuda").manual_seed(5))
    K = Kb.repeat_interleave(128, dim=2)[:, :, :900].contiguous()
    Q, K, V = (t.to(torch.bfloat16).contiguous() for t in (Q, K, V))
    out = api.forward(Q, K, V, beta, 128)
    ref = O.dense_attention(Q.double().cpu().numpy(), K.double().cpu().numpy(), V.double().cpu().numpy())
    P.check_close(out.double().cpu().numpy(), ref, torch.bfloat16, "identical keys")


def test_deterministic_and_stream_ordered():
    Q, K, V = I.make_qkv((6, 16, 16), heads=4, d=128, seed=9, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = api.forward(Q, K, V, 1.04)
        b = api.forward(Q, K, V, 1.04)
    s.synchronize()
    assert torch.equal(a, b)


def test_invalid_arguments_raise():
    Q, K, V = I.make_iid(1, 1, 256, 96, seed=1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.SolAttnError):
        api.forward(Q, K, V, 1.0)
    Q, K, V = I.make_iid(1, 1, 256, 128, seed=1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.SolAttnError):
        api.forward(Q, K, V, float("nan"))


# ------------------------------------------------------------------ workloads at full size

@pytest.mark.parametrize("beta", [0.5, 1.04, 1.5])
@pytest.mark.parametrize("name,bk", [("image-dit", 128), ("image-dit-d64", 128), ("image-dit-d64", 64)])
def test_image_dit(beta, name, bk):
    """The image-DiT workloads (24 heads, L = 16384) on every output row: the
    oracle takes about half a second per head here."""
    wl = I.WORKLOADS[name]
    Q, K, V = I.make_workload(wl, device="cuda")
    check_case(Q, K, V, (wl.block, bk), beta)


@pytest.mark.parametrize("beta", [-INF, 1.04])
@pytest.mark.parametrize("name,bk", [("image-dit", 128), ("image-dit", 64), ("image-dit-d64", 64)])
def test_image_dit_query_blocks_of_64(beta, name, bk):
    """The image-DiT tensors routed in 64-token query blocks (two to a
    128-row tile on the tensor cores), every output row."""
    wl = I.WORKLOADS[name]
    Q, K, V = I.make_workload(wl, device="cuda")
    check_case(Q, K, V, (64, bk), beta)


@pytest.mark.parametrize("name,beta,bk", [("wan-480p", 1.04, 128),
                                          ("wan-720p", -INF, 128), ("wan-720p", 0.5, 128), ("wan-720p", 1.04, 128),
                                          ("wan-720p", 1.5, 128), ("wan-720p", 2.0, 128),
                                          ("hunyuan-720p", 1.04, 128), ("hunyuan-720p", 1.5, 128),
                                          # key blocks of 64 tokens, two per tensor-core tile
                                          ("wan-480p", 1.04, 64), ("wan-720p", 1.04, 64), ("wan-720p", -INF, 64),
                                          ("hunyuan-720p", 1.04, 64)])
def test_video_workloads(name, beta, bk):
    wl = I.WORKLOADS[name]
    block = (wl.block, bk)
    Q, K, V = I.make_workload(wl, device="cuda")
    out, counts, sel = gpu_run(Q, K, V, block, beta)
    assert not torch.isnan(out).any()
    rng = np.random.default_rng(2)
    N = wl.n_blocks
    text_blocks = ()
    if wl.text_tokens:
        first_text = (wl.L - wl.text_tokens) // wl.block
        text_blocks = tuple(range(first_text, N))
    sample_heads = [0, wl.heads // 2, wl.heads - 1]
    gpu_rows, ref_rows = [], []
    for h in range(wl.heads):
        Qh, Kh = P.head_np(Q, 0, h), P.head_np(K, 0, h)
        r = O.route_head(Qh, Kh, wl.block, bk, beta)
        P.compare_selection(r, sel[0, h], counts[0, h])
        if h in sample_heads:
            k = 12 if beta != -INF else 4
            blocks = P.sample_blocks(N, counts[0, h], k, rng, text_blocks)
            ref = P.oracle_rows(Q, K, V, 0, h, block, beta, sel[0, h], blocks)
            rows = P.rows_of(blocks, wl.block, wl.L)
            ref_rows.append(ref[rows])
            gpu_rows.append(out[0, h].double().cpu().numpy()[rows])
    P.check_close(np.concatenate(gpu_rows), np.concatenate(ref_rows), Q.dtype, f"{name} beta={beta}")
    if beta == 1.04:
        frac = sel.mean()
        assert 0.05 < frac < 0.30, frac


# ------------------------------------------------------------------ many key blocks per head

@pytest.mark.parametrize("grid,d,bk,diagonal", [
    ((15, 100, 128), 128, 64, False),   # L = 192000, Nk = 3000: route_kernel, 8 score rows per CTA
    ((15, 100, 128), 128, 64, True),
    ((31, 100, 128), 64, 128, False),   # L = 396800, Nk = 3100 at d = 64: route_kernel
    ((10, 100, 128), 128, 64, False),   # L = 128000, Nk = 2000: the register-blocked router
    ((10, 100, 128), 128, 64, True),
])
def test_many_key_blocks(grid, d, bk, diagonal):
    """Heads with more pooled keys than the register-blocked router's score
    rows hold go through route_kernel; both must select what the oracle
    selects, and the attention kernel must handle the long selection rows."""
    Q, K, V = I.make_qkv(grid, heads=1, d=d, seed=41, device="cuda")
    check_case(Q, K, V, (128, bk), 1.04, sample_k=4, seed=3, diagonal=diagonal)


def test_query_block_pairs_with_long_selection_rows():
    """64-token query and key blocks with more than 64 mask words per row
    (L = 192000: Nq = Nk = 3000, 94 words): the producer counts a pair's
    union tiles by walking the rows from global memory instead of from
    registers; outputs match the oracle and the per-CTA record adds up to the
    union tiles."""
    Q, K, V = I.make_qkv((15, 100, 128), heads=1, d=128, seed=43, device="cuda")
    check_case(Q, K, V, (64, 64), 1.04, sample_k=4, seed=5)
    api.forward(Q, K, V, 1.04, (64, 64))
    rows = api.cta_times()
    counts, sel = api.stats(Q, K, 1.04, (64, 64), with_mask=True)
    sel = sel.cpu().numpy()[0, 0]
    Nq, Nk = sel.shape
    assert -(-Nk // 32) > 64
    a, b = sel[0::2], sel[1::2]
    if b.shape[0] < a.shape[0]:
        b = np.concatenate([b, a[-1:]])  # a lone last block pairs with itself
    union = a | b
    unsel = ~(a & b)
    chunks = -(-Nk // 128)
    unsel_chunks = sum(int(unsel[:, c * 128:(c + 1) * 128].any(axis=-1).sum()) for c in range(chunks))
    exact_tiles = int(((union.sum(axis=-1) + 1) // 2).sum())  # two 64-token key blocks per tile
    assert rows[:, 2].sum() == a.shape[0]
    assert rows[:, 3].sum() == exact_tiles + unsel_chunks


@pytest.mark.parametrize("d", [128, 64])
def test_largest_supported_key_block_count(d):
    """Nk = 6144, the most pooled keys per head the library accepts (L = 393216
    tokens in 64-token key blocks); one more block is rejected on the host."""
    Q, K, V = I.make_qkv((24, 128, 128), heads=1, d=d, seed=42, device="cuda")
    assert Q.shape[2] == 64 * 6144
    check_case(Q, K, V, (128, 64), 1.04, sample_k=3, seed=4)
    Q2 = torch.empty(1, 1, 64 * 6144 + 1, d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.SolAttnError):
        api.forward(Q2, Q2, Q2, 1.04, (128, 64))


# ------------------------------------------------------------------ keep-or-drop (correction off)

def check_keep_or_drop(Q, K, V, block, beta):
    bq, bk = P.pair(block)
    out = torch.full_like(Q, float("nan"))
    api.forward_ex(Q, K, V, beta, block, out=out, keep_or_drop=True)
    counts, sel = api.stats(Q, K, beta, block, with_mask=True)
    torch.cuda.synchronize()
    sel = sel.cpu().numpy()
    counts = counts.cpu().numpy()
    gpu_rows, ref_rows = [], []
    for b in range(Q.shape[0]):
        for h in range(Q.shape[1]):
            r = O.route_head(P.head_np(Q, b, h), P.head_np(K, b, h), bq, bk, beta)
            P.compare_selection(r, sel[b, h], counts[b, h])
            ref, _ = O.forward_head(P.head_np(Q, b, h), P.head_np(K, b, h), P.head_np(V, b, h), bq, bk,
                                    beta, sel=sel[b, h], correction=False)
            ref_rows.append(ref)
            gpu_rows.append(out[b, h].double().cpu().numpy())
    assert not torch.isnan(out).any()
    return P.check_close(np.concatenate(gpu_rows), np.concatenate(ref_rows), Q.dtype, f"keep-or-drop beta={beta}")


@pytest.mark.parametrize("block", [128, (128, 64), 64, (64, 128)])
@pytest.mark.parametrize("beta", [-INF, 0.5, 1.04, 2.0, INF])
def test_keep_or_drop_bf16(beta, block):
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=8, device="cuda")  # L = 1000, ragged tail
    check_keep_or_drop(Q, K, V, block, beta)


@pytest.mark.parametrize("block", [64, (64, 128)])
@pytest.mark.parametrize("beta", [0.5, 1.04])
def test_keep_or_drop_pair_with_an_empty_block(beta, block):
    """Query block 0's rows are 0, so its pooled query is exactly 0 (in any
    summation order), all its proxy scores are 0, sigma is 0 and Eq. 4's
    strict comparison selects nothing: without the correction its rows are 0,
    while block 1, which shares its 128-row tile, attends to its own
    selection."""
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=9, device="cuda")  # L = 1000
    Q[:, :, :64] = 0
    counts = api.stats(Q, K, beta, block)
    assert (counts[:, :, 0] == 0).all() and (counts[:, :, 1] > 0).all()
    err = check_keep_or_drop(Q, K, V, block, beta)
    out = api.forward_ex(Q, K, V, beta, block, keep_or_drop=True)
    assert (out[:, :, :64] == 0).all()
    check_case(Q, K, V, block, beta)  # with the correction block 0 takes the pooled path


@pytest.mark.parametrize("beta", [0.5, 1.04, INF])
def test_keep_or_drop_fp32(beta):
    wl = I.WORKLOADS["tiny-fp32"]
    Q, K, V = I.make_workload(wl, device="cuda")
    check_keep_or_drop(Q, K, V, wl.block, beta)


# ------------------------------------------------------------------ routing inside the attention kernel

@pytest.mark.parametrize("name,bk,beta", [("wan-480p", 128, 1.04), ("wan-480p", 64, 1.04), ("image-dit", 128, 0.5),
                                          ("image-dit-d64", 128, 1.5), ("hunyuan-720p", 64, 1.04),
                                          ("wan-720p", 128, -INF), ("wan-720p", 128, INF)])
def test_route_in_kernel_is_bit_identical(name, bk, beta):
    """The attention kernel's own Eq. 4 decisions (router arithmetic on the
    fp32 pooled vectors) select exactly the router's blocks, so the output is
    the same bits as with the router's mask."""
    wl = I.WORKLOADS[name]
    Q, K, V = I.make_workload(wl, device="cuda")
    a = api.forward_ex(Q, K, V, beta, (wl.block, bk))
    b = api.forward_ex(Q, K, V, beta, (wl.block, bk), route_in_kernel=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("block", [128, (128, 64)])
@pytest.mark.parametrize("beta", [-INF, 0.5, 1.04, INF])
def test_route_in_kernel_against_oracle(block, beta):
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=14, device="cuda")  # ragged L = 1000
    out = torch.full_like(Q, float("nan"))
    api.forward_ex(Q, K, V, beta, block, out=out, route_in_kernel=True)
    counts, sel = api.stats(Q, K, beta, block, with_mask=True)
    torch.cuda.synchronize()
    sel, counts = sel.cpu().numpy(), counts.cpu().numpy()
    bq, bk = P.pair(block)
    gpu_rows, ref_rows = [], []
    for h in range(2):
        r = O.route_head(P.head_np(Q, 0, h), P.head_np(K, 0, h), bq, bk, beta)
        P.compare_selection(r, sel[0, h], counts[0, h])
        ref_rows.append(P.oracle_rows(Q, K, V, 0, h, block, beta, sel[0, h], list(range(r["qgeom"].n))))
        gpu_rows.append(out[0, h].double().cpu().numpy())
    assert not torch.isnan(out).any()
    P.check_close(np.concatenate(gpu_rows), np.concatenate(ref_rows), torch.bfloat16, "route in kernel")


def test_route_in_kernel_with_keep_or_drop_and_diagonal_sigma():
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=128, seed=15, device="cuda")
    for kw in (dict(keep_or_drop=True), dict(diagonal_sigma=True), dict(keep_or_drop=True, diagonal_sigma=True)):
        a = api.forward_ex(Q, K, V, 1.04, 128, **kw)
        b = api.forward_ex(Q, K, V, 1.04, 128, route_in_kernel=True, **kw)
        torch.cuda.synchronize()
        assert torch.equal(a, b), kw


@pytest.mark.parametrize("d", [128, 64])
def test_output_aligned_to_16_bytes_only(d):
    """The kernel writes rows with 32-byte stores when the output allows it;
    a 16-byte-aligned (not 32-byte-aligned) output takes the 16-byte stores
    and gives the same bits."""
    Q, K, V = I.make_qkv((10, 10, 10), heads=2, d=d, seed=24, device="cuda")
    ref = api.forward(Q, K, V, 1.04, 128)
    buf = torch.empty(Q.numel() + 8, dtype=Q.dtype, device="cuda")
    out = buf[8:].view(Q.shape)  # 16 bytes past a 256-byte boundary
    assert out.data_ptr() % 32 == 16
    api.forward(Q, K, V, 1.04, 128, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


# ------------------------------------------------------------------ near-tie diagnostic

@pytest.mark.parametrize("name,beta,margin", [("image-dit", 1.04, 1e-3), ("wan-480p", 0.5, 1e-2),
                                              ("wan-480p", 1.04, 1e-3)])
def test_near_tie_counts_match_the_oracle(name, beta, margin):
    """sol_attn_near_ties counts, per query block, the key blocks whose proxy
    score lies within `margin` of tau_i.  The GPU's scores and thresholds are
    fp32 and the oracle's fp64, so a pair right at the margin may fall either
    way: the count must lie between the oracle's counts at margin -/+ 1e-4."""
    wl = I.WORKLOADS[name]
    Q, K, V = I.make_workload(wl, device="cuda")
    near = api.near_ties(Q, K, beta, wl.block, margin=margin).cpu().numpy()
    assert near.shape == (1, wl.heads, wl.n_blocks)
    total = 0
    for h in (0, wl.heads // 2, wl.heads - 1):
        r = O.route_head(P.head_np(Q, 0, h), P.head_np(K, 0, h), wl.block, wl.block, beta)
        gap = np.abs(r["s"] - r["tau"][:, None])
        lo = (gap < margin - 1e-4).sum(axis=1)
        hi = (gap < margin + 1e-4).sum(axis=1)
        assert np.all(lo <= near[0, h]) and np.all(near[0, h] <= hi), h
        total += int(near[0, h].sum())
    assert total > 0  # the margins above catch some pairs on these workloads
    for b in (-INF, INF):
        assert not api.near_ties(Q, K, b, wl.block, margin=margin).any()


def test_cta_times_for_query_block_pairs():
    """With 64-token query blocks a work item is the pair of blocks 2t and
    2t + 1 (one 128-row tile): the items add up to heads x ceil(Nq / 2) and
    the tiles to the union of each pair's selected blocks plus the chunks
    that hold a block unselected by either."""
    Q, K, V = I.make_qkv((10, 10, 10), heads=3, d=128, seed=10, device="cuda")  # L = 1000, Nq = 16
    Q2, K2, V2 = Q[:, :, :936], K[:, :, :936], V[:, :, :936]  # L = 936: Nq = 15, the last pair is one block
    for q, k, v in ((Q, K, V), (Q2.contiguous(), K2.contiguous(), V2.contiguous())):
        api.forward(q, k, v, 1.04, (64, 128))
        rows = api.cta_times()
        counts, sel = api.stats(q, k, 1.04, (64, 128), with_mask=True)
        sel = sel.cpu().numpy()[0]
        H, Nq, Nk = sel.shape
        npair = (Nq + 1) // 2
        assert rows[:, 2].sum() == H * npair
        tiles = 0
        for t in range(npair):
            rows_t = sel[:, 2 * t:2 * t + 2]
            union = rows_t.any(axis=1)
            unsel_any = (~rows_t).any(axis=1)
            tiles += int(union.sum()) + int(sum(unsel_any[:, c * 128:(c + 1) * 128].any(axis=-1).sum()
                                                for c in range(-(-Nk // 128))))
        assert rows[:, 3].sum() == tiles


def test_cta_times_account_for_every_item_and_tile():
    """The per-CTA record of an attention launch covers the whole call: the
    CTAs' item counts add up to batch x heads x Nq and their tile counts to
    the selected blocks plus the pooled-key chunks that hold an unselected
    block, per query block."""
    wl = I.WORKLOADS["wan-480p"]
    Q, K, V = I.make_workload(wl, device="cuda")
    api.forward(Q, K, V, 1.04, wl.block)
    rows = api.cta_times()
    counts, sel = api.stats(Q, K, 1.04, wl.block, with_mask=True)
    sel = sel.cpu().numpy()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    nitems = wl.heads * wl.n_blocks
    assert len(rows) == min(n_sm, nitems)
    assert np.all(rows[:, 1] > rows[:, 0])
    assert rows[:, 2].sum() == nitems
    Nk = sel.shape[-1]
    chunks = -(-Nk // 128)
    unsel_chunks = sum(((~sel[..., c * 128:(c + 1) * 128]).any(axis=-1)).sum() for c in range(chunks))
    assert rows[:, 3].sum() == int(sel.sum()) + int(unsel_chunks)
    lb = api.load_balance(rows)
    assert 1.0 <= lb["busy_max_over_mean"] < 1.5 and 0.0 <= lb["tail_idle_fraction"] < 0.5
