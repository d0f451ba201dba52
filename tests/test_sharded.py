"""One call split across ranks by heads (video_diffusion_b200.sharded), on
CPU ranks with gloo: the token -> head re-layout, each rank's share computed
by the float64 oracle (injected as the per-rank attention), the re-layout
back, against the single-rank oracle on the whole tensors.  The exchanges
only move data and the heads are independent, so the result must be equal
bit for bit, for world sizes 2 and 4, with heads and tokens that do not
divide evenly."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from video_diffusion_b200 import sharded as S

B, H, L, D, BLOCK, BETA = 1, 5, 301, 16, 64, 0.5


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = torch.Generator().manual_seed(7)
    base = torch.randn(B, H, L, D, generator=g, dtype=torch.float64)
    q = base + 0.5 * torch.randn(B, H, L, D, generator=g, dtype=torch.float64)
    k = base + 0.5 * torch.randn(B, H, L, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, L, D, generator=g, dtype=torch.float64)
    return q, k, v


def _oracle_attend(q, k, v, beta, block):
    from oracle import sol_attn as O
    out = O.forward(q.numpy(), k.numpy(), v.numpy(), block, block, beta)
    return torch.from_numpy(np.ascontiguousarray(out))


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = _inputs()
        # sequence-parallel layout: this rank's tokens of every head
        qs, ks, vs = (S.shard_tokens(t, world, rank).contiguous() for t in (q, k, v))
        o_seq = S.forward_ulysses(qs, ks, vs, BETA, H, L, BLOCK, attend=_oracle_attend)
        parts = [None] * world  # uneven shares: gathered as objects
        dist.all_gather_object(parts, o_seq.numpy())
        ulysses = torch.cat([torch.from_numpy(x) for x in parts], dim=2)
        # head-split layout: this rank's heads of every token, no exchange
        o_head = S.forward_heads(*(S.shard_heads(t, world, rank).contiguous() for t in (q, k, v)), BETA, BLOCK,
                                 attend=_oracle_attend)
        hparts = [None] * world
        dist.all_gather_object(hparts, o_head.numpy())
        heads = torch.cat([torch.from_numpy(x) for x in hparts], dim=1)
        results[rank] = ("ok", ulysses.numpy(), heads.numpy())
    except Exception as e:  # noqa: BLE001
        results[rank] = ("error", f"{type(e).__name__}: {e}"[:300], None)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_split_call_equals_single_rank_oracle(world):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert not p.is_alive(), "rank hung"
    q, k, v = _inputs()
    ref = _oracle_attend(q, k, v, BETA, BLOCK).numpy()
    for r in range(world):
        status, ulysses, heads = results[r]
        assert status == "ok", ulysses
        np.testing.assert_array_equal(ulysses, ref)
        np.testing.assert_array_equal(heads, ref)


def test_split_ranges_and_exchange_bytes():
    assert [S.split_range(10, 4, r) for r in range(4)] == [(0, 3), (3, 6), (6, 8), (8, 10)]
    assert S.split_sizes(5, 2) == [3, 2] and S.split_sizes(3, 4) == [1, 1, 1, 0]
    assert sum(S.split_sizes(75600, 8)) == 75600
    with pytest.raises(ValueError):
        S.split_range(10, 4, 4)
    # Wan 720p on 8 ranks: each rank sends 7/8 of its 1/8 token share of one
    # 774 MB bf16 tensor per exchange
    n = S.exchange_bytes((1, 40, 75600, 128), 2, 8, 0)
    assert n == 1 * 35 * 9450 * 128 * 2
    # a rank with no heads sends nothing for itself and receives an empty share
    x = torch.zeros(1, 3, 8, 4)
    assert S.shard_heads(x, 4, 3).shape == (1, 0, 8, 4)
    assert S.forward_heads(S.shard_heads(x, 4, 3), S.shard_heads(x, 4, 3), S.shard_heads(x, 4, 3), 1.0,
                           attend=None).shape == (1, 0, 8, 4)
