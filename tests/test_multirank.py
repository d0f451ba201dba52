"""Host test of the N > 1 path (gloo, world size 2, CPU): each rank runs an
independent replica (own seed), the job time is the max over ranks, and the
aggregate value counts every rank's call.  Also a rank that fails before the
reduction makes the other rank's collective end in an error, not a wait."""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results, fail_rank):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    from oracle import sol_attn as O
    from video_diffusion_b200 import inputs as I

    w, r, _ = bench.rank_info()
    assert (w, r) == (world, rank)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=20))
    try:
        wl = I.WORKLOADS["tiny-fp32"]
        Q, K, V = I.make_workload(wl, device="cpu", seed_offset=rank)
        out = O.forward(Q.double().numpy(), K.double().numpy(), V.double().numpy(), wl.block, wl.block, 1.04)
        checksum = torch.tensor([float(np.abs(out).sum())], dtype=torch.float64)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, checksum)
        if rank == fail_rank:
            raise RuntimeError("rank leaves before the reduction")
        my_ms = 10.0 + rank  # stand-in per-rank time
        ms = bench.reduce_max(my_ms, dist, "cpu")
        value = bench.aggregate_value(world, wl.dense_flops(), ms)
        results[rank] = ("ok", ms, value, [float(s) for s in sums])
    except Exception as e:  # noqa: BLE001
        results[rank] = ("error", type(e).__name__, str(e)[:200], None)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def _run(world, fail_rank=-1):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results, fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert not p.is_alive(), "rank hung"
    return dict(results)


def test_two_ranks_replicas_and_max_time():
    res = _run(2)
    assert res[0][0] == "ok" and res[1][0] == "ok", res
    # max over ranks seen by both
    assert res[0][1] == res[1][1] == 11.0
    from video_diffusion_b200 import inputs as I
    flops = I.WORKLOADS["tiny-fp32"].dense_flops()
    assert math.isclose(res[0][2], 2 * flops / 11e-3 / 1e12)
    # replicas are independent: different seeds give different outputs
    s0, s1 = res[0][3]
    assert s0 != s1


def test_failed_rank_ends_peer_collective_with_error():
    res = _run(2, fail_rank=1)
    assert res[1][0] == "error"
    assert res[0][0] == "error", res  # the survivor's all-reduce errors out instead of waiting forever
