"""Host-side pieces of bench.py that need no GPU: the profile lookup that
fills roofline.traffic, and the executed-FLOP count the roofline divides."""

import argparse
import json
import os

import numpy as np

import bench
from video_diffusion_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _args(**kw):
    a = dict(workload="wan-720p", beta=1.04, block_k=None, block_q=None)
    a.update(kw)
    return argparse.Namespace(**a)


def test_default_workload_has_a_dram_profile_found_by_its_key():
    """The default bench line looks up the DRAM capture of its own workload:
    the key must name the committed JSON record, which must parse (its
    number is used while the kernel sources are unchanged)."""
    wl = I.WORKLOADS["wan-720p"]
    key = bench.workload_key(wl, _args())
    assert key == "wan-720p_beta1.04"
    path = os.path.join(ROOT, "profiles", f"attn_tc_kernel__{key}_dram.json")
    assert os.path.exists(path)
    rec = json.load(open(path))
    assert rec["workload"] == "wan-720p" and rec["beta"] == 1.04
    assert "ncu" in rec["command"] and "--clock-control none" in rec["command"]
    # about the algorithmic bytes of one launch: Q, K, V read and O written once
    assert 3.0e9 < rec["dram_bytes_per_launch"] < 3.3e9
    if rec["kernel_source_sha256"] == bench.kernel_source_digest():
        assert bench.profiled_traffic(key) == rec["dram_bytes_per_launch"]
    else:
        assert bench.profiled_traffic(key) is None


def test_workload_key_names_other_key_block_sizes():
    wl = I.WORKLOADS["wan-720p"]
    assert bench.workload_key(wl, _args(block_k=64)) == "wan-720p_beta1.04_bk64"
    assert bench.workload_key(wl, _args(block_k=128)) == "wan-720p_beta1.04"
    assert bench.workload_key(wl, _args(block_q=64)) == "wan-720p_beta1.04_bq64"
    assert bench.workload_key(wl, _args(block_q=64, block_k=64)) == "wan-720p_beta1.04_bq64_bk64"
    assert bench.blocks_of(wl, _args(block_q=64)) == (64, 128)
    assert bench.attention_kernel_name(wl, (64, 128)) == "attn_tc_kernel"
    assert bench.profiled_traffic("no-such-workload_beta1") is None


def test_executed_flops_counts_selected_pairs_and_pooled_columns():
    """Three query and key blocks of 128, 128 and 64 tokens (L = 320), d = 2."""
    sel = np.array([[True, False, True], [False, False, False], [True, True, True]])
    d = 2
    got = bench.executed_flops(sel[None, None], 320, 128, 128, d)
    n = [128, 128, 64]
    exact = sum(4 * n[i] * n[j] * d for i in range(3) for j in range(3) if sel[i, j])
    # a query block with an unselected block scores all 3 pooled keys and
    # folds in its unselected ones; block 2 selects everything and has no
    # approximate work
    unsel = [int((~sel[i]).sum()) for i in range(3)]
    approx = sum(2 * n[i] * 3 * d + 2 * n[i] * unsel[i] * d for i in range(3) if unsel[i] > 0)
    assert got["exact"] == exact
    assert got["approx"] == approx
    assert got["total"] == exact + approx
    assert got["selected_fraction"] == sel.mean()


def _run_bench(*argv, env_extra=None):
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv], capture_output=True, text=True,
                          env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_oracle_line():
    """`bench.py --impl reference` times the float64 oracle on the host (no
    GPU) and prints the contract's line with the oracle as its baseline."""
    p = _run_bench("--impl", "reference", "--workload", "tiny-fp32", "--steps", "2", "--warmup", "3")
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == bench.UNIT and d["metric"] == bench.METRIC
    assert d["higher_is_better"] is True and d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    # one head per process: the tiny workload has one head, so one process
    assert cb["cores"] == 1 and cb["extrapolated"] is True and d["extrapolated"] is True
    t = d["timing"]
    assert t["heads_per_sample"] == 1 and t["blocks_per_head"] == 1
    # ms_per_step is what was measured (one sample), the value is the call extrapolated
    assert abs(d["ms_per_step"] - 1e3 * t["sample_wall_s"]) < 1e-6
    assert t["call_s_extrapolated"] > 0 and t["route_s_per_head"] > 0 and t["block_s"] > 0
    wl = I.WORKLOADS["tiny-fp32"]
    assert abs(d["value"] - wl.dense_flops() / t["call_s_extrapolated"] / 1e12) <= 1e-9 * d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == I.WORKLOADS["tiny-fp32"].name


def test_oracle_timer_extrapolates_one_call_from_per_head_times(monkeypatch):
    """The extrapolation is ceil(heads / processes) x (route + Nq x block):
    checked with a stand-in for the pool that returns fixed per-head times."""
    class FakePool:
        def map(self, fn, tasks):
            return [(2.0, 0.5, 1, 591, 0.08) for _ in tasks]

    t = bench.OracleTimer.__new__(bench.OracleTimer)
    t.wl = I.WORKLOADS["wan-720p"]
    t.key, t.beta, t.bq, t.bk, t.moments = "wan-720p", 1.04, 128, 128, "eq5"
    t.cores, t.procs, t.pool = 16, 16, FakePool()
    smp = t.sample(0, 1)
    assert smp["heads_sampled"] == 16 and smp["blocks_per_head"] == 1
    assert smp["call_s_extrapolated"] == 3 * (2.0 + 591 * 0.5)  # 40 heads on 16 processes: 3 rounds
    assert "16 processes" in t.describe(1) and "ceil(40/16)" in t.describe(1)
    assert bench.host_cores() >= 1


def test_reference_arm_other_ranks_exit_quietly():
    p = _run_bench("--impl", "reference", "--workload", "tiny-fp32", "--steps", "1",
                   env_extra={"RANK": "1", "WORLD_SIZE": "2"})
    assert p.returncode == 0, p.stderr
    assert not [l for l in p.stdout.splitlines() if l.startswith("{")]
