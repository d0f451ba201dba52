"""Benchmark of the Sol-Attn sparse attention forward (one JSON line on rank 0).

A step is one call of the whole path -- pooling, routing, work ordering and
the attention kernel -- on one seeded synthetic video-DiT-shaped input.  The
default workload is Wan2.1-14B 720p attention (40 heads, L = 75600 on a
21 x 45 x 80 latent grid, d = 128, blocks of 128) at beta = 1.04.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own
independent call (its own seeded inputs): the heads of different calls do not
interact, so there is no collective on the data path; timing is the max over
ranks.  `--impl reference` times the float64 CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/attention call and dense-equiv TFLOP/s at beta=1.04; % bf16 tensor peak"
UNIT = "TFLOP/s (dense-equivalent)"
NEAR_TIE_MARGIN = 1e-3  # |s_ij - tau_i| below this: a near tie (either decision is correct)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_digest() -> str:
    """sha256 over the attention kernel's sources with comments and blank
    lines removed (the profile's counters are only reported while the code is
    unchanged since they were taken; editing a comment does not count)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("attn_tc.cu", "sm100.cuh", "common.cuh"):
        text = open(os.path.join(ROOT, "video_diffusion_b200", "csrc", f)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip()).encode())
    return h.hexdigest()


def profiled_traffic(workload_key: str):
    """DRAM bytes per attention launch from the committed ncu record of this
    workload (profiles/<kernel>__<key>_dram.json), or None if there is none
    or the kernel changed since it was taken."""
    p = os.path.join(ROOT, "profiles", f"attn_tc_kernel__{workload_key}_dram.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    if rec.get("kernel_source_sha256") == kernel_source_digest():
        return float(rec["dram_bytes_per_launch"])
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# ----------------------------------------------------------------------------- work accounting

def block_tokens(L: int, B: int) -> np.ndarray:
    """Token count of each of the ceil(L / B) blocks."""
    N = -(-L // B)
    n = np.full(N, B, dtype=np.float64)
    n[-1] = L - (N - 1) * B
    return n


def executed_flops(sel: np.ndarray, L: int, Bq: int, Bk: int, d: int) -> dict:
    """Algorithmic FLOPs of one call from the selection [b, H, Nq, Nk] (bool).

    exact:  4 n_i n_j d for every selected pair (QK^T and PV);
    approx: 2 n_i Nk d (token-to-pooled-key scores) + 2 n_i |U_i| d (pooled PV).
    Padding, masked columns and skipped chunk columns are not counted.
    """
    Nk = sel.shape[-1]
    nq, nk = block_tokens(L, Bq), block_tokens(L, Bk)
    exact = 4.0 * d * np.einsum("bhij,i,j->", sel.astype(np.float64), nq, nk)
    unsel = (~sel).sum(axis=-1).astype(np.float64)  # |U_i|, [b, H, Nq]
    rows_with_approx = ((unsel > 0) * nq[None, None, :]).sum()
    approx = 2.0 * d * Nk * float(rows_with_approx) + 2.0 * d * float((unsel * nq[None, None, :]).sum())
    return {"exact": float(exact), "approx": float(approx), "total": float(exact + approx),
            "selected_fraction": float(sel.mean())}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 100 ms; only those taken between mark_start()
    and mark_end() (the timed region) are summarised."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(1.0)  # let the sampler start before the timed region
        except Exception:
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        import datetime as _dt
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 10:
                continue
            try:
                ts = _dt.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if self.t0 is not None and not (self.t0 - 0.05 <= ts <= (self.t1 or ts) + 0.05):
                    continue
                sm.append(float(r[2]))
                smax.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(names, r[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle timing (host)

def host_cores() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_head_task(task):
    """One worker process, one head: builds that head's inputs (untimed),
    then times the float64 oracle's pooling + routing of the whole head and
    its attention for `n_blocks` query blocks.  BLAS runs on one thread."""
    name, head_seed, beta, bq, bk, moments, n_blocks, block_seed = task
    import torch as _torch
    _torch.set_num_threads(1)
    from oracle import sol_attn as O
    from video_diffusion_b200 import inputs as I
    wl = I.WORKLOADS[name]
    Q, K, V = I.make_qkv(wl.grid, 1, wl.d, head_seed, 1, wl.text_tokens, wl.dtype, "cpu")
    Qh, Kh, Vh = (t[0, 0].double().numpy() for t in (Q, K, V))
    t0 = time.perf_counter()
    r = O.route_head(Qh, Kh, bq, bk, beta, moments)
    Vhat = O.pool_blocks(Vh, r["kgeom"], "sum")
    t1 = time.perf_counter()
    N = r["qgeom"].n
    rng = np.random.default_rng(block_seed)
    blocks = rng.choice(N, size=min(n_blocks, N), replace=False)
    scale = 1.0 / math.sqrt(wl.d)
    for i in blocks:
        s0, n = int(r["qgeom"].starts[i]), int(r["qgeom"].counts[i])
        O.attend_query_block(Qh[s0:s0 + n], Kh, Vh, r["kgeom"], r["Kbar"], Vhat, r["sel"][i], scale)
    t2 = time.perf_counter()
    return t1 - t0, (t2 - t1) / len(blocks), len(blocks), N, float(r["sel"].mean())


class OracleTimer:
    """Times the float64 oracle on the host as it would run one call: one
    process per head (BLAS pinned to one thread in each), as many processes as
    this process has cores.  One sample = one head per process, each timing
    its head's pooling + routing and `n_blocks` of its query blocks; the
    whole call is extrapolated from the per-head times:
        call = ceil(heads / processes) * (route + Nq * block).
    The pool is made with the spawn method (a forked pool can hang after CUDA
    is initialised)."""

    def __init__(self, wl_key: str, beta: float, bq: int, bk: int, moments: str):
        import multiprocessing as mp
        from video_diffusion_b200 import inputs as I
        self.wl = I.WORKLOADS[wl_key]
        self.key, self.beta, self.bq, self.bk, self.moments = wl_key, beta, bq, bk, moments
        self.cores = host_cores()
        self.procs = max(1, min(self.cores, self.wl.batch * self.wl.heads))
        for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ[var] = "1"
        self.pool = mp.get_context("spawn").Pool(self.procs)

    def sample(self, step: int, n_blocks: int) -> dict:
        tasks = [(self.key, self.wl.seed + 97 * step + p, self.beta, self.bq, self.bk, self.moments, n_blocks,
                  1000 * step + p) for p in range(self.procs)]
        t0 = time.perf_counter()
        res = self.pool.map(_oracle_head_task, tasks)
        wall = time.perf_counter() - t0
        route = statistics.mean(r[0] for r in res)
        block = statistics.mean(r[1] for r in res)
        N = res[0][3]
        heads = self.wl.batch * self.wl.heads
        call = math.ceil(heads / self.procs) * (route + N * block)
        return {"wall_s": wall, "route_s_per_head": route, "block_s": block, "blocks_per_head": res[0][2],
                "heads_sampled": len(res), "call_s_extrapolated": call, "selected_fraction": res[0][4]}

    def close(self):
        self.pool.close()
        self.pool.join()

    def describe(self, n_blocks: int) -> str:
        heads = self.wl.batch * self.wl.heads
        nq = -(-self.wl.L // self.bq)
        return (f"float64 oracle, {self.procs} processes (one head each, 1 BLAS thread): per head its pooling + "
                f"routing and {n_blocks} of {nq} query blocks timed; the call "
                f"({heads} heads x {nq} blocks) extrapolated as ceil({heads}/{self.procs}) x "
                f"(route + {nq} x block)")


def run_reference(args, wl):
    """The reference arm: the oracle timed on the host's cores.  Each step is
    one sample (one head per process, one query block each); `ms_per_step`
    is that sample's measured wall time, while `value` is the whole call's
    dense-equivalent rate extrapolated from the samples (marked so)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    bq, bk = blocks_of(wl, args)
    timer = OracleTimer(args.workload, args.beta, bq, bk, moments_of(args))
    samples = []
    try:
        for s in range(args.warmup + args.steps):
            smp = timer.sample(s, n_blocks=1)
            if s >= args.warmup:
                samples.append(smp)
    finally:
        timer.close()
    call_s = statistics.mean(x["call_s_extrapolated"] for x in samples)
    wall_ms = statistics.mean(x["wall_s"] for x in samples) * 1e3
    value = wl.dense_flops() / call_s / 1e12
    sample = timer.describe(1)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, args),
        "extrapolated": True,
        "timing": {"ms_per_step": "measured wall time of one sample (not of a whole call)",
                   "value": "whole call, extrapolated from the samples",
                   "call_s_extrapolated": call_s, "sample_wall_s": wall_ms / 1e3,
                   "route_s_per_head": statistics.mean(x["route_s_per_head"] for x in samples),
                   "block_s": statistics.mean(x["block_s"] for x in samples),
                   "heads_per_sample": samples[0]["heads_sampled"], "blocks_per_head": 1},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": timer.procs, "kind": "oracle", "sample": sample,
                         "extrapolated": True},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl, args):
    c = {"workload": wl.name, "beta": args.beta, "batch": wl.batch, "heads": wl.heads, "L": wl.L,
         "d": wl.d, "block": wl.block, "parallelism": f"replicas x{args.gpus} (independent calls)",
         "l2": f"inputs {3 * wl.batch * wl.heads * wl.L * wl.d * 2 / 1e9:.2f} GB per step "
               f"({'larger' if 3 * wl.batch * wl.heads * wl.L * wl.d * 2 > 126e6 else 'smaller'} than the "
               f"126 MB L2); no flush"}
    if args.block_k and args.block_k != wl.block:
        c["block_k"] = args.block_k
    if args.block_q and args.block_q != wl.block:
        c["block_q"] = args.block_q
    if args.diagonal_sigma:
        c["sigma"] = "diagonal estimator"
    if args.route_in_kernel:
        c["routing"] = "inside the attention kernel"
    return c


def moments_of(args) -> str:
    return "diagonal" if args.diagonal_sigma else "eq5"


def blocks_of(wl, args):
    return (args.block_q or wl.block, args.block_k or wl.block)


def attention_kernel_name(wl, blk) -> str:
    """The library runs tcgen05 for bf16, d in {64, 128}, Bq and Bk in {64, 128}."""
    tc = wl.dtype == torch.bfloat16 and wl.d in (64, 128) and blk[0] in (64, 128) and blk[1] in (64, 128)
    return "attn_tc_kernel" if tc else "attn_simt_kernel"


def workload_key(wl, args) -> str:
    """File-name key of a workload's profile summaries: registry name, beta and
    key block size when it differs from the query block."""
    key = f"{args.workload}_beta{args.beta:g}"
    if args.block_q and args.block_q != wl.block:
        key += f"_bq{args.block_q}"
    if args.block_k and args.block_k != wl.block:
        key += f"_bk{args.block_k}"
    return key


# ----------------------------------------------------------------------------- ranks

def rank_info():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def setup_dist(world: int, backend: str, device=None):
    """Process group for N > 1 (short timeout so a missing rank ends in an
    error, not a wait); None when running alone."""
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def reduce_max(x: float, pg, device) -> float:
    """Max of x over ranks (the job's time is its slowest rank's)."""
    if pg is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world: int, flops_per_call: float, ms_per_call: float) -> float:
    """Whole-job dense-equivalent TFLOP/s: every rank runs one call per step."""
    return world * flops_per_call / (ms_per_call * 1e-3) / 1e12


# ----------------------------------------------------------------------------- beta sweep

def sweep_beta(args):
    """Per beta: selected fraction, ms per call, dense-equivalent and executed
    TFLOP/s, speedup over the same kernel at beta = -inf, and the error of
    the output against that dense output."""
    from video_diffusion_b200 import api
    from video_diffusion_b200 import inputs as I
    wl = I.WORKLOADS[args.workload]
    blk = blocks_of(wl, args)
    diag = bool(args.diagonal_sigma)
    dev = torch.device("cuda", 0)
    Q, K, V = I.make_workload(wl, device=dev)
    peak = float(load_peaks()["bf16_tflops"])

    def timed(beta, out, keep_or_drop=False):
        for _ in range(args.warmup):
            api.forward_ex(Q, K, V, beta, blk, out=out, keep_or_drop=keep_or_drop, diagonal_sigma=diag)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.steps):
            api.forward_ex(Q, K, V, beta, blk, out=out, keep_or_drop=keep_or_drop, diagonal_sigma=diag)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    dense = torch.empty_like(Q)
    dense_ms = timed(-math.inf, dense)
    dref = dense.float()
    for tok in args.sweep_beta.split(","):
        beta = float(tok)
        out = torch.empty_like(Q)
        ms = dense_ms if beta == -math.inf else timed(beta, out)
        if beta == -math.inf:
            out = dense
        counts, sel = api.stats(Q, K, beta, blk, with_mask=True, diagonal_sigma=diag)
        work = executed_flops(sel.cpu().numpy(), wl.L, blk[0], blk[1], wl.d)
        near = int(api.near_ties(Q, K, beta, blk, margin=NEAR_TIE_MARGIN, diagonal_sigma=diag).sum())
        diff = out.float() - dref
        # the same beta with the correction off (keep-or-drop): what Eqs. 9-10 buy
        kod = torch.empty_like(Q)
        kod_ms = dense_ms if beta == -math.inf else timed(beta, kod, keep_or_drop=True)
        if beta == -math.inf:
            kod = dense
        kdiff = kod.float() - dref
        line = {"workload": wl.name, "block": list(blk), "sigma": moments_of(args), "beta": beta,
                "selected_fraction": work["selected_fraction"],
                "near_ties": near, "near_tie_margin": NEAR_TIE_MARGIN,
                "gaussian_fraction": 0.5 * math.erfc(beta / math.sqrt(2)) if math.isfinite(beta) else
                (1.0 if beta < 0 else 0.0),
                "ms_per_call": ms, "dense_equiv_tflops": wl.dense_flops() / (ms * 1e-3) / 1e12,
                "executed_tflops": work["total"] / (ms * 1e-3) / 1e12,
                "pct_bf16_peak": 100 * work["total"] / (ms * 1e-3) / 1e12 / peak,
                "speedup_vs_dense": dense_ms / ms, "target_speedup": 1.0 / (work["selected_fraction"] + 0.15),
                "rel_l2_vs_dense": float(diff.norm() / dref.norm()), "max_abs_vs_dense": float(diff.abs().max()),
                "keep_or_drop": {"ms_per_call": kod_ms, "rel_l2_vs_dense": float(kdiff.norm() / dref.norm()),
                                 "max_abs_vs_dense": float(kdiff.abs().max())}}
        print(json.dumps(line), flush=True)
        del out, sel, counts, diff, kod, kdiff


# ----------------------------------------------------------------------------- one call split by heads

def run_sharded(args, wl, world, rank, local, dev, pg):
    """One call of the workload split across the ranks by heads: `heads`
    gives each rank its heads of every token; `ulysses` gives each rank its
    token range of every head and times the seq -> head all-to-all of q, k
    and v, the rank's heads, and the head -> seq all-to-all of the output.
    The total work is fixed as N grows (strong scaling); timing is the max
    over ranks of CUDA-event time on the launching stream."""
    from video_diffusion_b200 import api
    from video_diffusion_b200 import sharded as S
    blk = blocks_of(wl, args)
    Q, K, V = I_make(wl, dev)
    counts, sel = api.stats(Q, K, args.beta, blk, with_mask=True)
    work = executed_flops(sel.cpu().numpy(), wl.L, blk[0], blk[1], wl.d)
    del counts, sel
    if args.mode == "heads":
        q, k, v = (S.shard_heads(t, world, rank).contiguous() for t in (Q, K, V))

        def call():
            return S.forward_heads(q, k, v, args.beta, blk)
    else:
        q, k, v = (S.shard_tokens(t, world, rank).contiguous() for t in (Q, K, V))

        def call():
            if pg is None:  # one rank: nothing to exchange
                return api.forward(q, k, v, args.beta, blk)
            return S.forward_ulysses(q, k, v, args.beta, wl.heads, wl.L, blk)
    del Q, K, V
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        call()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        clocks.mark_start()
        e0.record(stream)
        for _ in range(args.steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
    if pg is not None:
        pg.barrier()
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, pg, dev)
    heads_here = S.split_sizes(wl.heads, world)[rank]
    line = {
        "metric": METRIC, "value": wl.dense_flops() / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded smooth-field Q/K, V ~ N(0,1))",
        "config": dict(config_of(wl, args), parallelism=f"{args.mode} x{world} (one call split by heads)"),
        "ms_per_call": ms, "selected_fraction": work["selected_fraction"],
        "executed_tflop_per_call": work["total"] / 1e12,
        "heads_on_rank0": S.split_sizes(wl.heads, world)[0], "heads_here": heads_here,
        "exchange_bytes_per_rank": (4 * S.exchange_bytes((wl.batch, wl.heads, wl.L, wl.d), 2, world, 0)
                                    if args.mode == "ulysses" else 0),
        "gpu_launches": 4 * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def I_make(wl, dev):
    from video_diffusion_b200 import inputs as I
    return I.make_workload(wl, device=dev)


# ----------------------------------------------------------------------------- GPU arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan-720p")
    ap.add_argument("--beta", type=float, default=1.04)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block-q", type=int, default=None,
                    help="query block size (64 or 128); default: the workload's block")
    ap.add_argument("--block-k", type=int, default=None,
                    help="key block size (default: the workload's block size, the same as the query block)")
    ap.add_argument("--route-in-kernel", action="store_true",
                    help="let the attention kernel decide the selection itself (no selection mask)")
    ap.add_argument("--diagonal-sigma", action="store_true",
                    help="sigma_i of Eq. 4 from the diagonal moment estimator instead of Eq. 5")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "heads", "ulysses"],
                    help="N > 1: replicas = one independent call per rank (weak scaling); heads = one call "
                         "split across ranks by heads; ulysses = the same from sequence-sharded inputs, with "
                         "the all-to-all re-layouts before and after (strong scaling)")
    ap.add_argument("--sweep-beta", default=None,
                    help="comma-separated betas: print one line per beta (fraction, time, speedup and "
                         "error against the beta=-inf output) instead of the benchmark line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.sweep_beta:
        sweep_beta(args)
        return

    from video_diffusion_b200 import inputs as I
    wl = I.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return

    from video_diffusion_b200 import api

    world, rank, local = rank_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = setup_dist(world, "nccl", dev)
    if args.mode != "replicas":
        run_sharded(args, wl, world, rank, local, dev, pg)
        if pg is not None:
            pg.destroy_process_group()
        return

    def barrier():
        if pg is not None:
            pg.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, pg, dev)

    peaks = load_peaks()
    Q, K, V = I.make_workload(wl, device=dev, seed_offset=rank)
    out = torch.empty_like(Q)
    stream = torch.cuda.current_stream()

    blk = blocks_of(wl, args)
    diag = bool(args.diagonal_sigma)
    # selection statistics (same routing as the forward) for the FLOP count
    counts, sel = api.stats(Q, K, args.beta, blk, with_mask=True, diagonal_sigma=diag)
    work = executed_flops(sel.cpu().numpy(), wl.L, blk[0], blk[1], wl.d)
    # decisions within 1e-3 of tau_i (where fp32 and fp64 routing may differ)
    near = int(api.near_ties(Q, K, args.beta, blk, margin=NEAR_TIE_MARGIN, diagonal_sigma=diag).sum())
    del sel, counts

    for _ in range(args.warmup):
        api.forward_ex(Q, K, V, args.beta, blk, out=out, diagonal_sigma=diag, route_in_kernel=args.route_in_kernel)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for row in evs:  # torch creates the CUDA event on first record; the library then re-records it
        for e in row:
            e.record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        clocks.mark_start()
        start.record(stream)
        for s in range(args.steps):
            api.forward_ex(Q, K, V, args.beta, blk, out=out, events=evs[s], diagonal_sigma=diag,
                           route_in_kernel=args.route_in_kernel)
        end.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
    barrier()
    # busy spread over the CTAs of the last timed attention launch
    load_balance = api.load_balance(api.cta_times(stream))
    total_ms = start.elapsed_time(end)
    ms_step = max_over_ranks(total_ms / args.steps)
    stage = {"pool": [], "route": [], "attention": []}
    for e in evs:
        stage["pool"].append(e[0].elapsed_time(e[1]))
        stage["route"].append(e[1].elapsed_time(e[2]))
        stage["attention"].append(e[2].elapsed_time(e[3]))
    stage_ms = {k: statistics.mean(v) for k, v in stage.items()}
    clock_summary = clocks.summary()

    # in-house dense comparator: the same kernel with beta = -inf, timed like
    # the sparse call (same warm-up, the same number of calls, at least 20)
    dense_ms, dense_calls = None, 0
    if args.beta != -math.inf:
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(args.warmup):
            api.forward(Q, K, V, -math.inf, blk, out=out)
        dense_calls = max(args.steps, 20)
        barrier()
        torch.cuda.synchronize()
        d0.record(stream)
        for _ in range(dense_calls):
            api.forward(Q, K, V, -math.inf, blk, out=out)
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms = max_over_ranks(d0.elapsed_time(d1) / dense_calls)

    # end to end through the public call with host buffers: the library copies
    # each group of heads in, computes it and copies it back, overlapped
    e2e = None
    if not args.no_e2e:
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
        hO = torch.empty_like(hQ).pin_memory()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, min(args.steps, 5))
        api.forward_host(hQ, hK, hV, args.beta, blk, out=hO, diagonal_sigma=diag,
                         route_in_kernel=args.route_in_kernel)  # warm-up: staging memory, internal streams
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            api.forward_host(hQ, hK, hV, args.beta, blk, out=hO, diagonal_sigma=diag,
                             route_in_kernel=args.route_in_kernel)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e)
        e2e = {"value": aggregate_value(world, wl.dense_flops(), e2e_ms), "unit": UNIT, "ms_per_call": e2e_ms,
               "h2d_bytes_per_step": 3 * Q.numel() * Q.element_size(),
               "d2h_bytes_per_step": hO.numel() * hO.element_size(), "steps": n_e2e,
               "call": "sol_attn_forward_host (pinned host buffers, copies overlapped with compute)"}
        del hQ, hK, hV, hO

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        timer = OracleTimer(args.workload, args.beta, blk[0], blk[1], moments_of(args))
        try:
            smp = timer.sample(0, n_blocks=2)
        finally:
            timer.close()
        cpu = {"value": wl.dense_flops() / smp["call_s_extrapolated"] / 1e12, "unit": UNIT, "cores": timer.procs,
               "kind": "oracle", "sample": timer.describe(2), "extrapolated": True,
               "call_s_extrapolated": smp["call_s_extrapolated"], "sample_wall_s": smp["wall_s"]}

    attn_ms = max_over_ranks(stage_ms["attention"])
    achieved = work["total"] / (attn_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    value = aggregate_value(world, wl.dense_flops(), ms_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded smooth-field Q/K, V ~ N(0,1))",
        "config": config_of(wl, args),
        "ms_per_call": ms_step,
        "selected_fraction": work["selected_fraction"],
        "near_ties": {"margin": NEAR_TIE_MARGIN, "pairs": near,
                      "fraction_of_pairs": near / float(wl.batch * wl.heads * -(-wl.L // blk[0]) *
                                                        -(-wl.L // blk[1]))},
        "executed_tflop_per_call": work["total"] / 1e12,
        "executed_tflops": work["total"] / (ms_step * 1e-3) / 1e12,
        "pct_bf16_peak": 100.0 * work["total"] / (ms_step * 1e-3) / 1e12 / peak,
        "stages_ms": stage_ms,
        "load_balance": load_balance,
        "dense_ms_per_call": dense_ms,
        "dense_calls_timed": dense_calls,
        "speedup_vs_dense": (dense_ms / ms_step) if dense_ms else None,
        "target_speedup": 1.0 / (work["selected_fraction"] + 0.15),
        "roofline": {"kernel": attention_kernel_name(wl, blk), "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": profiled_traffic(workload_key(wl, args)),
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "frac_of_sustained": (achieved / float(peaks["bf16_tflops_sustained"])
                                           if peaks.get("bf16_tflops_sustained") else None)},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": (5 if diag else 4) * args.steps,
        "clocks": clock_summary,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
