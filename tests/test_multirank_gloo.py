"""The multi-GPU host path of bench.py, run as world-size-2 gloo ranks on CPU.

Each GPU is an independent replica routing its own tokens (the layer shards
by tokens; the forward pass has no exchange step), so the only collectives
are the timing barrier and the max-over-ranks reduction. These tests check
that logic without a GPU: the max over ranks, the whole-job throughput, that
replicas draw different tokens from one seeded recipe, and that only rank 0
of the reference arm does any work. The Quantile Balancing bias update (the
next row after the forward pass) does have an exchange step, an integer
all-reduce of per-expert margin histograms; its test checks that the summed
histograms give every rank the biases of the whole batch.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from sparse_mixture_experts_route_b200 import inputs as mi
        bench.barrier(world)
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world)
        shape = mi.custom_shape(16, 64, 4, 2, 64)
        x = mi.make_x(shape, seed=bench.replica_x_seed(rank))
        xf = x.float().contiguous()
        xs = [torch.empty_like(xf) for _ in range(world)]
        dist.all_gather(xs, xf)
        q.put((rank, slowest, bench.aggregate_tokens_per_s(shape.T, 4, world, slowest),
               all(torch.equal(xs[r], xf) == (r == rank) for r in range(world))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, tps, distinct in res:
        assert slowest == 15.0                       # the max over ranks, seen by every rank
        assert tps == pytest.approx(2 * 16 * 4 / 0.015)
        assert distinct                              # replicas route different tokens


def test_reference_arm_nonzero_rank_does_no_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    import json
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3", "--cpu-budget", "2"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == "moe_layer_tokens_per_s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def _qb_worker(rank, world, port, q):
    """Quantile Balancing across data-parallel ranks: each rank counts the
    margins of its own tokens, one integer all-reduce sums the histograms, and
    every rank recovers the same biases as one process holding the whole batch."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        m, n, k, lo, hi, bins = 600, 16, 2, -10.0, 10.0, 1000
        rng = np.random.default_rng(11)
        s = rng.normal(size=(m, n)) + 1.5 * np.log1p(np.arange(n))[::-1]   # the same batch on every rank
        b0 = np.zeros(n)
        mine = slice(rank * m // world, (rank + 1) * m // world)
        a = oracle.qb_cutoffs(s[mine], k, b0)
        H = torch.from_numpy(oracle.qb_histogram(s[mine], a, lo, hi, bins))
        dist.all_reduce(H, op=dist.ReduceOp.SUM)
        b_dist = oracle.qb_bias_from_histogram(H.numpy(), lo, hi, m, k)
        a_all = oracle.qb_cutoffs(s, k, b0)
        b_one = oracle.qb_bias_from_histogram(oracle.qb_histogram(s, a_all, lo, hi, bins), lo, hi, m, k)
        b_exact = oracle.qb_update(s, k, b0)
        q.put((rank, bool(np.array_equal(b_dist, b_one)),
               float(np.abs(b_dist - b_exact).max()), (hi - lo) / bins))
    finally:
        dist.destroy_process_group()


def test_quantile_balancing_histograms_all_reduce_over_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_qb_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, same_as_one_process, err, width in res:
        assert same_as_one_process
        assert err <= width + 1e-12
