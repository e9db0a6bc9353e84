"""Expert parallelism (sparse_mixture_experts_route_b200/ep.py) on CPU ranks.

The exchange protocol of ep_forward -- count all-to-all, row all-to-all in
exact or fixed-capacity mode, the owner's gather into expert-major order and
back, the return all-to-all and the combine -- runs unchanged on world-size 2
and 3 gloo groups. The local steps (router, dispatch tables, expert
feed-forward, row gathers, combine) are supplied by the oracle here, since the
CPU ranks have no GPU; on GPUs the same protocol calls the library's kernels.
Each rank's output must equal the oracle's whole layer for that rank's tokens
with every expert in one process, bit for bit: the oracle's per-row arithmetic
does not depend on which rows share an expert call, so any misplaced row,
count or weight shows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The local steps of ep_forward on the CPU oracle (test infrastructure)."""

    ffn_dtype = torch.float64

    def __init__(self, oracle):
        self.o = oracle

    def route(self, x, W_router, bias, k):
        lg = self.o.router_logits(x, W_router, bias)
        idx, w = self.o.topk(lg, k)
        return torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)), torch.from_numpy(w)

    def dispatch(self, x, idx, E):
        _, offsets, perm, inv = self.o.permute(idx.numpy(), E)
        return (torch.from_numpy(np.asarray(offsets, dtype=np.int32)),
                torch.from_numpy(np.asarray(perm, dtype=np.int32)),
                torch.from_numpy(np.asarray(inv, dtype=np.int32).reshape(idx.shape)))

    def gather(self, src, rows):
        out = torch.zeros(rows.shape[0], src.shape[1], dtype=src.dtype)
        m = rows >= 0
        out[m] = src[rows[m].long()]
        return out

    def expert_ffn(self, x_rows, offsets, W_gate_up, W_down):
        y = torch.zeros(x_rows.shape[0], x_rows.shape[1], dtype=torch.float64)
        for e in range(W_gate_up.shape[0]):
            a, b = int(offsets[e]), int(offsets[e + 1])
            if b > a:
                y[a:b] = torch.from_numpy(self.o.expert_ffn(x_rows[a:b], W_gate_up[e], W_down[e]))
        return y

    def combine(self, y_rows, inv, w):
        return torch.from_numpy(self.o.combine(y_rows.numpy(), inv.numpy(), w.numpy()))


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from sparse_mixture_experts_route_b200 import ep
        from sparse_mixture_experts_route_b200 import inputs as mi
        T, d, E, k, f, bias, mode, cap = case
        shape = mi.custom_shape(T * world, d, E, k, f, bias=bias)
        inp = mi.make_inputs(shape, seed=4)           # the same draw on every rank
        E_loc = E // world
        mine = slice(rank * T, (rank + 1) * T)
        x = inp.x[mine].contiguous()
        ops = OracleOps(oracle)
        out, stats = ep.ep_forward(x, inp.W_router, inp.bias,
                                   inp.W_gate_up[rank * E_loc:(rank + 1) * E_loc].contiguous(),
                                   inp.W_down[rank * E_loc:(rank + 1) * E_loc].contiguous(), k,
                                   mode=mode, capacity=cap, ops=ops)
        ref, ridx, rw = oracle.forward(x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
        # tokens none of whose rows were dropped (all of them unless the capacity is short)
        _, offsets, _, inv = oracle.permute(ridx, E)
        kept = np.ones(T, dtype=bool)
        if mode == "capacity" and cap is not None:
            g_pair = ridx // E_loc
            local = inv.reshape(T, k) - offsets[g_pair * E_loc]
            kept = (local < cap).all(axis=1)
        same = bool(np.array_equal(out.numpy()[kept], ref[kept]))
        q.put((rank, same, int(kept.sum()), int(stats.overflow), stats.send_rows.tolist(),
               stats.recv_rows.tolist()))
    finally:
        dist.destroy_process_group()


def _run(world, case):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    return sorted(q.get(timeout=10) for _ in range(world))


@pytest.mark.parametrize("world,case", [
    (2, (24, 64, 8, 3, 64, None, "exact", None)),
    (2, (24, 64, 8, 3, 64, "zipf", "capacity", None)),   # default capacity: T * min(k, E/G), never exceeded
    (3, (17, 64, 9, 2, 64, "zipf", "exact", None)),      # skewed loads, ragged counts, an uneven world
], ids=["w2_exact", "w2_capacity", "w3_exact_zipf"])
def test_ep_forward_equals_one_process_oracle(world, case):
    res = _run(world, case)
    T, k = case[0], case[3]
    sent = np.array([r[4] for r in res])
    recv = np.array([r[5] for r in res])
    assert np.array_equal(sent, recv.T)                   # what g sent to h is what h got from g
    assert sent.sum() == world * T * k                    # every (token, expert) row travelled once
    for rank, same, n_kept, overflow, _, _ in res:
        assert overflow == 0 and n_kept == T
        assert same, f"rank {rank} differs from the one-process oracle"


def test_ep_capacity_overflow_is_flagged_and_drops_only_overflowing_rows():
    """With a capacity below the Zipf-skewed load, the rows past C of a pair
    are dropped and the overflow flag is set; every token none of whose rows
    was dropped still equals the oracle exactly."""
    world, case = 2, (24, 64, 8, 3, 64, "zipf", "capacity", 10)
    res = _run(world, case)
    assert any(r[3] == 1 for r in res)
    for rank, same, n_kept, overflow, sent, _ in res:
        assert same, rank
        assert n_kept < 24 or max(sent) <= 10
