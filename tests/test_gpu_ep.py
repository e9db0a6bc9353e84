"""GPU side of expert parallelism: the row gather behind the exchange
(moe_gather_rows) bit for bit against indexing, and ep_forward on a one-rank
NCCL group (the only group one GPU can hold: NCCL refuses two ranks on one
device). With one rank every exchange is a local copy, but the whole path
runs -- count and row all-to-alls through NCCL, the index maps on the device,
the gathers, the grouped feed-forward of the rank's experts and the combine,
all in this library's kernels -- and must match the oracle within the layer
tolerance and the staged entry points (route, permute, expert_ffn,
unpermute) bit for bit. The protocol across several ranks is
tested on CPU ranks in test_ep_gloo.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs
import moe_parity as parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_mixture_experts_route_b200 import _lib
    _lib.get_device_error(clear=True)
    return _lib


def test_gather_rows_bit_exact_padding_and_bad_index(lib):
    g = torch.Generator().manual_seed(3)
    src = torch.randn(100, 72, generator=g).to(torch.bfloat16).cuda()
    rows = torch.randint(0, 100, (333,), generator=g, dtype=torch.int32)
    rows[::7] = -1                                        # padding rows
    out = lib.moe_gather_rows(src, rows.cuda())
    torch.cuda.synchronize()
    want = torch.zeros(333, 72, dtype=torch.bfloat16)
    m = rows >= 0
    want[m] = src.cpu()[rows[m].long()]
    assert torch.equal(out.cpu().view(torch.int16), want.view(torch.int16))
    assert lib.get_device_error() == 0
    # an index past the source writes a zero row and records the error code
    bad = torch.tensor([5, 100, 7], dtype=torch.int32).cuda()
    out = lib.moe_gather_rows(src, bad)
    assert lib.get_device_error(clear=True) == 5
    assert torch.equal(out[1].cpu(), torch.zeros(72, dtype=torch.bfloat16))
    assert torch.equal(out[0], src[5]) and torch.equal(out[2], src[7])
    assert lib.get_device_error() == 0


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("shape,mode", [((64, 256, 8, 2, 128, None), "exact"),
                                        ((300, 512, 16, 4, 256, "zipf"), "exact"),
                                        ((300, 512, 16, 4, 256, "zipf"), "capacity"),
                                        ((1, 7168, 896, 16, 512, None), "capacity")],
                         ids=["small_exact", "zipf_exact", "zipf_capacity", "T1_capacity"])
def test_ep_forward_one_rank(lib, nccl_group, shape, mode):
    from sparse_mixture_experts_route_b200 import ep
    T, d, E, k, f, bias = shape
    inp = moe_inputs.make_inputs(moe_inputs.custom_shape(T, d, E, k, f, bias=bias), seed=8, device="cuda")
    out, stats = ep.ep_forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k, mode=mode)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    assert int(stats.overflow) == 0 and int(stats.send_rows.sum()) == T * k
    ref, _, _ = oracle.forward(inp.x.cpu(), inp.W_router.cpu(), inp.bias.cpu() if inp.bias is not None else None,
                               inp.W_gate_up.cpu(), inp.W_down.cpu(), k)
    parity.assert_layer_close(out, ref, f"ep_forward {shape} {mode}")
    # one rank runs the staged steps on its rows: the same bits as those steps
    idx, w = lib.moe_route(inp.x, inp.W_router, inp.bias, k)
    offs, _, inv, xp = lib.moe_permute(inp.x, idx, E)
    _, y = lib.moe_expert_ffn(xp, offs, inp.W_gate_up, inp.W_down)
    staged = lib.moe_unpermute(y, inv, w)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), staged.view(torch.int16))
