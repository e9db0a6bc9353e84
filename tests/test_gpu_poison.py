"""Uninitialised-read check (a stand-in for a memory sanitizer, which is not
available here): every entry point that takes a workspace must give the same
bits whatever the workspace held before the call.

Each case runs once on a zeroed workspace, then on the same workspace filled
with 0xFF bytes (every ticket or counter at its largest value, every index
-1) and with the 32-bit pattern 0x7FC07FC0 (an fp32 NaN, and two bf16 NaNs),
and twice in a row on each, since a call leaves its own state behind. Nothing
in the library waits on a workspace value (tickets only decide which CTA
finishes a tile, and every wait is on a barrier in shared memory, with a time
limit), so a poisoned workspace can change results but cannot hang.

Shapes: the one-token step (few-token router with its completion tickets,
stream-K gate/up and down GEMMs), a K-split few-tile step, the many-token
tensor-core screen router with whole-tile GEMMs, 256-row token blocks, and
ragged tails."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_route_b200 import inputs as moe_inputs

pytestmark = pytest.mark.gpu

POISON = {"ff": 0xFFFFFFFF, "nan": 0x7FC07FC0}

SHAPES = [
    # (T, d, E, k, f, bias)
    (1, 7168, 896, 16, 512, None),
    (8, 1024, 8, 2, 128, None),
    (3, 1024, 8, 2, 192, "zipf"),
    (333, 320, 20, 3, 192, None),
    (600, 128, 4, 2, 128, None),
    (300, 512, 896, 16, 64, "zipf"),
]


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_mixture_experts_route_b200 import _lib
    _lib.get_device_error(clear=True)
    return _lib


def _fill(ws, pattern):
    n = ws.numel() // 4
    if n:
        ws[: n * 4].view(torch.int32).fill_(np.array(pattern, dtype=np.uint32).view(np.int32).item())
    ws[n * 4:].fill_(pattern & 0xFF)


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + (f"_{s[5]}" if s[5] else ""))
def test_forward_same_bits_whatever_the_workspace_held(lib, shape):
    T, d, E, k, f, bias = shape
    inp = moe_inputs.make_inputs(moe_inputs.custom_shape(T, d, E, k, f, bias=bias), seed=5, device="cuda")
    args = (inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    ws = torch.zeros(lib.moe_forward_workspace_size(T, d, E, k, f), dtype=torch.uint8, device="cuda")
    ref = lib.moe_forward(*args, workspace=ws).clone()
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    for name, pattern in POISON.items():
        _fill(ws, pattern)
        for rep in range(2):
            out = lib.moe_forward(*args, workspace=ws)
            torch.cuda.synchronize()
            assert lib.get_device_error() == 0, (name, rep)
            assert torch.equal(_bits(out), _bits(ref)), (name, rep)


@pytest.mark.parametrize("shape", SHAPES[:4], ids=lambda s: "x".join(map(str, s[:5])))
def test_steps_same_bits_whatever_the_workspace_held(lib, shape):
    """The separate steps: moe_route, moe_permute and moe_expert_ffn each on
    its own poisoned workspace."""
    T, d, E, k, f, bias = shape
    inp = moe_inputs.make_inputs(moe_inputs.custom_shape(T, d, E, k, f, bias=bias), seed=6, device="cuda")
    ws_r = torch.zeros(max(256, lib.route_workspace_size(T, d, E)), dtype=torch.uint8, device="cuda")
    ws_p = torch.zeros(max(256, lib.permute_workspace_size(T, E, k)), dtype=torch.uint8, device="cuda")
    ws_f = torch.zeros(max(256, lib.expert_ffn_workspace_size(T * k, E)), dtype=torch.uint8, device="cuda")

    def run():
        idx, w = lib.moe_route(inp.x, inp.W_router, inp.bias, k, workspace=ws_r)
        offs, perm, inv, xp = lib.moe_permute(inp.x, idx, E, workspace=ws_p)
        h, y = lib.moe_expert_ffn(xp, offs, inp.W_gate_up, inp.W_down, workspace=ws_f)
        torch.cuda.synchronize()
        return [t.clone() for t in (idx, w, offs, perm, inv, xp, h, y)]

    ref = run()
    assert lib.get_device_error() == 0
    for name, pattern in POISON.items():
        for ws in (ws_r, ws_p, ws_f):
            _fill(ws, pattern)
        for rep in range(2):
            got = run()
            assert lib.get_device_error() == 0, (name, rep)
            for a, b in zip(got, ref):
                assert torch.equal(_bits(a), _bits(b)), (name, rep)
