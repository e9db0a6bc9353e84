"""GPU parity of the Stable LatentMoE layer (moe_latent_forward) against the
oracle's fp64 layer ("Kimi K3: Open Frontier Intelligence", section
"Operational Execution Flow"; the readings for the lost SiTU-GLU and output
formulas are stated in include/moe.h and in the oracle).

Shapes span one token, few tokens (stream-K GEMMs), ragged feature tiles, the
heavily loaded 256-row-block GEMMs, a Zipf router bias, no shared experts, and
the page's widths (d = 7168, l = 3584) with 64 experts; SiTU-GLU and SwiGLU
both. The bar is the layer tolerance (max |out - ref| <= 1e-2 max |ref|, mean
relative error <= 5e-3), and two calls give the same bits."""
import numpy as np
import pytest
import torch

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


LATENT_SHAPES = [
    # (T, d, l, E, k, f, S, fs, bias, act)
    (64, 256, 128, 8, 2, 128, 2, 192, None, 1),
    (1, 1024, 512, 32, 4, 256, 2, 256, None, 1),
    (9, 512, 192, 16, 4, 64, 1, 128, "zipf", 1),
    (700, 256, 192, 4, 2, 128, 2, 128, None, 1),
    (300, 512, 256, 16, 4, 192, 0, 0, None, 0),
    (128, 7168, 3584, 64, 8, 512, 2, 1024, None, 1),
]


@pytest.mark.parametrize("shape", LATENT_SHAPES, ids=lambda s: "x".join(map(str, s[:8])) + f"_act{s[9]}"
                         + (f"_{s[8]}" if s[8] else ""))
def test_latent_forward_matches_oracle(lib, shape):
    T, d, l, E, k, f, S, fs, bias, act = shape
    base = moe_inputs.custom_shape(T, d, E, k, f, bias=bias)
    li = moe_inputs.make_latent_inputs(base, l, S, fs, seed=12, device="cuda")
    args = (li.x, li.W_router, li.bias, li.W_dn, li.W_up, li.W_gate_up, li.W_down, li.gamma, li.Ws_gate_up,
            li.Ws_down, k)
    out = lib.moe_latent_forward(*args, act=act)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    cpu = lambda t: t.cpu() if t is not None else None
    ref = oracle.latent_forward(cpu(li.x), cpu(li.W_router), cpu(li.bias), cpu(li.W_dn), cpu(li.W_up),
                                cpu(li.W_gate_up), cpu(li.W_down), cpu(li.gamma), cpu(li.Ws_gate_up),
                                cpu(li.Ws_down), k, act=act)
    e = parity.assert_layer_close(out, ref, f"latent {shape}")
    print(shape, e)
    out2 = lib.moe_latent_forward(*args, act=act)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
