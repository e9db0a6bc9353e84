"""The allocation-free router entry point, moe_route_noalloc.

It serves callers that cannot allocate device memory themselves (a host
framework that owns every device allocation, or a serving loop that may not
call an allocator between steps): its scratch is a fixed array inside the
library instead of a caller-provided workspace. This file is collected last so
that a run stopping at the first failure has already run every other test;
it passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs

pytestmark = pytest.mark.gpu


def _route_both(lib, shape, seed):
    inp = moe_inputs.make_inputs(shape, seed=seed, device="cuda")
    T, k = shape.T, shape.k
    idx_ref, w_ref = lib.moe_route(inp.x, inp.W_router, inp.bias, k)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    # through the C ABI directly: device pointers, sizes and the stream only
    st = lib.raw.moe_route_noalloc(
        ctypes.c_void_p(inp.x.data_ptr()), ctypes.c_void_p(inp.W_router.data_ptr()),
        ctypes.c_void_p(inp.bias.data_ptr()) if inp.bias is not None else None,
        T, shape.d, shape.E, k, ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == lib.MOE_OK, lib.raw.moe_status_string(st)
    torch.cuda.synchronize()
    return inp, idx.cpu().numpy(), w.cpu().numpy(), idx_ref.cpu().numpy(), w_ref.cpu().numpy()


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    """Consecutive calls with different sizes share the fixed scratch. Each is
    compared with moe_route (the same routing, bit for bit: same indices, same
    weight bits) and with the CPU oracle (indices bit-exact, weights within
    1e-5 relative). The one-token call, whose router keeps its completion
    tickets in the shared scratch, runs both before and after a 16-token call
    of the same width."""
    from sparse_mixture_experts_route_b200 import _lib as lib
    one = moe_inputs.custom_shape(1, 7168, 896, 16, 512, name="decode1")       # few-token router, T = 1
    first = moe_inputs.custom_shape(16, 7168, 896, 16, 512, name="decode16")   # 3.2 MB of scratch
    second = moe_inputs.custom_shape(7, 256, 64, 4, 64, bias="zipf", name="small")  # different sizes, bias
    for shape, seed in ((one, 2), (first, 0), (one, 3), (second, 1), (one, 2)):
        inp, idx, w, idx_ref, w_ref = _route_both(lib, shape, seed)
        assert np.array_equal(idx, idx_ref), shape.name
        assert np.array_equal(w.view(np.uint32), w_ref.view(np.uint32)), shape.name
        lg = oracle.router_logits(inp.x.cpu(), inp.W_router.cpu(),
                                  inp.bias.cpu() if inp.bias is not None else None)
        ridx, rw = oracle.topk(lg, shape.k)
        assert np.array_equal(idx, ridx), shape.name
        np.testing.assert_allclose(w, rw, rtol=1e-5, atol=1e-7, err_msg=shape.name)
    assert lib.get_device_error() == 0


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    from sparse_mixture_experts_route_b200 import _lib as lib
    # d = 7168, E = 896: 20 tokens fit in the fixed 4 MiB scratch, 21 do not
    assert lib.route_workspace_size(20, 7168, 896) <= lib.ROUTE_NOALLOC_SCRATCH_BYTES
    assert lib.route_workspace_size(21, 7168, 896) > lib.ROUTE_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(21, 7168, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(7168, 896, dtype=torch.float32, device="cuda")
    idx = torch.empty(21, 16, dtype=torch.int32, device="cuda")
    w = torch.empty(21, 16, dtype=torch.float32, device="cuda")
    with pytest.raises(lib.MoEError) as ei:
        lib.moe_route_noalloc(x, W, None, 16, idx, w)
    assert ei.value.status == lib.MOE_ERR_UNSUPPORTED
