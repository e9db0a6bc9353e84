"""Parity at the full workload sizes, in the launch configuration bench.py
times (moe_forward on one stream). Routing (indices, per-expert offsets, the
count invariant) is compared for EVERY token; the layer output is compared on
sampled tokens, which the oracle computes one by one from only the experts
they select (the full weights stay on the device)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs
import moe_parity as parity

pytestmark = pytest.mark.gpu

FULL = [("prefill", 8), ("decode", 24), ("skewed", 10), ("sweep_T1", 1), ("sweep_T8", 8), ("sweep_T32", 12),
        ("sweep_T128", 12), ("sweep_T512", 12)]


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_mixture_experts_route_b200 import _lib
    _lib.get_device_error(clear=True)
    return _lib


@pytest.mark.parametrize("name,n_sample", FULL, ids=[f[0] for f in FULL])
def test_full_size_workload(lib, name, n_sample):
    shape = moe_inputs.WORKLOADS[name]
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    inp = moe_inputs.make_inputs(shape, seed=0, device="cuda")
    # the bench's launch: the fused forward
    out = lib.moe_forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    # routing of every token, bit for bit
    idx, w = lib.moe_route(inp.x, inp.W_router, inp.bias, k)
    offs, perm, inv, _ = lib.moe_permute(None, idx, E, with_rows=False)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    _, ridx, rw = parity.oracle_route(inp, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=parity.W_RTOL, atol=parity.W_ATOL)
    counts, roffs, rperm, rinv = oracle.permute(ridx, E)
    assert counts.sum() == T * k
    assert np.array_equal(offs.cpu().numpy(), roffs)
    assert np.array_equal(perm.cpu().numpy(), rperm)
    assert np.array_equal(inv.cpu().numpy(), rinv)
    # sampled outputs: always the first and last token, plus seeded picks
    rng = np.random.default_rng(1234)
    sample = sorted(set([0, T - 1] + rng.choice(T, size=min(T, n_sample), replace=False).tolist()))
    ref, sidx, _ = parity.oracle_sampled_forward(inp, k, sample)
    assert np.array_equal(sidx, ridx[sample])
    got = out[torch.as_tensor(sample, device="cuda")]
    e = parity.assert_layer_close(got, ref, name)
    print(name, "touched", int((counts > 0).sum()), "max rows", int(counts.max()), e)
    # deterministic: the same launch again gives the same bits
    out2 = lib.moe_forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    assert torch.equal(out, out2)
    del inp, out, out2
    torch.cuda.empty_cache()
