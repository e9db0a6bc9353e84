"""Parity at the full workload sizes, in the launch configuration bench.py
times (moe_forward on one stream).

Routing (indices, per-expert offsets, permutations, the count invariant) is
compared for EVERY token, the router weights under their per-path tolerance.
The layer output is compared in full on the decode workload and on every point
of the decode sweep; on prefill and on the skewed workload (the oracle would
take minutes for every token) on a seeded subset of 512 tokens, always holding
the first and the last token. The oracle computes those rows expert by expert
from only the selected experts' weights, fetched one expert at a time, on all
host threads."""
import time

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs
import moe_parity as parity

pytestmark = pytest.mark.gpu

# (workload, tokens whose output is compared: None = all)
FULL = [("prefill", 512), ("decode", None), ("skewed", 512), ("sweep_T1", None), ("sweep_T8", None),
        ("sweep_T32", None), ("sweep_T128", None), ("sweep_T512", None)]


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
    lg, ridx, rw = parity.oracle_route(inp, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    w_err, w_tol = parity.assert_route_weights(w, rw, inp.x.cpu(), inp.W_router.cpu(),
                                               inp.bias.cpu() if inp.bias is not None else None, k, lg, ridx,
                                               what=name)
    counts, roffs, rperm, rinv = oracle.permute(ridx, E)
    assert counts.sum() == T * k
    assert np.array_equal(offs.cpu().numpy(), roffs)
    assert np.array_equal(perm.cpu().numpy(), rperm)
    assert np.array_equal(inv.cpu().numpy(), rinv)
    # the layer output: every token, or a seeded subset with the first and last
    if n_sample is None or n_sample >= T:
        tokens = np.arange(T)
    else:
        rng = np.random.default_rng(1234)
        tokens = np.array(sorted(set([0, T - 1] + rng.choice(T, size=n_sample - 2, replace=False).tolist())))
    t0 = time.perf_counter()
    ref = parity.oracle_tokens_forward(inp, k, tokens, ridx[tokens], rw[tokens])
    t_oracle = time.perf_counter() - t0
    got = out[torch.as_tensor(tokens, device="cuda")]
    e = parity.assert_layer_close(got, ref, name)
    # per token as well, at twice the layer's mean-relative bar: one wrong tile
    # (a few tokens' rows of one expert) cannot hide in the workload's average
    g64 = parity.to_np64(got)
    tok_rel = np.abs(g64 - ref).sum(axis=1) / np.maximum(np.abs(ref).sum(axis=1), 1e-300)
    assert np.all(tok_rel <= 2 * parity.MEAN_REL), (name, int(tokens[tok_rel.argmax()]), float(tok_rel.max()))
    print(f"{name}: {len(tokens)} of {T} tokens compared, touched {int((counts > 0).sum())}, "
          f"max rows {int(counts.max())}, {e}, worst token mean rel {tok_rel.max():.3g}, weights max rel {w_err:.3g} (tol {w_tol:.3g}), "
          f"oracle {t_oracle:.1f} s")
    # deterministic: the same launch again gives the same bits
    out2 = lib.moe_forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    assert torch.equal(out, out2)
    del inp, out, out2
    torch.cuda.empty_cache()
