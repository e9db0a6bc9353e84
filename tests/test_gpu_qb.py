"""GPU parity of the Quantile Balancing half ("Kimi K3: Open Frontier
Intelligence", section "Systems Optimization, Load Balancing, and Post-Training
Alignment": per-expert biases from the (1 - k/n)-quantile of the routing
margins, recovered from binned histograms that data-parallel ranks add up).

Everything here is integer or decided in fp32, so it is compared bit for bit:
  * moe_router_logits against oracle.router_logits (the canonical fp32 order);
  * moe_qb_histogram's cutoffs alpha and counts H against
    oracle.qb_histogram_f32, the oracle's fp32-decision histogram (itself pinned
    against the fp64 definition in the CPU tests);
  * moe_qb_bias's bins against oracle.qb_quantile_bins, and its fp32 biases
    against -(lo + bin * w) evaluated in fp32 here, and within fp32 rounding of
    oracle.qb_bias_from_histogram (fp64).
The integer all-reduce between the two calls is the caller's; a sum of two
batches' histograms stands in for it here (the two-rank version runs on CPU
ranks in test_multirank_gloo.py)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_mixture_experts_route_b200 import _lib
    _lib.get_device_error(clear=True)
    return _lib


def _logits(lib, T, d, E, seed, bias=None):
    shape = moe_inputs.custom_shape(T, d, E, 2, 64, bias=bias)
    inp = moe_inputs.make_inputs(shape, seed=seed, device="cpu")
    b = inp.bias
    lg = lib.moe_router_logits(inp.x.cuda(), inp.W_router.cuda(), b.cuda() if b is not None else None)
    torch.cuda.synchronize()
    ref = oracle.router_logits(inp.x, inp.W_router, b)
    return lg, ref


# (T, d, E, bias): ragged last chunk (d % 128 = 64), E not a multiple of the
# 64-expert tile, 1024 experts, the model-width router with the Zipf bias
@pytest.mark.parametrize("shape", [(100, 320, 20, None), (513, 192, 1024, None), (300, 7168, 896, "zipf"),
                                   (1, 128, 2, None)], ids=lambda s: "x".join(map(str, s)))
def test_router_logits_bit_exact(lib, shape):
    T, d, E, bias = shape
    lg, ref = _logits(lib, T, d, E, seed=0, bias=bias)
    assert np.array_equal(lg.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert lib.get_device_error() == 0


def _hist_both(lib, lg_gpu, lg_cpu, bias, k, lo, hi, bins, H_gpu=None, H_cpu=None):
    alpha, H = lib.moe_qb_histogram(lg_gpu, bias.cuda() if bias is not None else None, k, lo, hi, bins, H=H_gpu)
    torch.cuda.synchronize()
    ralpha, rH = oracle.qb_histogram_f32(lg_cpu, k, lo, hi, bins,
                                         bias=bias.numpy() if bias is not None else None, H=H_cpu)
    assert np.array_equal(alpha.cpu().numpy().view(np.uint32), ralpha.view(np.uint32))
    assert np.array_equal(H.cpu().numpy(), rH)
    return alpha, H, rH


# (T, d, E, k, bins, lo, hi): the margins of these routers span about
# [-2, 1], [-3.1, 1.1], [-12, 4.4], [-1.1, 0.7] and [-1.5, 0.3]; [lo, hi) cuts
# both tails of the first four so the end bins collect the clamped margins;
# E > 256 takes the 32-value-per-lane cutoff kernel; bins = 1 counts every
# margin once; 1536 bins is the largest count
QB_SHAPES = [(1000, 256, 64, 4, 1000, -1.5, 0.5), (2048, 512, 384, 8, 1000, -2.5, 0.8),
             (777, 7168, 896, 16, 1000, -5.0, 1.0), (300, 128, 16, 3, 1, -1.0, 0.5),
             (5, 128, 1024, 16, 1536, -10.0, 10.0)]


@pytest.mark.parametrize("shape", QB_SHAPES, ids=lambda s: "x".join(map(str, s[:5])))
def test_qb_histogram_and_bins_bit_exact(lib, shape):
    T, d, E, k, bins, lo, hi = shape
    lg, ref = _logits(lib, T, d, E, seed=1)
    assert np.array_equal(lg.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    # current biases: a small seeded perturbation, as after earlier steps
    g = torch.Generator().manual_seed(7)
    bias = (torch.rand(E, generator=g, dtype=torch.float32) - 0.5) * 0.5
    alpha, H, rH = _hist_both(lib, lg, ref, bias, k, lo, hi, bins)
    assert np.all(rH.sum(axis=1) == T)          # every token counted once per expert
    b_bins, b_bias = lib.moe_qb_bias(H, lo, hi, T, k)
    torch.cuda.synchronize()
    rbins = oracle.qb_quantile_bins(rH, T, k)
    assert np.array_equal(b_bins.cpu().numpy(), rbins.astype(np.int32))
    # the fp32 bias of the stated arithmetic, evaluated in fp32 here
    f32 = np.float32
    w = f32(f32(hi) - f32(lo)) / f32(bins)
    want = -(f32(lo) + rbins.astype(np.float32) * w)
    assert np.array_equal(b_bias.cpu().numpy().view(np.uint32), want.astype(np.float32).view(np.uint32))
    # and within fp32 rounding of the oracle's fp64 update from the same counts
    rb = oracle.qb_bias_from_histogram(rH, lo, hi, T, k)
    np.testing.assert_allclose(b_bias.cpu().numpy(), rb, rtol=1e-6, atol=1e-6 * max(abs(lo), abs(hi)))
    assert lib.get_device_error() == 0


def test_qb_two_batches_add_into_one_histogram(lib):
    """Two batches counted into one H (what the caller's integer all-reduce
    does across ranks): the same counts as the oracle adding both, and the same
    bins as counting all tokens at once."""
    d, E, k, bins, lo, hi = 256, 128, 8, 1000, -6.0, 3.0
    lg1, ref1 = _logits(lib, 700, d, E, seed=2)
    lg2, ref2 = _logits(lib, 333, d, E, seed=3)
    bias = torch.zeros(E, dtype=torch.float32)
    _, H, rH = _hist_both(lib, lg1, ref1, bias, k, lo, hi, bins)
    _, H, rH = _hist_both(lib, lg2, ref2, bias, k, lo, hi, bins, H_gpu=H, H_cpu=rH)
    _, rH_all = oracle.qb_histogram_f32(np.concatenate([ref1, ref2]), k, lo, hi, bins, bias=bias.numpy())
    assert np.array_equal(rH, rH_all)
    b_bins, _ = lib.moe_qb_bias(H, lo, hi, 1033, k)
    torch.cuda.synchronize()
    assert np.array_equal(b_bins.cpu().numpy(), oracle.qb_quantile_bins(rH_all, 1033, k).astype(np.int32))


def test_qb_nan_margins_count_in_bin_zero(lib):
    """A token with k + 1 logits at +inf has cutoff +inf; those experts'
    margins are inf - inf = NaN and count in bin 0 on both sides, the others'
    are -inf (also bin 0); a finite token beside it is counted normally."""
    E, k, bins, lo, hi = 16, 3, 10, -4.0, 4.0
    g = torch.Generator().manual_seed(11)
    lg = torch.randn(2, E, generator=g, dtype=torch.float32)
    lg[0, [2, 5, 9, 14]] = float("inf")
    _, H, rH = _hist_both(lib, lg.cuda(), lg.numpy(), None, k, lo, hi, bins)
    assert np.all(rH[:, 0] >= 1)                 # token 0 lands in bin 0 for every expert
    assert np.all(rH.sum(axis=1) == 2)


def test_qb_steps_balance_a_skewed_router(lib):
    """QB iterated on the GPU from the Zipf-biased router: each step counts the
    margins under the current biases (bit-exact against the oracle) and takes
    the new biases from the quantile bins. The first step's biases lie within
    one bin of the oracle's exact update; after six steps the largest expert
    load is within 20% of T k / E (16x before the first step)."""
    T, d, E, k, bins, lo, hi = 4096, 512, 64, 4, 1000, -12.0, 4.0
    lg, ref = _logits(lib, T, d, E, seed=4, bias="zipf")

    def max_load(bias):
        top = np.argsort(-(ref.astype(np.float64) + bias), axis=1, kind="stable")[:, :k]
        return np.bincount(top.ravel(), minlength=E).max() / (T * k / E)

    b = torch.zeros(E, dtype=torch.float32)
    assert max_load(b.numpy()) > 10.0
    for step in range(6):
        _, H, _ = _hist_both(lib, lg, ref, b, k, lo, hi, bins)
        _, b_gpu = lib.moe_qb_bias(H, lo, hi, T, k)
        torch.cuda.synchronize()
        if step == 0:
            exact = oracle.qb_update(ref, k)
            width = (hi - lo) / bins
            # the histogram quantile is the lower edge of the exact quantile's bin
            got = b_gpu.cpu().numpy().astype(np.float64)
            assert np.all(got >= exact - 1e-5) and np.all(got <= exact + width + 1e-5)
        b = b_gpu.cpu()
    assert max_load(b.numpy().astype(np.float64)) < 1.2
    assert lib.get_device_error() == 0
