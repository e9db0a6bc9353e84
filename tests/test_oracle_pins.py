"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle step against something fixed independently:
hand-derived IEEE-754 values, closed forms, brute force on tiny inputs,
invariants the definition implies, or a library routine (numpy / scipy) that
computes the same well-defined quantity by other code. A plausible slip in the
oracle -- a dropped term, a swapped gate/up half, a wrong index, an unstable
sort, renormalised weights -- fails at least one of them
(``test_oracle_mutations.py`` plants such slips and checks that).

Passages: the gating code on "Kimi K3: The Open Model That Just Cornered the AI
Frontier" (section "Mixture-of-Experts with Dynamic Load Balancing") and the
routed-expert sum on "Kimi K3: Open Frontier Intelligence" (section
"Operational Execution Flow").
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
U32 = 2.0 ** -24  # unit roundoff of binary32


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _np_bf16_to_f64(t):
    return t.to(torch.float64).numpy()


def _silu(a):
    return a / (1.0 + np.exp(-a))


def _dense_swiglu(x64, Wgu64, Wd64):
    f = Wd64.shape[0]
    g = x64 @ Wgu64[:, :f]
    u = x64 @ Wgu64[:, f:]
    return (_silu(g) * u) @ Wd64


# ------------------------------------------------------------- router order

def _router_case(case):
    d, E = case["d"], case["E"]
    if case["x"] == "all 1.0":
        x = np.ones((1, d), dtype=np.float32)
    else:
        x = np.asarray(case["x"], dtype=np.float32).reshape(1, d)
    if isinstance(case["W"], str):
        W = np.ones((d, E), dtype=np.float32)
        W[0, 0] = 2.0 ** 24
    else:
        W = np.asarray(case["W"], dtype=np.float32).reshape(d, E)
    b = None if case["bias"] is None else np.asarray([case["bias"]] * E, dtype=np.float32)
    return x, W, b


def test_router_order_golden():
    data = json.load(open(os.path.join(GOLDEN, "router_order.json")))
    for case in data["cases"]:
        x, W, b = _router_case(case)
        got = oracle.router_logits(_bf16(x), W, b)
        assert got.shape == (1, case["E"])
        assert float(got[0, 0]) == case["expected"], (case["name"], float(got[0, 0]))
        for other in case["other_orders"].values():
            assert other != case["expected"]


def test_router_within_fp32_error_bound_of_exact_dot():
    """|l - l_exact| <= gamma_n * sum|x_i W_ie| (+ u*|b|) with n = 128 + chunks + 1.

    l_exact is the fp64 dot product from numpy; the bound is the textbook
    forward error of a recursive fp32 sum of fma terms (Higham, Accuracy and
    Stability of Numerical Algorithms, ch. 3).
    """
    rng = np.random.default_rng(7)
    for (T, d, E, use_bias) in [(5, 384, 33, False), (3, 7168, 64, True), (4, 200, 9, True)]:
        x = _bf16(rng.standard_normal((T, d)))
        W = (rng.standard_normal((d, E)) * 0.02).astype(np.float32)
        b = (rng.standard_normal(E) * 2).astype(np.float32) if use_bias else None
        got = oracle.router_logits(x, W, b).astype(np.float64)
        x64 = x.to(torch.float64).numpy()
        exact = x64 @ W.astype(np.float64)
        absd = np.abs(x64) @ np.abs(W.astype(np.float64))
        n = 128 + math.ceil(d / 128) + 1
        gamma = n * U32 / (1 - n * U32)
        bound = gamma * absd
        if b is not None:
            exact = exact + b
            bound = bound + gamma * np.abs(b) + U32 * np.abs(exact)
        assert np.all(np.abs(got - exact) <= bound), np.max(np.abs(got - exact) / bound)
        # and it is not the fp64 value rounded once (the order matters somewhere)
        assert got.dtype == np.float64


def test_router_rows_independent_and_bias_shift():
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((6, 256)))
    W = (rng.standard_normal((256, 10)) * 0.02).astype(np.float32)
    full = oracle.router_logits(x, W)
    for t in range(6):
        assert np.array_equal(oracle.router_logits(x[t:t + 1], W)[0], full[t])
    # a bias of exactly 0 changes nothing (x + 0 == x)
    assert np.array_equal(oracle.router_logits(x, W, np.zeros(10, np.float32)), full)


# ------------------------------------------------------------ softmax/top-k

def test_topk_golden_closed_forms():
    data = json.load(open(os.path.join(GOLDEN, "gate_topk.json")))
    for case in data["cases"]:
        if "logits" in case:
            lg = np.asarray(case["logits"], dtype=np.float32)[None]
        else:
            lg = np.log(np.asarray(case["logits_ln_of"], dtype=np.float64)).astype(np.float32)[None]
        idx, w = oracle.topk(lg, case["k"])
        assert idx[0].tolist() == case["idx"], case["name"]
        np.testing.assert_allclose(w[0], case["w"], rtol=1e-6, err_msg=case["name"])


def test_topk_vs_brute_force_sort_and_library_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(11)
    for (T, E, k) in [(50, 8, 2), (20, 384, 8), (10, 896, 16), (7, 5, 5)]:
        lg = (rng.standard_normal((T, E)) * 1.7).astype(np.float32)
        # plant exact ties
        lg[:, E // 2] = lg[:, 0]
        lg[0, :] = 0.25
        idx, w, probs = oracle.topk(lg, k, want_probs=True)
        ref_p = softmax(lg.astype(np.float64), axis=1)
        np.testing.assert_allclose(probs, ref_p, rtol=1e-13, atol=0)
        order = np.argsort(-lg.astype(np.float64), axis=1, kind="stable")[:, :k]
        assert np.array_equal(idx, order)
        np.testing.assert_allclose(w, np.take_along_axis(ref_p, order, 1), rtol=1e-13)
        np.testing.assert_allclose(probs.sum(1), 1.0, atol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 0)
        # weights are NOT renormalised: their sum is below 1 whenever k < E
        if k < E:
            assert np.all(w.sum(1) < 1.0)


# ------------------------------------------------------------------ permute

def test_permute_invariants_and_stable_sort():
    rng = np.random.default_rng(5)
    for (T, E, k) in [(64, 8, 2), (300, 37, 5), (1, 16, 16), (129, 896, 16)]:
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm_token, inv_perm = oracle.permute(idx, E)
        assert counts.sum() == T * k
        assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
        assert offsets[0] == 0 and offsets[-1] == T * k
        assert np.array_equal(np.diff(offsets), counts)
        # library stable sort of the flattened (t, j) pairs by expert
        order = np.argsort(idx.ravel(), kind="stable")
        assert np.array_equal(perm_token, order // k)
        inv_ref = np.empty(T * k, dtype=np.int64)
        inv_ref[order] = np.arange(T * k)
        assert np.array_equal(inv_perm.ravel(), inv_ref)
        # bijection and inverse
        assert np.array_equal(np.sort(inv_perm.ravel()), np.arange(T * k))
        assert np.array_equal(perm_token[inv_perm], np.repeat(np.arange(T), k).reshape(T, k))
        for e in range(E):
            seg = perm_token[offsets[e]:offsets[e + 1]]
            assert np.all(np.diff(seg) > 0)


def test_permute_then_combine_of_x_is_weight_sum_times_x():
    rng = np.random.default_rng(9)
    T, d, E, k = 40, 64, 6, 3
    x = _bf16(rng.standard_normal((T, d)))
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k))
    counts, offsets, perm_token, inv_perm = oracle.permute(idx, E)
    x64 = x.to(torch.float64).numpy()
    x_perm = x64[perm_token]
    out = oracle.combine(x_perm, inv_perm, w)
    np.testing.assert_allclose(out, w.sum(1)[:, None] * x64, rtol=1e-14, atol=1e-300)


# --------------------------------------------------------------- expert FFN

def test_expert_ffn_vs_numpy_matmul():
    rng = np.random.default_rng(13)
    for (n, d, f) in [(1, 64, 64), (37, 128, 256), (5, 256, 96)]:
        x = _bf16(rng.standard_normal((n, d)))
        Wgu = _bf16(rng.standard_normal((d, 2 * f)) / math.sqrt(d))
        Wd = _bf16(rng.standard_normal((f, d)) / math.sqrt(f))
        y, h = oracle.expert_ffn(x, Wgu, Wd, want_h=True)
        x64, Wg64, Wd64 = (_np_bf16_to_f64(t) for t in (x, Wgu, Wd))
        g = x64 @ Wg64[:, :f]
        u = x64 @ Wg64[:, f:]
        np.testing.assert_allclose(h, _silu(g) * u, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(y, _dense_swiglu(x64, Wg64, Wd64), rtol=1e-10, atol=1e-12)


def test_silu_closed_forms():
    # SiLU(0) = 0, SiLU(a) - SiLU(-a) = a, SiLU(ln 3) = 0.75 ln 3
    d, f = 4, 4
    Wgu = np.zeros((d, 2 * f), dtype=np.float32)
    Wd = np.eye(f, d, dtype=np.float32)
    Wgu[0, :f] = [0.0, 1.0, -1.0, 2.0]   # gate columns
    Wgu[1, f:] = 1.0                     # up columns = x[1]
    x = np.array([[1.0, 1.0, 0.0, 0.0]], dtype=np.float32)
    y = oracle.expert_ffn(_bf16(x), _bf16(Wgu), _bf16(Wd))
    s = lambda a: a / (1 + math.exp(-a))
    np.testing.assert_allclose(y[0], [0.0, s(1.0), s(-1.0), s(2.0)], rtol=1e-15)
    assert abs((y[0, 1] - y[0, 2]) - 1.0) < 1e-15
    # gate and up halves are not interchangeable: zero up half -> zero output
    Wgu2 = Wgu.copy()
    Wgu2[1, f:] = 0.0
    assert np.all(oracle.expert_ffn(_bf16(x), _bf16(Wgu2), _bf16(Wd)) == 0.0)


# ------------------------------------------------------------- whole layer

def _tiny_layer(E=8, k=2, T=64, d=128, f=256, seed=0, bias=None):
    shape = moe_inputs.custom_shape(T, d, E, k, f, bias=bias)
    return moe_inputs.make_inputs(shape, seed=seed)


def test_forward_E1_k1_is_dense_swiglu():
    inp = _tiny_layer(E=1, k=1, T=33, d=128, f=64)
    out, idx, w = oracle.forward(inp.x, inp.W_router, None, inp.W_gate_up, inp.W_down, 1)
    assert np.all(idx == 0) and np.all(w == 1.0)
    ref = _dense_swiglu(_np_bf16_to_f64(inp.x), _np_bf16_to_f64(inp.W_gate_up[0]), _np_bf16_to_f64(inp.W_down[0]))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_forward_identical_experts_is_prob_sum_times_ffn():
    inp = _tiny_layer(E=6, k=3, T=25, d=128, f=64)
    Wgu = inp.W_gate_up[:1].expand(6, -1, -1).contiguous()
    Wd = inp.W_down[:1].expand(6, -1, -1).contiguous()
    out, idx, w = oracle.forward(inp.x, inp.W_router, None, Wgu, Wd, 3)
    ffn = _dense_swiglu(_np_bf16_to_f64(inp.x), _np_bf16_to_f64(Wgu[0]), _np_bf16_to_f64(Wd[0]))
    np.testing.assert_allclose(out, w.sum(1)[:, None] * ffn, rtol=1e-10, atol=1e-12)


def test_forward_zero_token_and_hot_expert_and_duplicate_column():
    inp = _tiny_layer(E=8, k=2, T=16, d=128, f=64)
    x = inp.x.clone()
    x[5] = 0
    out, idx, w = oracle.forward(x, inp.W_router, None, inp.W_gate_up, inp.W_down, 2)
    assert idx[5].tolist() == [0, 1]
    np.testing.assert_allclose(w[5], [1 / 8, 1 / 8], rtol=1e-15)
    assert np.all(out[5] == 0.0)
    # +100 bias on expert 3: every token puts expert 3 in slot 0
    b = np.zeros(8, np.float32)
    b[3] = 100.0
    _, idx, w = oracle.forward(inp.x, inp.W_router, b, inp.W_gate_up, inp.W_down, 2)
    assert np.all(idx[:, 0] == 3)
    counts, *_ = oracle.permute(idx, 8)
    assert counts[3] == 16
    # duplicated router column: equal logits, the lower index ranks first
    Wr = inp.W_router.clone()
    Wr[:, 6] = Wr[:, 1]
    lg = oracle.router_logits(inp.x, Wr)
    assert np.array_equal(lg[:, 6], lg[:, 1])
    idx, _ = oracle.topk(lg, 3)
    for row in idx.tolist():
        if 6 in row:
            assert 1 in row and row.index(1) < row.index(6)


def test_tiny_workload_vs_numpy_cross_implementation():
    """Whole tiny layer (T=64, d=128, E=8, k=2, f=256, seed 0) against an
    independent numpy fp64 implementation with its own fp64 routing."""
    inp = moe_inputs.make_inputs(moe_inputs.WORKLOADS["tiny"], seed=0)
    k = 2
    out, idx, w = oracle.forward(inp.x, inp.W_router, None, inp.W_gate_up, inp.W_down, k)
    x64 = _np_bf16_to_f64(inp.x)
    lg = x64 @ inp.W_router.numpy().astype(np.float64)
    # the fp64 and fp32 routings agree wherever the k-th / (k+1)-th gap is
    # larger than the fp32 error bound; check that holds for this draw
    srt = np.sort(lg, axis=1)[:, ::-1]
    gap = srt[:, k - 1] - srt[:, k]
    assert np.all(gap > 1e-4)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    assert np.array_equal(order, idx)
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    wref = np.take_along_axis(p, order, 1)
    np.testing.assert_allclose(w, wref, rtol=1e-5)
    ref = np.zeros_like(x64)
    for t in range(x64.shape[0]):
        for j in range(k):
            e = order[t, j]
            ref[t] += wref[t, j] * _dense_swiglu(x64[t:t + 1], _np_bf16_to_f64(inp.W_gate_up[e]),
                                                  _np_bf16_to_f64(inp.W_down[e]))[0]
    np.testing.assert_allclose(out, ref, rtol=2e-5, atol=1e-7)


def test_forward_token_subset_matches_full():
    inp = moe_inputs.make_inputs(moe_inputs.WORKLOADS["tiny"], seed=0)
    full, idx, w = oracle.forward(inp.x, inp.W_router, None, inp.W_gate_up, inp.W_down, 2)
    sel = [0, 7, 63, 7]
    sub, sidx, sw = oracle.forward(inp.x, inp.W_router, None, inp.W_gate_up, inp.W_down, 2, tokens=sel)
    assert np.array_equal(sidx, idx[sel])
    np.testing.assert_allclose(sub, full[sel], rtol=1e-13, atol=1e-15)


def test_skewed_bias_recipe():
    b = moe_inputs.zipf_bias(896).numpy()
    assert b[0] == 0.0
    np.testing.assert_allclose(b[9], -1.5 * math.log(10.0), rtol=1e-6)
    assert np.all(np.diff(b) < 0)


def test_oracle_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.topk(np.zeros((2, 4), np.float32), 5)
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 9]], dtype=np.int32), 4)
    with pytest.raises(FloatingPointError):
        oracle.topk(np.array([[0.0, np.nan]], dtype=np.float32), 1)


# ------------------------------------------------------------ MXFP4 weights
#
# The serving format of the MoE weights on "Kimi K3: Open Frontier
# Intelligence" (section "Systems Optimization, Load Balancing, and
# Post-Training Alignment"), read as the OCP MX format. The expected values
# below are derived here from the bit fields of E2M1 (sign, two exponent bits
# with bias 1, one mantissa bit) and of the E8M0 scale, not from the oracle's
# table.

def _e2m1_value(code):
    sign = -1.0 if code & 8 else 1.0
    e, m = (code >> 1) & 3, code & 1
    mag = (m / 2.0) if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)  # subnormal when e == 0
    return sign * mag


def _bits_to_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def test_mxfp4_element_values_from_the_bit_fields():
    codes = np.arange(16, dtype=np.uint8).reshape(16, 1).repeat(2, axis=0)  # K = 32, N = 1
    for q, s in ((127, 0), (130, 3), (120, -7)):
        scales = np.full((1, 1), q, dtype=np.uint8)
        got = _bits_to_f64(oracle.mxfp4_dequantize(codes, scales))[:, 0]
        want = np.array([_e2m1_value(int(c)) * 2.0 ** s for c in codes[:, 0]])
        assert np.array_equal(got, want)
        assert np.array_equal(np.signbit(got), codes[:, 0] >= 8)  # -0 keeps its sign


def _brute_force_mxfp4(block):
    """Scale exponent and codes of one 32-value block by exhaustive search."""
    amax = max(abs(v) for v in block)
    s = -127 if amax == 0 else max(-127, min(127, math.frexp(amax)[1] - 1 - 2))
    codes = []
    for v in block:
        a = abs(v) / 2.0 ** s
        # the nearest of the eight magnitudes; on a tie the even code
        best = min(range(8), key=lambda c: (abs(a - abs(_e2m1_value(c))), c & 1))
        codes.append(best | (8 if math.copysign(1.0, v) < 0 else 0))
    return s, codes


def test_mxfp4_quantize_vs_brute_force_nearest_with_even_ties():
    g = torch.Generator().manual_seed(7)
    K, N = 96, 5
    w = (torch.randn(K, N, generator=g) * torch.tensor([1.0, 1e-3, 30.0, 1.0, 1.0])).to(torch.bfloat16)
    wf = w.to(torch.float64).numpy()
    # column 3: exact ties and saturating values on a scale of 2^0 (block max 6)
    wf[:32, 3] = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -2.5, -5.0, 0.0] + [0.1] * 20
    wf[32:64, 3] = [7.5, 7.0, 6.5] + [1.0] * 29          # max 7.5: scale 2^0, 7.5 and 7.0 saturate to 6
    wf[64:96, 3] = 0.0                                   # an all-zero block
    wf[:32, 4] = -0.0                                    # negative zeros
    w = torch.from_numpy(wf).to(torch.bfloat16)
    wf = w.to(torch.float64).numpy()
    codes, scales = oracle.mxfp4_quantize(w)
    for b in range(K // 32):
        for n in range(N):
            s, want = _brute_force_mxfp4(list(wf[32 * b:32 * b + 32, n]))
            assert int(scales[b, n]) == s + 127, (b, n)
            assert codes[32 * b:32 * b + 32, n].tolist() == want, (b, n)
    # the tie and saturation cases by hand: 0.25->0, 0.75->1, 1.25->1, 1.75->2,
    # 2.5->2, 3.5->4, 5->4 (ties to the even code); 7.5, 7.0, 6.5 -> 6
    deq = _bits_to_f64(oracle.mxfp4_dequantize(codes, scales))
    assert deq[:8, 3].tolist() == [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert deq[32:35, 3].tolist() == [6.0, 6.0, 6.0]
    assert int(scales[2, 3]) == 0 and not codes[64:96, 3].any()


def test_mxfp4_dequantised_values_requantise_to_themselves():
    g = np.random.default_rng(11)
    K, N = 128, 7
    codes = g.integers(0, 16, size=(K, N), dtype=np.uint8)
    scales = g.integers(100, 150, size=(K // 32, N), dtype=np.uint8)
    deq = oracle.mxfp4_dequantize(codes, scales)
    c2, s2 = oracle.mxfp4_quantize(deq)
    assert np.array_equal(_bits_to_f64(oracle.mxfp4_dequantize(c2, s2)), _bits_to_f64(deq))


def test_mxfp4_error_within_half_a_step():
    """|v - q(v)| is at most half the E2M1 spacing at |v| (0.25, 0.5 or 1 times
    the scale), or |v| - 6 * scale where v saturates."""
    g = torch.Generator().manual_seed(3)
    w = torch.randn(256, 16, generator=g).to(torch.bfloat16)
    wf = w.to(torch.float64).numpy()
    codes, scales = oracle.mxfp4_quantize(w)
    deq = _bits_to_f64(oracle.mxfp4_dequantize(codes, scales))
    scale = 2.0 ** (np.repeat(scales.astype(np.int64), 32, axis=0) - 127)
    a = np.abs(wf) / scale
    half_step = np.where(a < 2.0, 0.25, np.where(a < 4.0, 0.5, 1.0))
    bound = np.maximum(half_step, a - 6.0) * scale
    assert np.all(np.abs(wf - deq) <= bound)
    assert np.all(np.abs(wf).reshape(8, 32, 16).max(axis=1) / scale[::32] >= 4.0)  # block max lands in [4, 8)


# MXFP8 activations: E4M3 elements decoded and rounded by torch's own
# float8_e4m3fn type (a library implementation of the same format), E8M0 scale
# from frexp; saturation (which torch's cast does not do) by hand.

def test_mxfp8_element_values_match_torch_e4m3fn():
    codes = np.array([c for c in range(256) if (c & 0x7f) != 0x7f], dtype=np.uint8)
    codes = np.concatenate([codes, codes[:2]]).reshape(2, 128)  # 254 + 2 = 256 values, 32-aligned rows
    for q in (127, 131, 119):
        scales = np.full((2, 4), q, dtype=np.uint8)
        got = oracle.mxfp8_dequantize(codes, scales)
        want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy() * 2.0 ** (q - 127)
        assert np.array_equal(got, want)
        assert np.array_equal(np.signbit(got), codes >= 0x80)


def test_mxfp8_quantize_vs_torch_cast_and_saturation():
    g = torch.Generator().manual_seed(5)
    v = torch.randn(6, 64, generator=g, dtype=torch.float64)
    v[1] *= 1e-4
    v[2] *= 300.0
    v[3, :32] = 0.0
    v[4, :8] = torch.tensor([256.0, 0.5 * 2.0 ** -9, 1.5 * 2.0 ** -9, 3.0 * 2.0 ** -10, 452.0, 456.0, -460.0, 511.0])
    v[5, :32] = -0.0
    vn = v.numpy()
    codes, scales = oracle.mxfp8_quantize(vn)
    deq = oracle.mxfp8_dequantize(codes, scales)
    for r in range(6):
        for b in range(2):
            blk = vn[r, 32 * b:32 * b + 32]
            amax = np.abs(blk).max()
            s = -127 if amax == 0 else max(-127, min(127, math.frexp(amax)[1] - 1 - 8))
            assert int(scales[r, b]) == s + 127, (r, b)
            a = blk / 2.0 ** s
            inrange = np.abs(a) <= 448.0
            ref = torch.from_numpy(a[inrange].copy()).to(torch.float8_e4m3fn).to(torch.float64).numpy() * 2.0 ** s
            assert np.array_equal(deq[r, 32 * b:32 * b + 32][inrange], ref), (r, b)
            assert np.all(deq[r, 32 * b:32 * b + 32][~inrange] == np.sign(blk[~inrange]) * 448.0 * 2.0 ** s)
    # by hand, on a scale of 2^0 (block max 511): ties to the even code, saturation
    assert deq[4, :8].tolist() == [256.0, 0.0, 2.0 ** -8, 2.0 ** -8, 448.0, 448.0, -448.0, 448.0]
    assert int(scales[3, 0]) == 0 and not codes[3, :32].any()
    assert np.all(codes[5, :32] == 0x80)  # -0 keeps its sign


def test_mxfp8_dequantised_values_requantise_to_themselves():
    g = np.random.default_rng(13)
    codes = g.integers(0, 256, size=(8, 96), dtype=np.uint8)
    codes[(codes & 0x7f) == 0x7f] = 0x7e
    scales = g.integers(100, 150, size=(8, 3), dtype=np.uint8)
    deq = oracle.mxfp8_dequantize(codes, scales)
    assert np.array_equal(oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(deq)), deq)


def test_mx_expert_ffn_vs_numpy_composition():
    """The MX feed-forward equals its definition assembled here from the pinned
    pieces and numpy matmuls: x' and h' are MXFP8 round trips, W' the MXFP4
    dequantised weights, and the gate is the first f columns."""
    g = torch.Generator().manual_seed(9)
    n, d, f = 6, 96, 64
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    Wgu = (torch.randn(d, 2 * f, generator=g) / d ** 0.5).to(torch.bfloat16)
    Wd = (torch.randn(f, d, generator=g) / f ** 0.5).to(torch.bfloat16)
    gq = oracle.mxfp4_quantize(Wgu)
    dq = oracle.mxfp4_quantize(Wd)
    y, h = oracle.expert_ffn_mx(x, *gq, *dq, want_h=True)
    xq = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(x.to(torch.float64).numpy()))
    wgu = _bits_to_f64(oracle.mxfp4_dequantize(*gq))
    wd = _bits_to_f64(oracle.mxfp4_dequantize(*dq))
    gu = xq @ wgu
    hh = _silu(gu[:, :f]) * gu[:, f:]
    hq = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(hh))
    np.testing.assert_allclose(h, hq, rtol=0, atol=1e-12 * np.abs(hq).max())
    np.testing.assert_allclose(y, hq @ wd, rtol=0, atol=1e-12 * np.abs(hq @ wd).max())
    assert not np.allclose(hq, hh)  # the h round trip is not a no-op on these values


# ------------------------------------------------------------ Quantile Balancing
#
# The reading of "Kimi K3: Open Frontier Intelligence", section "Systems
# Optimization, Load Balancing, and Post-Training Alignment" (oracle_qb_* in
# moe_oracle.cpp): the bias update is the dual step of the balanced-assignment
# LP. The pins characterise each quantity by what it must satisfy, not by
# recomputing it the same way.

def _qb_scores(m, n, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(m, n)) + skew * np.log1p(np.arange(n))[::-1]


@pytest.mark.parametrize("m,n,k", [(40, 8, 2), (97, 16, 3), (5, 4, 3)])
def test_qb_cutoff_is_the_k_plus_first_biased_score(m, n, k):
    s = _qb_scores(m, n, 1)
    b = np.random.default_rng(2).normal(size=n) * 0.3
    a = oracle.qb_cutoffs(s, k, b)
    v = s + b
    # exactly k biased scores above the cutoff, and the cutoff is one of them
    assert np.all((v > a[:, None]).sum(1) == k)
    assert np.all(np.isclose(v, a[:, None], rtol=0, atol=0).sum(1) >= 1)


def _dual_obj(beta, mu, q):
    return q * beta + np.maximum(0.0, mu - beta).sum()


@pytest.mark.parametrize("m,n,k", [(40, 8, 2), (50, 8, 2), (97, 16, 3), (64, 64, 8)])
def test_qb_update_minimises_the_dual_over_each_expert_price(m, n, k):
    """For the cutoffs alpha, beta_j = -b_new_j minimises the LP dual's
    expert-j term q * beta + sum_i max(0, s_ij - alpha_i - beta), q = m k / n:
    a convex piecewise-linear function whose minimum lies at one of the
    margins, so a brute-force scan over all margins finds its minimum."""
    s = _qb_scores(m, n, 3, skew=0.5)
    b0 = np.random.default_rng(4).normal(size=n) * 0.2
    a = oracle.qb_cutoffs(s, k, b0)
    beta = -oracle.qb_update(s, k, b0)
    q = m * k / n
    for j in range(n):
        mu = s[:, j] - a
        best = min(_dual_obj(c, mu, q) for c in mu)
        assert _dual_obj(beta[j], mu, q) <= best + 1e-12
        # and beta_j is itself a margin (the quantile is an order statistic)
        assert np.any(mu == beta[j])


def test_qb_update_balances_a_skewed_router():
    """What the update is for: iterating it on scores with a strong per-expert
    skew brings the biased top-k loads close to the target m k / n."""
    m, n, k = 2000, 16, 2
    s = _qb_scores(m, n, 5, skew=2.0)

    def loads(b):
        top = np.argsort(-(s + b), axis=1, kind="stable")[:, :k]
        return np.bincount(top.ravel(), minlength=n)

    b = np.zeros(n)
    before = loads(b).max() / (m * k / n)
    for _ in range(20):
        b = oracle.qb_update(s, k, b)
    after = loads(b).max() / (m * k / n)
    assert before > 3.0
    assert after < 1.15


def test_qb_histogram_counts_and_quantile_within_one_bin():
    m, n, k = 300, 12, 3
    s = _qb_scores(m, n, 7, skew=0.3)
    a = oracle.qb_cutoffs(s, k)
    lo, hi, bins = -8.0, 8.0, 1000
    H = oracle.qb_histogram(s, a, lo, hi, bins)
    assert np.all(H.sum(1) == m)
    mu = s - a[:, None]
    assert np.all((mu >= lo) & (mu < hi))
    # bin edges: a margin at a bin's lower edge lands in that bin
    width = (hi - lo) / bins
    Hc = oracle.qb_histogram(np.array([[lo + 7 * width, lo], [hi + 1.0, lo - 1.0]]), np.zeros(2), lo, hi, bins)
    assert Hc[0, 7] == 1 and Hc[0, bins - 1] == 1 and Hc[1, 0] == 2
    exact = oracle.qb_update(s, k)
    approx = oracle.qb_bias_from_histogram(H, lo, hi, m, k)
    # the lower edge of the quantile's bin: beta_hist <= beta <= beta_hist + width
    assert np.all(approx >= exact - 1e-12)
    assert np.all(approx <= exact + width + 1e-12)


def test_qb_histograms_add_across_batches():
    """Counts of two halves of a batch add up to the counts of the whole (the
    property the integer all-reduce over data-parallel ranks relies on)."""
    m, n, k = 200, 8, 2
    s = _qb_scores(m, n, 9)
    a = oracle.qb_cutoffs(s, k)
    whole = oracle.qb_histogram(s, a, -6, 6, 100)
    H = oracle.qb_histogram(s[:77], a[:77], -6, 6, 100)
    oracle.qb_histogram(s[77:], a[77:], -6, 6, 100, H=H)
    assert np.array_equal(H, whole)
    assert np.array_equal(oracle.qb_bias_from_histogram(H, -6, 6, m, k),
                          oracle.qb_bias_from_histogram(whole, -6, 6, m, k))


def test_qb_fp32_histogram_matches_fp64_away_from_bin_edges():
    """The fp32-decision histogram (the GPU's arithmetic) counts what the fp64
    definition counts, except margins within fp32 rounding of a bin edge, which
    may move to the neighbouring bin."""
    m, n, k, lo, hi, B = 400, 12, 3, -8.0, 8.0, 1000
    for seed in range(4):
        s = np.random.default_rng(seed).normal(size=(m, n)).astype(np.float32)
        b = (np.random.default_rng(seed + 50).normal(size=n) * 0.25).astype(np.float32)
        a32, H32 = oracle.qb_histogram_f32(s, k, lo, hi, B, bias=b)
        # the cutoff: the (k+1)-th largest of the fp32 sums s + b
        v32 = s + b
        assert np.all((v32 > a32[:, None]).sum(1) == k) and np.all((v32 == a32[:, None]).sum(1) >= 1)
        H64 = oracle.qb_histogram(s.astype(np.float64), a32.astype(np.float64), lo, hi, B)
        assert np.all(H32.sum(1) == m) and np.all(H64.sum(1) == m)
        mu = s.astype(np.float64) - a32.astype(np.float64)[:, None]
        pos = B * (mu - lo) / (hi - lo)
        near = int((np.abs(pos - np.round(pos)) < 1e-4).sum())
        assert int(np.abs(H32 - H64).sum()) <= 2 * near
    # without a bias each token's cutoff expert has a margin of exactly 0, on a
    # bin edge here; both arithmetics put all m of them in the same bin
    s = np.random.default_rng(9).normal(size=(m, n)).astype(np.float32)
    a32, H32 = oracle.qb_histogram_f32(s, k, lo, hi, B)
    H64 = oracle.qb_histogram(s.astype(np.float64), a32.astype(np.float64), lo, hi, B)
    zero_bin = B // 2
    assert H32[:, zero_bin].sum() >= m and H64[:, zero_bin].sum() >= m
    assert H32[:, zero_bin - 1].sum() == H64[:, zero_bin - 1].sum()


def test_qb_quantile_bins_are_the_bias_bins():
    m, n, k, lo, hi, B = 300, 10, 2, -6.0, 6.0, 600
    s = np.random.default_rng(13).normal(size=(m, n))
    a = oracle.qb_cutoffs(s, k)
    H = oracle.qb_histogram(s, a, lo, hi, B)
    bins = oracle.qb_quantile_bins(H, m, k)
    bias = oracle.qb_bias_from_histogram(H, lo, hi, m, k)
    assert np.allclose(-bias, lo + bins * (hi - lo) / B, rtol=0, atol=1e-12)
    # at least ceil(m k / n) margins lie in or above the bin, fewer strictly above it
    r = -(-m * k // n)
    for j in range(n):
        assert H[j, bins[j]:].sum() >= r and H[j, bins[j] + 1:].sum() < r


# ------------------------------------------------------------ Stable LatentMoE
# "Kimi K3: Open Frontier Intelligence", section "Operational Execution Flow":
# shared experts on x, routed experts on a latent z = x W_dn, RMSNorm of the
# routed sum, W_up back to width d; SiTU-GLU with beta1 = 4, beta2 = 25 and
# |SiTU-GLU| <= 100. The page lost SiTU-GLU's formula (parity unpinned beyond
# what follows): pinned are the stated bound, the SwiGLU limit of large caps,
# RMSNorm's invariants, and the layer's reductions to the plain layer.

def _bf(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def test_glu_ffn_swiglu_matches_expert_ffn_and_numpy():
    g = torch.Generator().manual_seed(21)
    n, K, F = 5, 96, 40
    x = torch.randn(n, K, generator=g).to(torch.bfloat16)
    Wgu = (torch.randn(K, 2 * F, generator=g) / K ** 0.5).to(torch.bfloat16)
    Wd = (torch.randn(F, K, generator=g) / F ** 0.5).to(torch.bfloat16)
    y = oracle.glu_ffn(x, Wgu, Wd, act=oracle.ACT_SWIGLU)
    assert np.array_equal(y, oracle.expert_ffn(x, Wgu, Wd))          # the pinned step 5, same arithmetic
    xd, wg, wd = (t.to(torch.float64).numpy() for t in (x, Wgu, Wd))
    gu = xd @ wg
    ref = (gu[:, :F] / (1 + np.exp(-gu[:, :F])) * gu[:, F:]) @ wd
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


def test_situ_glu_bound_and_swiglu_limit():
    g = torch.Generator().manual_seed(22)
    n, K, F, N = 64, 32, 48, 16
    x = (torch.randn(n, K, generator=g, dtype=torch.float64) * 40.0).numpy()    # far past both caps
    Wgu = (torch.randn(K, 2 * F, generator=g) * 3.0).to(torch.bfloat16)
    Wd = torch.eye(F, N).to(torch.bfloat16)
    _, h = oracle.glu_ffn(x, Wgu, Wd, act=oracle.ACT_SITU, want_h=True)
    assert np.abs(h).max() <= oracle.SITU_BETA1 * oracle.SITU_BETA2           # the stated bound, 100
    assert np.abs(h).max() > 0.99 * 100.0                                       # and it is reached
    # huge caps: SiTU-GLU is SwiGLU (beta tanh(v / beta) -> v)
    x2 = torch.randn(n, K, generator=g, dtype=torch.float64).numpy()
    big = 1e150
    y_s = oracle.glu_ffn(x2, Wgu, Wd, act=oracle.ACT_SITU, beta1=big, beta2=big)
    y_w = oracle.glu_ffn(x2, Wgu, Wd, act=oracle.ACT_SWIGLU)
    np.testing.assert_allclose(y_s, y_w, rtol=1e-12, atol=1e-300)
    # zero gate row or zero second factor: exactly zero; sign follows SiLU(g) * v
    x0 = np.zeros((1, K))
    assert not np.any(oracle.glu_ffn(x0, Wgu, Wd, act=oracle.ACT_SITU))
    _, hs = oracle.glu_ffn(x2, Wgu, Wd, act=oracle.ACT_SITU, want_h=True)
    _, hw = oracle.glu_ffn(x2, Wgu, Wd, act=oracle.ACT_SWIGLU, want_h=True)
    assert np.array_equal(np.sign(hs), np.sign(hw))
    assert np.all(np.abs(hs) <= np.abs(hw) + 1e-15)                           # a cap never enlarges


def test_rmsnorm_invariants():
    rng = np.random.default_rng(23)
    u = rng.normal(size=(6, 40)) * rng.uniform(0.1, 10, size=(6, 1))
    r = oracle.rmsnorm(u, eps=0.0)
    np.testing.assert_allclose((r ** 2).mean(axis=1), 1.0, rtol=1e-12)       # unit RMS
    np.testing.assert_allclose(oracle.rmsnorm(7.25 * u, eps=0.0), r, rtol=1e-12)  # scale invariant
    assert np.array_equal(np.sign(r), np.sign(u))
    gamma = rng.uniform(0.5, 2.0, size=40).astype(np.float32)
    np.testing.assert_allclose(oracle.rmsnorm(u, gamma, eps=0.0), r * gamma.astype(np.float64), rtol=1e-12)
    assert not np.any(oracle.rmsnorm(np.zeros((2, 40)), eps=1e-6))            # zero row stays zero
    # eps: the denominator is sqrt(mean(u^2) + eps), so a row of RMS s shrinks by s / sqrt(s^2 + eps)
    s = np.sqrt((u[0] ** 2).mean())
    np.testing.assert_allclose(oracle.rmsnorm(u[:1], eps=0.5), r[:1] * s / np.sqrt(s * s + 0.5), rtol=1e-12)


def _latent_inputs(T, d, l, E, k, f, S, fs, seed, bias=None):
    shape = moe_inputs.custom_shape(T, d, E, k, f, bias=bias)
    inp = moe_inputs.make_inputs(shape, seed=seed)
    g = torch.Generator().manual_seed(seed + 100)
    Wdn = (torch.randn(d, l, generator=g) / d ** 0.5).to(torch.bfloat16)
    Wup = (torch.randn(l, d, generator=g) / l ** 0.5).to(torch.bfloat16)
    Wgu = (torch.randn(E, l, 2 * f, generator=g) / l ** 0.5).to(torch.bfloat16)
    Wd = (torch.randn(E, f, l, generator=g) / f ** 0.5).to(torch.bfloat16)
    Wsg = (torch.randn(S, d, 2 * fs, generator=g) / d ** 0.5).to(torch.bfloat16) if S else None
    Wsd = (torch.randn(S, fs, d, generator=g) / fs ** 0.5).to(torch.bfloat16) if S else None
    return inp, Wdn, Wup, Wgu, Wd, Wsg, Wsd


def test_latent_layer_with_identity_projections_is_rmsnorm_of_the_plain_layer():
    T, d, E, k, f = 40, 64, 8, 3, 32
    inp, *_ = _latent_inputs(T, d, d, E, k, f, 0, 0, seed=24, bias="zipf")
    eye = torch.eye(d).to(torch.bfloat16)
    out, u = oracle.latent_forward(inp.x, inp.W_router, inp.bias, eye, eye, inp.W_gate_up, inp.W_down, None,
                                   None, None, k, act=oracle.ACT_SWIGLU, eps=0.0, want_u=True)
    plain, _, _ = oracle.forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    np.testing.assert_allclose(u, plain, rtol=1e-12, atol=1e-14)              # the routed sum is the plain layer
    np.testing.assert_allclose(out, oracle.rmsnorm(plain, eps=0.0), rtol=1e-12, atol=1e-14)


def test_latent_layer_against_numpy_composition():
    """Projection, dispatch, combine, RMSNorm, W_up and the shared experts'
    sum, composed in numpy around the pinned pieces (router, top-k, GLU)."""
    T, d, l, E, k, f, S, fs = 33, 64, 48, 6, 2, 32, 2, 40
    inp, Wdn, Wup, Wgu, Wd, Wsg, Wsd = _latent_inputs(T, d, l, E, k, f, S, fs, seed=25)
    gamma = np.linspace(0.5, 1.5, l).astype(np.float32)
    out = oracle.latent_forward(inp.x, inp.W_router, None, Wdn, Wup, Wgu, Wd, gamma, Wsg, Wsd, k)
    x = inp.x.to(torch.float64).numpy()
    lg = oracle.router_logits(inp.x, inp.W_router, None)
    idx, w = oracle.topk(lg, k)
    z = x @ Wdn.to(torch.float64).numpy()
    u = np.zeros((T, l))
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            u[t] += w[t, j] * oracle.glu_ffn(z[t:t + 1], Wgu[e], Wd[e])[0]
    un = u / np.sqrt((u ** 2).mean(axis=1, keepdims=True) + 1e-6) * gamma.astype(np.float64)
    ref = un @ Wup.to(torch.float64).numpy()
    for s in range(S):
        ref += oracle.glu_ffn(x, Wsg[s], Wsd[s])
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_latent_layer_with_silent_routed_experts_is_the_shared_experts():
    T, d, l, E, k, f, S, fs = 20, 64, 32, 4, 2, 32, 2, 48
    inp, Wdn, Wup, Wgu, Wd, Wsg, Wsd = _latent_inputs(T, d, l, E, k, f, S, fs, seed=26)
    out = oracle.latent_forward(inp.x, inp.W_router, None, Wdn, Wup, torch.zeros_like(Wgu), Wd, None, Wsg, Wsd, k,
                                act=oracle.ACT_SWIGLU)
    ref = sum(oracle.expert_ffn(inp.x, Wsg[s], Wsd[s]) for s in range(S))   # pinned step 5 per shared expert
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
