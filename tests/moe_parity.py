"""Comparison helpers shared by the GPU parity tests (no kernel arithmetic here).

Float tolerance for layer outputs, from the stated bar for bf16 inputs with
fp32 accumulation: max |out - ref| <= 1e-2 * max |ref| and mean relative error
sum |out - ref| / sum |ref| <= 5e-3 (the sum form, because a per-element
ratio is ill-conditioned where ref ~ 0).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

MAX_ABS_FRAC = 1e-2
MEAN_REL = 5e-3

# Router weights (the probabilities of the selected experts; the indices are
# compared bit for bit). Every router path except the many-token screen
# computes the exact-order fp32 logit of every expert, so its weights differ
# from the oracle's fp64 softmax of the same logits only by fp32 rounding: expf
# (2 ulp), the fp32 sum of at most 1024 terms taken as lane sums of <= 32 and a
# 5-level warp tree, and one division, about 2.5e-6 relative in all. 1e-5
# leaves a 4x margin.
W_RTOL = 1e-5
W_ATOL = 1e-7

# The many-token router (the library takes it when T >= 256, d % 64 == 0,
# d <= 8192 and E >= 16) screens the logits on tensor cores and recomputes the
# exact-order logit only for the experts inside a window around the k-th
# largest. The softmax denominator then sums exact terms for those candidates
# and screened terms exp(A_e - m) for the rest. The kernel's own error model
# (the one its window rests on) bounds each screened logit by
#   |A_e - L_e| <= delta_e = 2^-11 * sum_i |x_i W_ie| + 2^-20 * (max|A| + max|b| + 1).
# Every expert outside the window is outside the top-k, so with p the exact
# probabilities (the oracle's) the denominator's relative error is at most
#   beta = sum_{e not in top-k} p_e * (exp(delta_e) - 1),
# and each weight's relative error at most (beta + r) / (1 - beta - r) + r with
# r = W_RTOL covering the fp32 rounding above. screened_weight_rtol computes
# this bound per token on the CPU.
SCREEN_EPS_REL = 2.0 ** -11
SCREEN_EPS_ABS = 2.0 ** -20


def uses_screen(T: int, d: int, E: int) -> bool:
    """Whether the library routes this shape through the tensor-core screen."""
    return T >= 256 and d % 64 == 0 and d <= 8192 and E >= 16


def screened_weight_rtol(x, W_router, bias, logits, idx) -> np.ndarray:
    """Per-token relative bound on the screened router's weights (see above).

    x [T, d] bf16 and W_router [d, E] fp32 (CPU tensors), bias [E] or None,
    logits [T, E] the oracle's exact-order fp32 logits, idx [T, k] its top-k."""
    xa = torch.as_tensor(x).cpu().to(torch.float64).abs()
    wa = torch.as_tensor(W_router).cpu().to(torch.float64).abs()
    s_abs = (xa @ wa).numpy()                                 # sum_i |x_i W_ie|
    L = np.asarray(logits, dtype=np.float64)
    bmax = float(torch.as_tensor(bias).abs().max()) if bias is not None else 0.0
    amax = np.abs(L).max(axis=1) + SCREEN_EPS_REL * s_abs.max(axis=1)   # >= max_e |A_e|
    delta = SCREEN_EPS_REL * s_abs + SCREEN_EPS_ABS * (amax + bmax + 1.0)[:, None]
    p = np.exp(L - L.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    outside = np.ones_like(p, dtype=bool)
    np.put_along_axis(outside, np.asarray(idx, dtype=np.int64), False, axis=1)
    beta = (p * np.expm1(delta) * outside).sum(axis=1)
    r = W_RTOL
    return (beta + r) / (1.0 - beta - r) + r


def assert_route_weights(w, rw, x, W_router, bias, k, logits=None, idx=None, what=""):
    """Router weights against the oracle's: 1e-5 relative on the exact routers,
    the per-token bound above on the screened one. Returns the largest
    observed relative error and the tolerance applied (the largest, per token)."""
    w = to_np64(w)
    rw = np.asarray(rw, dtype=np.float64)
    T = w.shape[0]
    d, E = W_router.shape
    rel = np.abs(w - rw) / np.maximum(rw, 1e-300)
    if not uses_screen(T, d, E):
        np.testing.assert_allclose(w, rw, rtol=W_RTOL, atol=W_ATOL, err_msg=what)
        return float(rel.max()), W_RTOL
    if logits is None or idx is None:
        logits = oracle.router_logits(x, W_router, bias)
        idx, _ = oracle.topk(logits, k)
    tol = screened_weight_rtol(x, W_router, bias, logits, idx)
    bad = np.abs(w - rw) > tol[:, None] * rw + W_ATOL
    assert not bad.any(), (what, "screened weights outside the derived bound",
                           np.argwhere(bad)[:5], float(rel.max()), float(tol.min()))
    return float(rel.max()), float(tol.max())


def to_np64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def layer_error(out, ref) -> dict:
    o = to_np64(out)
    r = to_np64(ref)
    err = np.abs(o - r)
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    return {"max_abs": float(err.max()) if err.size else 0.0, "max_ref": scale,
            "mean_rel": float(err.sum() / max(np.abs(r).sum(), 1e-300)) if r.size else 0.0}


def assert_layer_close(out, ref, what=""):
    e = layer_error(out, ref)
    assert e["max_abs"] <= MAX_ABS_FRAC * e["max_ref"] + 1e-30, (what, e)
    assert e["mean_rel"] <= MEAN_REL, (what, e)
    return e


def oracle_route(inp, k, tokens=None):
    """Oracle steps 1-3 on CPU copies of the seeded inputs (all or some tokens):
    (logits, top-k indices, top-k weights)."""
    x = inp.x.cpu() if tokens is None else inp.x.cpu()[torch.as_tensor(tokens)]
    Wr = inp.W_router.cpu()
    b = inp.bias.cpu() if inp.bias is not None else None
    lg = oracle.router_logits(x, Wr, b)
    idx, w = oracle.topk(lg, k)
    return lg, idx, w


def oracle_tokens_forward(inp, k, tokens, idx, w, workers=None):
    """Oracle layer output [len(tokens), d] (fp64) for the listed tokens, given
    their oracle routing idx / w ([len(tokens), k]). Each selected expert's
    weights are fetched to the host on their own (full-size weights stay on the
    device) and its rows go through oracle.expert_ffn; experts run on a pool of
    host threads (the oracle releases the interpreter while it computes), then
    oracle.combine adds the k rows of each token in slot order."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    tokens = np.asarray(tokens, dtype=np.int64)
    idx = np.asarray(idx)
    n = len(tokens)
    d = inp.x.shape[1]
    x_sel = inp.x[torch.as_tensor(tokens, device=inp.x.device)].cpu()
    y = np.zeros((n * k, d), dtype=np.float64)

    def one_expert(e):
        rows = np.argwhere(idx == e)  # (token position, slot), ascending token
        ye = oracle.expert_ffn(x_sel[torch.as_tensor(rows[:, 0])], inp.W_gate_up[int(e)].cpu(),
                               inp.W_down[int(e)].cpu())
        y[rows[:, 0] * k + rows[:, 1]] = ye

    experts = np.unique(idx)
    # experts with many rows first, so one heavy expert does not finish last
    experts = experts[np.argsort(-np.bincount(idx.ravel())[experts], kind="stable")]
    with ThreadPoolExecutor(max_workers=workers or os.cpu_count() or 1) as ex:
        list(ex.map(one_expert, experts))
    inv = np.arange(n * k, dtype=np.int32).reshape(n, k)
    return oracle.combine(y, inv, np.asarray(w, dtype=np.float64))


def oracle_sampled_forward(inp, k, tokens):
    """Oracle layer output, routing indices and weights for the listed tokens only."""
    tokens = np.asarray(tokens, dtype=np.int64)
    _, idx, w = oracle_route(inp, k, tokens)
    return oracle_tokens_forward(inp, k, tokens, idx, w), idx, w
