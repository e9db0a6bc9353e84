"""GPU parity of every C-ABI step against the CPU oracle, on seeded inputs at
sizes the oracle finishes in seconds that still span several tiles and ragged
tails (partial router chunks, partial feature tiles, multi-block experts,
empty experts). Routing indices, counts, offsets and permutations are compared
bit for bit; floating-point outputs use the layer tolerance in parity.py."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_route_b200 import inputs as moe_inputs
import moe_parity as parity

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_mixture_experts_route_b200 import _lib
    _lib.get_device_error(clear=True)
    return _lib


def _inputs(T, d, E, k, f, seed=0, bias=None):
    shape = moe_inputs.custom_shape(T, d, E, k, f, bias=bias)
    return moe_inputs.make_inputs(shape, seed=seed, device="cpu")


def _cuda(inp):
    return type(inp)(inp.shape, inp.x.cuda(), inp.W_router.cuda(),
                     inp.bias.cuda() if inp.bias is not None else None,
                     inp.W_gate_up.cuda(), inp.W_down.cuda())


SHAPES = [
    # (T, d, E, k, f)
    (64, 128, 8, 2, 256),      # the tiny workload
    (333, 320, 20, 3, 192),    # ragged: last router chunk of 64, half feature tiles, 999 rows
    (1, 256, 16, 4, 128),      # a single token
    (2560, 256, 1024, 16, 64), # router without split (many tiles), 1024 experts
    (50, 128, 8, 8, 128),      # k = E
    (200, 192, 5, 1, 64),      # k = 1, E not a multiple of 4
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_route_bit_exact(lib, shape):
    T, d, E, k, f = shape
    inp = _inputs(T, d, E, k, f)
    g = _cuda(inp)
    idx, w = lib.moe_route(g.x, g.W_router, None, k)
    torch.cuda.synchronize()
    lg, ridx, rw = parity.oracle_route(inp, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    parity.assert_route_weights(w, rw, inp.x, inp.W_router, None, k, lg, ridx)
    assert lib.get_device_error() == 0


# The few-token router (T <= 16, E % 4 == 0): one launch that streams every
# chunk of W_router at once and reduces in the last CTAs (for one token with
# d <= 8192 a CTA per 8 experts walks all of d instead). Ragged last chunk
# (d % 128 == 64), partial last expert group (E % 128 != 0), one chunk only,
# k = E, 1024 experts, the full-width decode shape, and a bias.
STREAM_SHAPES = [
    # (T, d, E, k, bias)
    (1, 7168, 896, 16, None),
    (1, 7168, 896, 16, "zipf"),
    (3, 320, 20, 3, None),
    (4, 256, 200, 8, "zipf"),
    (5, 128, 1024, 16, None),
    (16, 448, 132, 4, None),
    (16, 64, 8, 8, None),
    (9, 7168, 384, 8, "zipf"),
    (2, 128, 6, 1, None),     # E % 4 != 0: the split-chunk router instead
    (1, 9216, 64, 4, "zipf"),  # one token with d > 8192: the chunk-partial one-token router
]


@pytest.mark.parametrize("shape", STREAM_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_route_few_tokens(lib, shape):
    T, d, E, k, bias = shape
    inp = _inputs(T, d, E, k, 64, bias=bias)
    g = _cuda(inp)
    for _ in range(2):  # the tickets return to zero: a second call reuses the workspace as is
        ws = torch.empty(lib.route_workspace_size(T, d, E), dtype=torch.uint8, device="cuda") if _ == 0 else ws
        idx, w = lib.moe_route(g.x, g.W_router, g.bias, k, workspace=ws)
        torch.cuda.synchronize()
        assert lib.get_device_error() == 0
        lg, ridx, rw = parity.oracle_route(inp, k)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        parity.assert_route_weights(w, rw, inp.x, inp.W_router, inp.bias, k, lg, ridx)


@pytest.mark.parametrize("T", [1, 6])
def test_route_all_equal_logits(lib, T):
    """All-zero tokens: every logit is 0, so all E = 896 experts tie. The
    histogram top-k sees more than 64 candidates and hands over to the
    arg-max rounds: experts 0..k-1 in order, each with weight 1/E."""
    d, E, k = 256, 896, 16
    x = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    Wr = torch.randn(d, E, dtype=torch.float32, device="cuda") * 0.02
    idx, w = lib.moe_route(x, Wr, None, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    assert idx.tolist() == [list(range(k))] * T
    np.testing.assert_allclose(w.cpu().numpy(), np.full((T, k), 1.0 / E), rtol=1e-6)


def test_route_few_tokens_ties_and_unaligned_weights(lib):
    """Exact ties and all-zero tokens on the few-token router; a W_router that is
    not 16-byte aligned (4-byte offset) takes the split-chunk router, same bits."""
    T, d, E, k = 6, 384, 12, 3
    inp = _inputs(T, d, E, k, 64)
    Wr = inp.W_router.clone()
    Wr[:, 7] = Wr[:, 2]
    x = inp.x.clone()
    x[1] = 0
    bias = torch.zeros(E, dtype=torch.float32)
    bias[5] = 0.25
    lg = oracle.router_logits(x, Wr, bias)
    ridx, rw = oracle.topk(lg, k)
    idx, w = lib.moe_route(x.cuda(), Wr.cuda(), bias.cuda(), k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    parity.assert_route_weights(w, rw, x, Wr, bias, k, lg, ridx)
    assert idx[1].tolist() == [5, 0, 1]
    store = torch.empty(d * E + 1, dtype=torch.float32, device="cuda")
    Wr_off = store[1:].view(d, E)
    Wr_off.copy_(Wr.cuda())
    assert Wr_off.data_ptr() % 16 != 0
    idx2, w2 = lib.moe_route(x.cuda(), Wr_off, bias.cuda(), k)
    assert torch.equal(idx2, idx)
    parity.assert_route_weights(w2, rw, x, Wr, bias, k, lg, ridx)
    assert lib.get_device_error() == 0


def test_route_bias_ties_zero_rows(lib):
    T, d, E, k, f = 96, 384, 12, 3, 64
    inp = _inputs(T, d, E, k, f)
    Wr = inp.W_router.clone()
    Wr[:, 7] = Wr[:, 2]            # exact ties between experts 2 and 7
    x = inp.x.clone()
    x[10] = 0                      # all-zero token: logits all 0 (+bias)
    x[11] = 0
    bias = torch.zeros(E, dtype=torch.float32)
    bias[5] = 0.25
    for b in (None, bias):
        idx, w = lib.moe_route(x.cuda(), Wr.cuda(), b.cuda() if b is not None else None, k)
        lg = oracle.router_logits(x, Wr, b)
        ridx, rw = oracle.topk(lg, k)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        parity.assert_route_weights(w, rw, x, Wr, b, k, lg, ridx)
    # the zero tokens with a bias on expert 5 pick 5 then 0, 1
    assert idx[10].tolist() == [5, 0, 1]


def test_route_zipf_bias_and_hot_expert(lib):
    T, d, E, k, f = 257, 256, 64, 4, 64
    inp = _inputs(T, d, E, k, f, bias="zipf")
    g = _cuda(inp)
    idx, w = lib.moe_route(g.x, g.W_router, g.bias, k)
    lg, ridx, rw = parity.oracle_route(inp, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    parity.assert_route_weights(w, rw, inp.x, inp.W_router, inp.bias, k, lg, ridx)
    hot = torch.zeros(E, dtype=torch.float32)
    hot[3] = 100.0
    idx, _ = lib.moe_route(g.x, g.W_router, hot.cuda(), k)
    assert torch.all(idx[:, 0] == 3)


@pytest.mark.parametrize("shape", [(64, 128, 8, 2, 256), (333, 320, 20, 3, 192), (2000, 128, 896, 16, 64),
                                   (1, 128, 4, 4, 64)], ids=lambda s: "x".join(map(str, s)))
def test_permute_bit_exact(lib, shape):
    T, d, E, k, f = shape
    inp = _inputs(T, d, E, k, f)
    _, ridx, _ = parity.oracle_route(inp, k)
    counts, offsets, perm_token, inv_perm = oracle.permute(ridx, E)
    x = inp.x.cuda()
    g_off, g_perm, g_inv, g_xp = lib.moe_permute(x, torch.from_numpy(ridx).cuda(), E)
    torch.cuda.synchronize()
    assert np.array_equal(g_off.cpu().numpy(), offsets)
    assert np.array_equal(g_perm.cpu().numpy(), perm_token)
    assert np.array_equal(g_inv.cpu().numpy(), inv_perm)
    assert torch.equal(g_xp.cpu(), inp.x[torch.from_numpy(perm_token).long()])
    assert lib.get_device_error() == 0


def test_permute_all_tokens_one_expert(lib):
    T, E, k = 700, 16, 1
    idx = torch.full((T, k), 9, dtype=torch.int32)
    x = torch.randn(T, 64).to(torch.bfloat16)
    off, perm, inv, xp = lib.moe_permute(x.cuda(), idx.cuda(), E)
    exp = [0] * 10 + [T] * 7
    assert off.cpu().tolist() == exp
    assert perm.cpu().tolist() == list(range(T))
    assert torch.equal(xp.cpu(), x)


def _ffn_check(lib, inp, k):
    E, f = inp.W_down.shape[0], inp.W_down.shape[1]
    _, ridx, rw = parity.oracle_route(inp, k)
    counts, offsets, perm_token, inv_perm = oracle.permute(ridx, E)
    x_perm = inp.x[torch.from_numpy(perm_token).long()]
    h, y = lib.moe_expert_ffn(x_perm.cuda(), torch.from_numpy(offsets).cuda(), inp.W_gate_up.cuda(),
                              inp.W_down.cuda())
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref_h = np.zeros((len(perm_token), f))
    ref_y = np.zeros((len(perm_token), inp.x.shape[1]))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        ye, he = oracle.expert_ffn(x_perm[a:b], inp.W_gate_up[e], inp.W_down[e], want_h=True)
        ref_h[a:b] = he
        ref_y[a:b] = ye
    parity.assert_layer_close(h, ref_h, "h")
    parity.assert_layer_close(y, ref_y, "y_perm")
    # per-expert as well, so one wrong expert cannot hide in the average
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            parity.assert_layer_close(y[a:b], ref_y[a:b], f"expert {e}")
    return h, y


@pytest.mark.parametrize("shape", [(64, 128, 8, 2, 256), (333, 320, 20, 3, 192), (1, 256, 16, 4, 128),
                                   (400, 128, 6, 2, 384), (600, 128, 4, 2, 256)],
                         ids=lambda s: "x".join(map(str, s)))
def test_expert_ffn(lib, shape):
    T, d, E, k, f = shape
    _ffn_check(lib, _inputs(T, d, E, k, f), k)


# Few output tiles: the gate/up GEMM splits K over 2 or 4 CTAs per tile and
# the last split adds the fp32 partials in order (f = 192: a half-empty
# feature tile). Two calls give identical bits (the tickets return to zero).
@pytest.mark.parametrize("shape", [(8, 1024, 8, 2, 128), (4, 2048, 16, 4, 256), (3, 1024, 8, 2, 192)],
                         ids=lambda s: "x".join(map(str, s)))
def test_expert_ffn_k_split(lib, shape):
    T, d, E, k, f = shape
    inp = _inputs(T, d, E, k, f)
    h, y = _ffn_check(lib, inp, k)
    _, ridx, _ = parity.oracle_route(inp, k)
    _, offsets, perm_token, _ = oracle.permute(ridx, E)
    x_perm = inp.x[torch.from_numpy(perm_token).long()]
    h2, y2 = lib.moe_expert_ffn(x_perm.cuda(), torch.from_numpy(offsets).cuda(), inp.W_gate_up.cuda(),
                                inp.W_down.cuda())
    assert torch.equal(h, h2) and torch.equal(y, y2)


def test_forward_one_token_full_width(lib):
    """T = 1 at d = 7168, E = 896, k = 16, f = 512 (the first decode-sweep point):
    few-token router, one-block dispatch, K-split gate/up GEMM."""
    T, d, E, k, f = 1, 7168, 896, 16, 512
    inp = _inputs(T, d, E, k, f)
    g = _cuda(inp)
    out = lib.moe_forward(g.x, g.W_router, None, g.W_gate_up, g.W_down, k)
    out2 = lib.moe_forward(g.x, g.W_router, None, g.W_gate_up, g.W_down, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    assert torch.equal(out, out2)
    ref, _, _ = oracle.forward(inp.x, inp.W_router, None, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(out, ref, "forward T=1")


def test_expert_ffn_hot_expert_multi_block(lib):
    # every token in expert 3 -> 300 rows = token blocks of 128, 128, 44; other experts empty
    T, d, E, k, f = 300, 128, 8, 1, 128
    inp = _inputs(T, d, E, k, f)
    inp.W_router.zero_()
    inp.W_router[:, 3] = 0.0
    b = torch.zeros(E)
    b[3] = 100.0
    inp = type(inp)(inp.shape, inp.x, inp.W_router, b, inp.W_gate_up, inp.W_down)
    _ffn_check(lib, inp, k)


def test_unpermute(lib):
    T, d, k = 77, 192, 3
    rows = T * k
    y = (torch.randn(rows, d) * 3).to(torch.bfloat16)
    inv = torch.randperm(rows).to(torch.int32).reshape(T, k)
    w = torch.rand(T, k, dtype=torch.float32)
    out = lib.moe_unpermute(y.cuda(), inv.cuda(), w.cuda())
    ref = oracle.combine(parity.to_np64(y), inv.numpy(), w.numpy().astype(np.float64))
    absref = oracle.combine(np.abs(parity.to_np64(y)), inv.numpy(), np.abs(w.numpy().astype(np.float64)))
    # fp32 fma chain of k terms, then one bf16 rounding
    gam = k * U32 / (1 - k * U32)
    bound = 2.0 ** -8 * np.abs(ref) + gam * absref * (1 + 2.0 ** -8) + 1e-30
    assert np.all(np.abs(parity.to_np64(out) - ref) <= bound)


# (600, 128, 4, 2, 128): about 300 rows per expert, so the gate/up GEMM takes
# 256-row token blocks (N = 256 MMAs) with partial remainders
# (32, 256, 2, 2, 128) and (33, ...): every expert has exactly T rows, one
# token block each with N = 32 and N = 48 MMAs
# (1, 128, 6, 2, 64): one token with E % 4 != 0, so the split-chunk router and
# the dispatch kernel run instead of the fused one-token path
@pytest.mark.parametrize("shape", SHAPES + [(300, 128, 8, 2, 128), (600, 128, 4, 2, 128), (32, 256, 2, 2, 128),
                                            (33, 256, 2, 2, 128), (1, 128, 6, 2, 64)],
                         ids=lambda s: "x".join(map(str, s)))
def test_forward(lib, shape):
    T, d, E, k, f = shape
    inp = _inputs(T, d, E, k, f)
    g = _cuda(inp)
    out = lib.moe_forward(g.x, g.W_router, None, g.W_gate_up, g.W_down, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref, ridx, rw = oracle.forward(inp.x, inp.W_router, None, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(out, ref, "forward")
    # the same call twice gives identical bits (no order decided by atomics)
    out2 = lib.moe_forward(g.x, g.W_router, None, g.W_gate_up, g.W_down, k)
    assert torch.equal(out, out2)


def test_forward_zipf_bias(lib):
    T, d, E, k, f = 256, 256, 64, 8, 128
    inp = _inputs(T, d, E, k, f, bias="zipf")
    g = _cuda(inp)
    out = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k)
    ref, _, _ = oracle.forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(out, ref, "forward zipf")


# Experts average more than 128 rows, so the gate/up GEMM takes 256-row
# blocks (both TMEM slots per tile), and the dispatch is the multi-block one.
# The Zipf-like bias gives experts with several full blocks and experts with
# a few rows side by side; f = 384 makes the down K six blocks, d = 320 a
# half-empty second output tile.
@pytest.mark.parametrize("shape", [(1500, 256, 16, 4, 384), (2100, 320, 12, 2, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_forward_heavy_and_light_experts(lib, shape):
    T, d, E, k, f = shape
    inp = _inputs(T, d, E, k, f, bias="zipf")
    _, ridx, _ = parity.oracle_route(inp, k)
    counts = np.bincount(ridx.ravel(), minlength=E)
    assert T * k > 2048 and T * k > 128 * E
    assert (counts >= 256).any() and ((counts > 0) & (counts < 256)).any(), counts
    g = _cuda(inp)
    out = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k)
    out2 = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    assert torch.equal(out, out2)
    ref, _, _ = oracle.forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(out, ref, "forward heavy and light experts")
    _ffn_check(lib, inp, k)


@pytest.mark.parametrize("shape", [(333, 320, 20, 3, 192), (600, 128, 4, 2, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_forward_host_buffers(lib, shape):
    """moe_forward_host: x and out in pinned host memory, copies inside the
    call; same bits as moe_forward, and within tolerance of the oracle.
    Two calls on two streams with their own workspaces give the same result."""
    T, d, E, k, f = shape
    inp = _inputs(T, d, E, k, f, bias="zipf")
    g = _cuda(inp)
    x_host = g.x.cpu().pin_memory()
    dev = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k)
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]
    outs = [lib.moe_forward_host(x_host, g.W_router, g.bias, g.W_gate_up, g.W_down, k, stream=st) for st in streams]
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    for o in outs:
        assert o.device.type == "cpu" and torch.equal(o, dev.cpu())
    ref, _, _ = oracle.forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(outs[0], ref, "forward host buffers")
    # a device pointer where host memory is required is refused
    with pytest.raises(lib.MoEError):
        ws = torch.empty(lib.moe_forward_host_workspace_size(T, d, E, k, f), dtype=torch.uint8, device="cuda")
        st = lib.raw.moe_forward_host(g.x.data_ptr(), g.W_router.data_ptr(), None, g.W_gate_up.data_ptr(),
                                      g.W_down.data_ptr(), T, d, E, k, f, outs[0].data_ptr(), ws.data_ptr(),
                                      ws.numel(), None)
        lib._check(st, "moe_forward_host")


def test_bounded_wait_reports_instead_of_hanging(lib):
    assert lib.get_device_error(clear=True) == 0
    lib.selftest_wait_timeout(2000)  # 2 ms on a barrier nothing signals
    assert lib.get_device_error(clear=True) == lib.DEVERR_SELFTEST_TIMEOUT
    assert lib.get_device_error(clear=True) == 0
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def test_python_binding_rejects_bad_tensors(lib):
    x = torch.zeros(4, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(TypeError):
        lib.moe_route(x, torch.zeros(128, 8, device="cuda"), None, 2)
    xb = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.MoEError):
        lib.moe_route(xb, torch.zeros(128, 8, device="cuda"), None, 9)


@pytest.mark.parametrize("E,k,bias_on", [(64, 8, False), (896, 16, True)])
def test_route_tensor_core_screen_ties_and_fallback(lib, E, k, bias_on):
    """Many tokens (the tensor-core screen + exact re-check router): exact ties
    from duplicated router columns, all-zero tokens (every logit equal, so the
    candidate window overflows and every expert is recomputed), and a bias."""
    T, d = 300, 512
    inp = _inputs(T, d, E, k, 64, bias="zipf" if bias_on else None)
    Wr = inp.W_router.clone()
    Wr[:, E - 1] = Wr[:, 1]
    Wr[:, E // 2] = Wr[:, 0]
    x = inp.x.clone()
    x[7] = 0
    x[299] = 0
    idx, w = lib.moe_route(x.cuda(), Wr.cuda(), inp.bias.cuda() if inp.bias is not None else None, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    lg = oracle.router_logits(x, Wr, inp.bias)
    ridx, rw = oracle.topk(lg, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    parity.assert_route_weights(w, rw, x, Wr, inp.bias, k, lg, ridx)


# Steps of at most 32 tokens run both GEMMs in one cooperative launch whose
# CTAs take K chunks of the tiles from a shared queue (down chunks wait for
# their expert's h rows). The staged entry points run the two GEMMs as two
# launches with their own K split. Both are checked against the oracle; the
# one-launch result must be the same bits on every call (each tile's chunk
# partials are added in chunk order whichever CTA computed them), also after a
# call of another shape has used the workspace, and it may differ from the
# staged result only by the order of the fp32 partial sums.
@pytest.mark.parametrize("shape", [(1, 7168, 896, 16, 512, None), (3, 1024, 8, 2, 192, "zipf"),
                                   (8, 2048, 64, 8, 256, None), (32, 512, 16, 4, 320, None),
                                   (17, 256, 4, 4, 128, None), (1, 256, 16, 4, 2048, None),
                                   (1, 9216, 16, 4, 128, None)],
                         ids=lambda s: "x".join(map(str, s[:5])) + (f"_{s[5]}" if s[5] else ""))
def test_forward_one_launch_ffn_matches_staged_steps(lib, shape):
    T, d, E, k, f, bias = shape
    inp = _inputs(T, d, E, k, f, bias=bias)
    g = _cuda(inp)
    T2 = 2 if T != 2 else 3
    ws = torch.empty(max(lib.moe_forward_workspace_size(T, d, E, k, f), lib.moe_forward_workspace_size(T2, d, E, k, f)),
                     dtype=torch.uint8, device="cuda")
    out = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k, workspace=ws)
    idx, w = lib.moe_route(g.x, g.W_router, g.bias, k)
    offs, perm, inv, xp = lib.moe_permute(g.x, idx, E)
    _, y = lib.moe_expert_ffn(xp, offs, g.W_gate_up, g.W_down)
    staged = lib.moe_unpermute(y, inv, w)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref, _, _ = oracle.forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(out, ref, "one-launch feed-forward")
    parity.assert_layer_close(staged, ref, "staged feed-forward")
    diff = (out.float() - staged.float()).abs()
    scale = staged.float().abs().amax(dim=1, keepdim=True).clamp_min(1e-30)
    assert float((diff / scale).max()) <= 2.0 ** -6, "one-launch and staged results differ beyond summation order"
    # another shape through the same workspace, then this one again: same bits
    lib.moe_forward(g.x[:1].repeat(T2, 1), g.W_router, g.bias, g.W_gate_up, g.W_down, k, workspace=ws)
    out2 = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k, workspace=ws)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("shape", [(1, 7168, 896, 16, 512, None), (1, 7168, 896, 16, 512, "zipf"),
                                   (1, 8192, 64, 1, 128, None), (1, 64, 20, 3, 64, None),
                                   (1, 1024, 12, 12, 192, None), (1, 2048, 1024, 16, 256, "zipf")],
                         ids=lambda s: "x".join(map(str, s[:5])) + (f"_{s[5]}" if s[5] else ""))
def test_one_token_single_launch_matches_separate_launches(lib, shape):
    """One token: moe_forward runs router, dispatch, both GEMMs and the combine
    in one cooperative launch; moe_forward_timed runs them as three launches
    (router, one-launch feed-forward, combine). Same arithmetic in the same
    order, so the same bits; both within the layer tolerance of the oracle.
    Shapes: the one-token decode step with and without a router bias, the
    largest d of the one-token router, a single 64-row chunk with E not a
    multiple of 8, k = E, and the most experts (128 router CTAs). A second
    call gives the same bits (the launch's counters are cleared each call)."""
    T, d, E, k, f, bias = shape
    inp = _inputs(T, d, E, k, f, bias=bias, seed=4)
    g = _cuda(inp)
    ws = torch.zeros(lib.moe_forward_workspace_size(T, d, E, k, f), dtype=torch.uint8, device="cuda")
    one = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k, workspace=ws).clone()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(lib.TIMED_STAGES))]
    three = torch.empty_like(one)
    lib.moe_forward_timed(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k, evs, three, ws)
    again = lib.moe_forward(g.x, g.W_router, g.bias, g.W_gate_up, g.W_down, k, workspace=ws)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref, _, _ = oracle.forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
    parity.assert_layer_close(one, ref, "one-token single launch")
    assert torch.equal(one.view(torch.int16), three.view(torch.int16)), "single launch differs from three launches"
    assert torch.equal(one.view(torch.int16), again.view(torch.int16))
