"""GPU parity of the MX expert path: MXFP4 expert weights and MXFP8 activations,
the serving format of "Kimi K3: Open Frontier Intelligence", section "Systems
Optimization, Load Balancing, and Post-Training Alignment".

  * moe_mx_pack_experts against oracle.mxfp4_quantize, bit for bit: every E2M1
    code (unpacked from the two-per-byte K-major rows) and every E8M0 scale
    (read back out of the 512-byte atoms);
  * moe_forward_mx against the oracle's MX layer: the oracle's own routing,
    its own MXFP4 codes of each selected expert (never the GPU's), and
    oracle.expert_ffn_mx (x and h each take an MXFP8 round trip, fp64
    arithmetic between them), combined in slot order; layer tolerance.

Shapes run smallest first: one expert with one token tile, a few tiles, the
one-token step at full width (stream-K on both GEMMs), a few-token step whose
tiles are split over many CTAs, multi-tile experts through the many-pair
dispatch, and a decode-like step with whole-tile gate/up scheduling."""
from concurrent.futures import ThreadPoolExecutor
import os

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


def _unpack_codes(wq, E, N, K):
    """Packed rows [E][N][K/2] (element 2i in the low nibble of byte i) ->
    codes [E][K][N], the oracle's orientation."""
    b = wq.cpu().numpy().reshape(E, N, K // 2)
    codes = np.empty((E, N, K), dtype=np.uint8)
    codes[..., 0::2] = b & 0xF
    codes[..., 1::2] = b >> 4
    return codes.transpose(0, 2, 1)


def _unpack_scales(sf, E, N, K):
    """Scale atoms [E][N/128][K/128][512], row m and block kb of a 128 x 128
    tile at byte 16 (m % 32) + 4 (m / 32) + kb -> scales [E][K/32][N]."""
    a = sf.cpu().numpy().reshape(E, N // 128, K // 128, 512)
    n = np.arange(N)[None, :]
    kb = np.arange(K // 32)[:, None]
    off = 16 * (n % 32) + 4 * ((n % 128) // 32) + kb % 4
    return a[:, n // 128, kb // 4, off]


def _oracle_codes(W, experts, threads=None):
    """oracle.mxfp4_quantize of W[e] ([K, N] bf16 on any device) for each listed expert."""
    def one(e):
        return e, oracle.mxfp4_quantize(W[int(e)].cpu())
    with ThreadPoolExecutor(max_workers=threads or os.cpu_count() or 1) as ex:
        return dict(ex.map(one, experts))


@pytest.mark.parametrize("shape", [(2, 256, 128), (3, 512, 384), (1, 7168, 512)],
                         ids=lambda s: "x".join(map(str, s)))
def test_mx_pack_experts_bit_exact(lib, shape):
    E, d, f = shape
    inp = moe_inputs.make_inputs(moe_inputs.custom_shape(1, d, E, 1, f), seed=3, device="cuda")
    ex = lib.moe_mx_pack_experts(inp.W_gate_up, inp.W_down)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    gu_c = _unpack_codes(ex.wq_gate_up, E, 2 * f, d)
    gu_s = _unpack_scales(ex.sf_gate_up, E, 2 * f, d)
    dn_c = _unpack_codes(ex.wq_down, E, d, f)
    dn_s = _unpack_scales(ex.sf_down, E, d, f)
    ref_gu = _oracle_codes(inp.W_gate_up, range(E))
    ref_dn = _oracle_codes(inp.W_down, range(E))
    for e in range(E):
        assert np.array_equal(gu_c[e], ref_gu[e][0]), e
        assert np.array_equal(gu_s[e], ref_gu[e][1]), e
        assert np.array_equal(dn_c[e], ref_dn[e][0]), e
        assert np.array_equal(dn_s[e], ref_dn[e][1]), e


def _oracle_mx_forward(inp, k, ridx, rw):
    """The oracle's MX layer for every token: per selected expert, the oracle's
    MXFP4 codes of its weights and oracle.expert_ffn_mx of its rows."""
    T, d = inp.x.shape
    x = inp.x.cpu()
    experts = np.unique(ridx)
    gu = _oracle_codes(inp.W_gate_up, experts)
    dn = _oracle_codes(inp.W_down, experts)
    y = np.zeros((T * k, d), dtype=np.float64)

    def one(e):
        rows = np.argwhere(ridx == e)
        y[rows[:, 0] * k + rows[:, 1]] = oracle.expert_ffn_mx(x[torch.as_tensor(rows[:, 0])], *gu[e], *dn[e])

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(one, experts))
    return oracle.combine(y, np.arange(T * k, dtype=np.int32).reshape(T, k), rw)


MX_SHAPES = [
    # (T, d, E, k, f, bias)
    (4, 256, 1, 1, 128, None),        # one expert, one token tile, one feature tile
    (20, 256, 4, 2, 256, None),       # a few tiles
    (1, 7168, 896, 16, 512, None),    # the one-token step: stream-K on both GEMMs
    (8, 1024, 8, 2, 256, "zipf"),     # few tiles: every tile split over several CTAs
    (300, 512, 16, 4, 256, None),     # about 75 rows per expert, ragged tiles
    (800, 256, 8, 3, 128, None),      # 2400 pairs: many-pair dispatch, 3 tiles per expert
    (128, 1024, 64, 4, 2048, None),   # decode-like: whole-tile gate/up, stream-K down
]


@pytest.mark.parametrize("shape", MX_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + (f"_{s[5]}" if s[5] else ""))
def test_forward_mx_matches_oracle(lib, shape):
    T, d, E, k, f, bias = shape
    inp = moe_inputs.make_inputs(moe_inputs.custom_shape(T, d, E, k, f, bias=bias), seed=0, device="cuda")
    ex = lib.moe_mx_pack_experts(inp.W_gate_up, inp.W_down)
    out = lib.moe_forward_mx(inp.x, inp.W_router, inp.bias, ex, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    _, ridx, rw = parity.oracle_route(inp, k)
    ref = _oracle_mx_forward(inp, k, ridx, rw)
    e = parity.assert_layer_close(out, ref, f"forward_mx {shape}")
    print(shape, e)
    # a second call on a fresh workspace gives the same bits (stream-K tickets
    # return to zero; no order is decided by atomics)
    out2 = lib.moe_forward_mx(inp.x, inp.W_router, inp.bias, ex, k)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
