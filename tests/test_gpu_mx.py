"""GPU parity of the MX quantisers (moe_mxfp8_quantize, moe_mxfp4_quantize)
against the CPU oracle: every code and every scale byte must match bit for
bit. Inputs span the cases the format has: bf16 subnormals and magnitudes
near 2^120, all-zero blocks, -0, values that saturate (E4M3 above 448, E2M1
above 6 after scaling), exact ties between two codes, ragged grids (block
counts that are not a multiple of the launch's 256 threads), and a whole
expert stack quantised in one call."""
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


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.cpu().to(torch.float64).numpy()


MXFP8_SHAPES = [(1, 32), (67, 7168), (300, 2080), (5, 512)]


@pytest.mark.parametrize("shape", MXFP8_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_mxfp8_quantize_bit_exact(lib, shape):
    x = moe_inputs.make_mx_values(shape, -1, seed=11)
    codes, scales = lib.moe_mxfp8_quantize(x.cuda())
    torch.cuda.synchronize()
    rc, rs = oracle.mxfp8_quantize(_f64(x))
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert lib.get_device_error() == 0


def test_mxfp8_quantize_special_values(lib):
    """Hand-placed cases in one row of blocks: all zero, -0 only, a block whose
    maximum is the bf16 maximum, one made of bf16 subnormals, exact midpoints
    between E4M3 codes (ties to even), and values that saturate at 448."""
    bf = torch.bfloat16
    blocks = [
        torch.zeros(32),
        torch.full((32,), -0.0),
        torch.cat([torch.tensor([3.3895313892515355e38, -1.0, 2.0**100]), torch.ones(29)]),
        torch.tensor([2.0**-133 * (i + 1) for i in range(32)]),
        # amax 256 gives s = 0: 1 + 1/16 lies halfway between 1 and 1.125, 17 between 16 and 18
        torch.cat([torch.tensor([256.0, 1.0625, -1.0625, 1.1875, 17.0, 19.0, -2.0**-10, 3 * 2.0**-10]),
                   torch.zeros(24)]),
        # amax 510 (exact in bf16) gives s = 0 and elements beyond 448 saturate
        torch.cat([torch.tensor([510.0, 464.0, -480.0, 450.0]), torch.ones(28)]),
    ]
    x = torch.stack([torch.cat(blocks)]).to(bf)
    codes, scales = lib.moe_mxfp8_quantize(x.cuda())
    torch.cuda.synchronize()
    rc, rs = oracle.mxfp8_quantize(_f64(x))
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)
    got = codes.cpu().numpy()
    assert got[0, 32] == 0x80                 # -0 keeps its sign
    assert not np.any((got & 0x7F) == 0x7F)   # never a NaN code


def test_mxfp8_full_width_activations_sampled(lib):
    """The prefill activations [4096, 7168] in one launch; 96 rows checked
    against the oracle, and no NaN code anywhere."""
    shape = moe_inputs.WORKLOADS["prefill"]
    x = moe_inputs.make_x(shape, seed=0, device="cuda")
    codes, scales = lib.moe_mxfp8_quantize(x)
    torch.cuda.synchronize()
    rows = torch.randperm(shape.T, generator=torch.Generator().manual_seed(5))[:96].sort().values
    rc, rs = oracle.mxfp8_quantize(_f64(x[rows.cuda()]))
    assert np.array_equal(codes[rows.cuda()].cpu().numpy(), rc)
    assert np.array_equal(scales[rows.cuda()].cpu().numpy(), rs)
    assert not bool(((codes & 0x7F) == 0x7F).any())


MXFP4_SHAPES = [(32, 1), (64, 40), (1024, 2080), (96, 777)]


@pytest.mark.parametrize("shape", MXFP4_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_mxfp4_quantize_bit_exact(lib, shape):
    w = moe_inputs.make_mx_values(shape, -2, seed=13)
    codes, scales = lib.moe_mxfp4_quantize(w.cuda())
    torch.cuda.synchronize()
    rc, rs = oracle.mxfp4_quantize(w)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert int(codes.max()) <= 15
    assert lib.get_device_error() == 0


def test_mxfp4_quantize_expert_stack(lib):
    """[E, K, N] in one call equals each expert quantised on its own."""
    w = moe_inputs.make_mx_values((3, 256, 300), -2, seed=17)
    codes, scales = lib.moe_mxfp4_quantize(w.cuda())
    torch.cuda.synchronize()
    assert tuple(codes.shape) == (3, 256, 300) and tuple(scales.shape) == (3, 8, 300)
    for e in range(3):
        rc, rs = oracle.mxfp4_quantize(w[e])
        assert np.array_equal(codes[e].cpu().numpy(), rc)
        assert np.array_equal(scales[e].cpu().numpy(), rs)


def test_mxfp4_quantize_special_values(lib):
    """One column of blocks: all zero, -0 only, bf16 subnormals, ties between
    E2M1 codes after scaling (amax 4 gives s = 0: 2.5 lies between 2 and 3,
    5 between 4 and 6, 0.25 between 0 and 0.5), and saturation above 6."""
    col = torch.cat([
        torch.zeros(32),
        torch.full((32,), -0.0),
        torch.tensor([2.0**-133 * (i % 5) for i in range(32)]),
        torch.cat([torch.tensor([4.0, 2.5, -2.5, 3.5, 0.25, 0.75, -1.25, 1.75]), torch.zeros(24)]),
        torch.cat([torch.tensor([7.5, 5.0, -7.0, 6.5]), torch.ones(28)]),
    ]).reshape(-1, 1)
    w = torch.cat([col, -col], dim=1).to(torch.bfloat16).contiguous()
    codes, scales = lib.moe_mxfp4_quantize(w.cuda())
    torch.cuda.synchronize()
    rc, rs = oracle.mxfp4_quantize(w)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_mxfp4_full_size_expert_weights_sampled(lib):
    """Four experts' W_gate_up at the model width ([4, 7168, 4096], one call);
    24 columns of each expert checked against the oracle (blocks run down a
    column, so a column slice quantises on its own)."""
    shape = moe_inputs.custom_shape(1, 7168, 4, 1, 2048)
    w_gu, _ = moe_inputs.make_experts(shape, seed=3, device="cuda")
    codes, scales = lib.moe_mxfp4_quantize(w_gu)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(9)
    for e in range(4):
        cols = torch.randperm(4096, generator=g)[:24].sort().values.cuda()
        rc, rs = oracle.mxfp4_quantize(w_gu[e][:, cols].contiguous())
        assert np.array_equal(codes[e][:, cols].cpu().numpy(), rc)
        assert np.array_equal(scales[e][:, cols].cpu().numpy(), rs)
    assert int(codes.max()) <= 15
    assert lib.get_device_error() == 0
