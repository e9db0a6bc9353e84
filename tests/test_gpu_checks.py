"""The index-checking build, libmoe_checks.so (a stand-in for a memory checker,
which is not available here): every data-dependent row or expert offset is
checked on the device before use; a bad one is recorded as
MOE_DEVERR_INDEX_CHECK and the access is skipped.

In a fresh process that loads that build (MOE_LIBRARY=checks):
  * forward passes over one-token, few-token, screened-router, 256-row-block
    and many-pair shapes record no error and give the same bits as the normal
    build (the checks change no arithmetic);
  * a combine whose row list points one past y_perm records the error and
    still returns, the context usable;
  * an expert feed-forward whose offsets claim more rows than it was given
    records the error and schedules no tile.
Bad indices go only to this build, whose checks guard the accesses."""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from sparse_mixture_experts_route_b200 import inputs as moe_inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(1, 7168, 896, 16, 512, None), (8, 1024, 8, 2, 128, None), (333, 320, 20, 3, 192, "zipf"),
          (600, 128, 4, 2, 128, None), (1200, 256, 16, 4, 128, None)]

CHILD = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    from sparse_mixture_experts_route_b200 import _lib as lib
    from sparse_mixture_experts_route_b200 import inputs as mi
    assert lib.LIB_PATH.endswith("libmoe_checks.so"), lib.LIB_PATH
    outs = []
    for (T, d, E, k, f, bias) in {shapes!r}:
        inp = mi.make_inputs(mi.custom_shape(T, d, E, k, f, bias=bias), seed=9, device="cuda")
        out = lib.moe_forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)
        torch.cuda.synchronize()
        assert lib.get_device_error() == 0, (T, d, E, k, f)
        outs.append(out.cpu())
    torch.save(outs, {path!r})
    # a combine row one past y_perm [T k, d]
    T, d, k = 5, 64, 3
    y = torch.randn(T * k, d, device="cuda").to(torch.bfloat16)
    inv = torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k).contiguous()
    inv[2, 1] = T * k
    w = torch.ones(T, k, device="cuda")
    out = lib.moe_unpermute(y, inv, w)
    torch.cuda.synchronize()
    assert lib.get_device_error(clear=True) == lib.DEVERR_INDEX_CHECK
    good = lib.moe_unpermute(y, torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k).contiguous(), w)
    torch.cuda.synchronize()
    assert torch.equal(out[0], good[0]) and torch.equal(out[4], good[4])
    # expert offsets claiming 40 rows of a 32-row x_perm
    E, d, f = 4, 128, 64
    x_perm = torch.randn(32, d, device="cuda").to(torch.bfloat16)
    offs = torch.tensor([0, 8, 16, 24, 40], dtype=torch.int32, device="cuda")
    Wgu = torch.randn(E, d, 2 * f, device="cuda").to(torch.bfloat16)
    Wd = torch.randn(E, f, d, device="cuda").to(torch.bfloat16)
    h0 = torch.full((32, f), 7.0, device="cuda").to(torch.bfloat16)
    y0 = torch.full((32, d), 7.0, device="cuda").to(torch.bfloat16)
    ws = torch.zeros(lib.expert_ffn_workspace_size(32, E), dtype=torch.uint8, device="cuda")
    st = lib.raw.moe_expert_ffn(x_perm.data_ptr(), offs.data_ptr(), Wgu.data_ptr(), Wd.data_ptr(), 32, d, E, f,
                                h0.data_ptr(), y0.data_ptr(), ws.data_ptr(), ws.numel(),
                                torch.cuda.current_stream().cuda_stream)
    assert st == lib.MOE_OK, st
    torch.cuda.synchronize()
    assert lib.get_device_error(clear=True) == lib.DEVERR_INDEX_CHECK
    assert bool((y0 == 7.0).all()) and bool((h0 == 7.0).all())   # no tile ran
    assert float(torch.ones(3, device="cuda").sum()) == 3.0        # the context is usable
    print("checks ok")
""")


def test_index_checking_build(tmp_path):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_mixture_experts_route_b200 import build
    build.build(checks=True)
    path = str(tmp_path / "outs.pt")
    env = dict(os.environ, MOE_LIBRARY="checks")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, shapes=SHAPES, path=path)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "checks ok" in r.stdout
    from sparse_mixture_experts_route_b200 import _lib as lib
    assert lib.LIB_PATH.endswith("libmoe.so")
    outs = torch.load(path)
    for (T, d, E, k, f, bias), got in zip(SHAPES, outs):
        inp = moe_inputs.make_inputs(moe_inputs.custom_shape(T, d, E, k, f, bias=bias), seed=9, device="cuda")
        want = lib.moe_forward(inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k).cpu()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), (T, d, E, k, f)
    assert lib.get_device_error() == 0
