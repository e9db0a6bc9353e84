"""Seeded synthetic workloads for the sparse Mixture-of-Experts layer forward pass.

This module is shared by the CUDA path's tests and bench and by the CPU oracle's
tests. It only draws random numbers and fixes shapes: it holds none of the
layer's arithmetic (no router, softmax, top-k, permutation, FFN or combine).

Shapes follow the model-card figures quoted on the pages:
  * "Kimi K3: What Open-Source Frontier Models Reveal About RL Scaling for
    Reasoning", section "The Architecture: MoE, Latent Attention, and Massive
    Context": 384 experts, 8 selected per token;
  * "Kimi K3: The Open Model That Just Cornered the AI Frontier", section
    "Mixture-of-Experts with Dynamic Load Balancing": 256 experts, top-4;
  * "Kimi K3: Open Frontier Intelligence", section "Operational Execution
    Flow": 896 routed experts, 16 active per token; hidden size 7168.

Distributions (one reading, stated once here):
  x         ~ N(0, 1), rounded to bf16 (round-to-nearest-even)
  W_router  ~ N(0, 0.02^2), fp32 (0.02 is the standard deviation)
  W_gate_up ~ N(0, 1/d), rounded to bf16, layout [E, d, 2f]
              (columns 0..f-1 feed the gate, f..2f-1 the up projection)
  W_down    ~ N(0, 1/f), rounded to bf16, layout [E, f, d]
  bias      (skewed workload only) b_e = 1.5 * ln(1 / rank_e), rank_e = e + 1

Each tensor draws from its own stream of one seed: x 0, W_router 1,
W_gate_up 2, W_down 3.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class MoEShape:
    """Sizes of one MoE layer invocation.

    T tokens, d model width, E experts, k experts per token, f expert hidden
    width. ``bias`` names the router bias recipe (None or "zipf").
    """

    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    bias: Optional[str] = None
    note: str = field(default="", compare=False)

    def with_T(self, T: int, name: Optional[str] = None) -> "MoEShape":
        return MoEShape(name or f"{self.name}_T{T}", T, self.d, self.E, self.k, self.f, self.bias, self.note)

    def flops(self) -> float:
        """Algorithmic FLOPs: router 2*T*d*E plus experts 6*T*k*d*f."""
        return 2.0 * self.T * self.d * self.E + 6.0 * self.T * self.k * self.d * self.f

    def as_dict(self) -> dict:
        return {"workload": self.name, "T": self.T, "d": self.d, "E": self.E, "k": self.k, "f": self.f,
                "router_bias": self.bias or "none"}


#: The workloads. "tiny" is small enough for the oracle in seconds; the rest
#: carry the model-card shapes.
WORKLOADS = {
    "tiny": MoEShape("tiny", 64, 128, 8, 2, 256, note="oracle-sized"),
    "prefill": MoEShape("prefill", 4096, 7168, 384, 8, 2048, note="384 experts top-8"),
    "decode": MoEShape("decode", 128, 7168, 256, 4, 2048, note="256 experts top-4"),
    "skewed": MoEShape("skewed", 8192, 7168, 896, 16, 512, bias="zipf", note="896 experts top-16, Zipf-like bias"),
}
#: Prefill-shaped but with 32 experts (2.8 GB of weights, still > L2): the
#: size used for full ncu captures of the kernels.
WORKLOADS["prefill_small"] = MoEShape("prefill_small", 1024, 7168, 32, 8, 2048, note="profiling size")
#: Skewed-shaped (Zipf-like bias, top-16) with 128 experts: 2.8 GB of weights.
WORKLOADS["skewed_small"] = MoEShape("skewed_small", 2048, 7168, 128, 16, 512, bias="zipf", note="profiling size")
#: Decode-shaped (T=128, top-4, f=2048) with 32 experts: 2.8 GB of bf16
#: weights, 0.75 GB in the MX format (both more than L2), for full ncu captures.
WORKLOADS["decode_small"] = MoEShape("decode_small", 128, 7168, 32, 4, 2048, note="profiling size")
#: One token, 16 of 64 experts at the sweep's widths: 1.4 GB of weights (more
#: than L2) for full ncu captures of the one-token step's kernels.
WORKLOADS["onetoken_small"] = MoEShape("onetoken_small", 1, 7168, 64, 16, 512, note="profiling size")
SWEEP_T = (1, 8, 32, 128, 512)
for _T in SWEEP_T:
    WORKLOADS[f"sweep_T{_T}"] = MoEShape(f"sweep_T{_T}", _T, 7168, 896, 16, 512, note="decode sweep")

STREAM_X, STREAM_WR, STREAM_WGU, STREAM_WD = 0, 1, 2, 3


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def zipf_bias(E: int) -> torch.Tensor:
    """Per-expert router bias b_e = 1.5 * ln(1 / (e + 1)), fp32 (Zipf-like load)."""
    e = torch.arange(E, dtype=torch.float64)
    return (1.5 * torch.log(1.0 / (e + 1.0))).to(torch.float32)


@dataclass
class MoEInputs:
    """One seeded draw of every operand of the layer, on one device."""

    shape: MoEShape
    x: torch.Tensor                 # [T, d] bf16
    W_router: torch.Tensor          # [d, E] fp32
    bias: Optional[torch.Tensor]    # [E] fp32 or None
    W_gate_up: torch.Tensor         # [E, d, 2f] bf16
    W_down: torch.Tensor            # [E, f, d] bf16


def make_x(shape: MoEShape, seed: int = 0, device="cpu") -> torch.Tensor:
    g = _gen(seed, STREAM_X, device)
    return torch.randn(shape.T, shape.d, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_router(shape: MoEShape, seed: int = 0, device="cpu") -> torch.Tensor:
    g = _gen(seed, STREAM_WR, device)
    return torch.randn(shape.d, shape.E, generator=g, device=device, dtype=torch.float32) * 0.02


def _randn_bf16(shape_t, std: float, g, device, chunk_rows: int = 64) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and rounded to bf16, one slab of the leading
    dimension at a time so a 20+ GB weight never needs an fp32 copy."""
    out = torch.empty(shape_t, dtype=torch.bfloat16, device=device)
    lead = shape_t[0]
    for s in range(0, lead, chunk_rows):
        e = min(lead, s + chunk_rows)
        tmp = torch.randn((e - s,) + tuple(shape_t[1:]), generator=g, device=device, dtype=torch.float32)
        tmp.mul_(std)
        out[s:e].copy_(tmp)
        del tmp
    return out


def make_experts(shape: MoEShape, seed: int = 0, device="cpu"):
    g2 = _gen(seed, STREAM_WGU, device)
    W_gate_up = _randn_bf16((shape.E, shape.d, 2 * shape.f), 1.0 / math.sqrt(shape.d), g2, device)
    g3 = _gen(seed, STREAM_WD, device)
    W_down = _randn_bf16((shape.E, shape.f, shape.d), 1.0 / math.sqrt(shape.f), g3, device)
    return W_gate_up, W_down


def make_inputs(shape: MoEShape, seed: int = 0, device="cpu") -> MoEInputs:
    """Draw x, W_router, bias, W_gate_up, W_down for ``shape`` on ``device``."""
    x = make_x(shape, seed, device)
    W_router = make_router(shape, seed, device)
    bias = zipf_bias(shape.E).to(device) if shape.bias == "zipf" else None
    W_gate_up, W_down = make_experts(shape, seed, device)
    return MoEInputs(shape, x, W_router, bias, W_gate_up, W_down)


def custom_shape(T: int, d: int, E: int, k: int, f: int, bias: Optional[str] = None, name: str = "custom") -> MoEShape:
    return MoEShape(name, T, d, E, k, f, bias)


def make_mx_values(shape_t, block_axis: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """bf16 test values for MX block quantisation, blocks of 32 along
    ``block_axis`` (-1 for activations, -2 for [.., K, N] weights): N(0, 1)
    draws, a quarter of the blocks shifted by a random power of two in
    [2^-140, 2^120] (so bf16 subnormals and huge magnitudes occur), one
    element in eight shrunk by 2^-[0, 24] (a wide range inside a block),
    one block in 32 set to zero, one element in 64 set to -0. Plain random
    numbers: no quantisation arithmetic."""
    g = _gen(seed, 7, "cpu")
    v = torch.randn(shape_t, generator=g, dtype=torch.float32)
    ax = block_axis % len(shape_t)
    vb = v.movedim(ax, -1)
    bshape = tuple(vb.shape[:-1]) + (vb.shape[-1] // 32, 1)
    e_blk = torch.randint(-140, 121, bshape, generator=g, dtype=torch.int32)
    shifted = torch.rand(bshape, generator=g) < 0.25
    zero_blk = torch.rand(bshape, generator=g) < 1.0 / 32
    vb = vb.reshape(tuple(vb.shape[:-1]) + (vb.shape[-1] // 32, 32))
    # ldexp in fp64 so 2^e itself never under- or overflows before rounding
    vd = vb.to(torch.float64) * torch.pow(2.0, torch.where(shifted, e_blk, 0).to(torch.float64))
    shrink = torch.rand(vd.shape, generator=g) < 0.125
    e_el = torch.randint(0, 25, vd.shape, generator=g, dtype=torch.int32).to(torch.float64)
    vd = torch.where(shrink, vd * torch.pow(2.0, -e_el), vd)
    vd = torch.where(zero_blk, torch.zeros_like(vd), vd)
    neg0 = torch.rand(vd.shape, generator=g) < 1.0 / 64
    vd = torch.where(neg0, torch.full_like(vd, -0.0), vd)
    out = vd.reshape(tuple(vb.shape[:-2]) + (-1,)).to(torch.bfloat16).movedim(-1, ax).contiguous()
    return out.to(device)


@dataclass
class LatentInputs:
    """One seeded draw of the Stable LatentMoE layer's operands."""

    shape: MoEShape                  # T, d (model width), E, k, f (routed expert width), bias
    l: int                           # latent width
    x: torch.Tensor                  # [T, d] bf16
    W_router: torch.Tensor           # [d, E] fp32
    bias: Optional[torch.Tensor]     # [E] fp32 or None
    W_dn: torch.Tensor               # [d, l] bf16
    W_up: torch.Tensor               # [l, d] bf16
    W_gate_up: torch.Tensor          # [E, l, 2f] bf16
    W_down: torch.Tensor             # [E, f, l] bf16
    gamma: torch.Tensor              # [l] fp32
    Ws_gate_up: Optional[torch.Tensor]   # [S, d, 2fs] bf16
    Ws_down: Optional[torch.Tensor]      # [S, fs, d] bf16


def make_latent_inputs(shape: MoEShape, l: int, S: int, fs: int, seed: int = 0, device="cpu") -> LatentInputs:
    """x and W_router as make_inputs (streams 0 and 1); W_dn ~ N(0, 1/d),
    W_up ~ N(0, 1/l), routed W_gate_up ~ N(0, 1/l) and W_down ~ N(0, 1/f),
    shared Ws_gate_up ~ N(0, 1/d) and Ws_down ~ N(0, 1/fs), all rounded to
    bf16; gamma = 1 + N(0, 0.1^2) fp32. Streams 4..10 of the seed."""
    d, E, f = shape.d, shape.E, shape.f
    x = make_x(shape, seed, device)
    W_router = make_router(shape, seed, device)
    bias = zipf_bias(E).to(device) if shape.bias == "zipf" else None
    W_dn = _randn_bf16((d, l), 1.0 / math.sqrt(d), _gen(seed, 4, device), device)
    W_up = _randn_bf16((l, d), 1.0 / math.sqrt(l), _gen(seed, 5, device), device)
    W_gate_up = _randn_bf16((E, l, 2 * f), 1.0 / math.sqrt(l), _gen(seed, 6, device), device)
    W_down = _randn_bf16((E, f, l), 1.0 / math.sqrt(f), _gen(seed, 7, device), device)
    gamma = 1.0 + 0.1 * torch.randn(l, generator=_gen(seed, 8, device), device=device, dtype=torch.float32)
    if S > 0:
        Ws_gate_up = _randn_bf16((S, d, 2 * fs), 1.0 / math.sqrt(d), _gen(seed, 9, device), device)
        Ws_down = _randn_bf16((S, fs, d), 1.0 / math.sqrt(fs), _gen(seed, 10, device), device)
    else:
        Ws_gate_up = Ws_down = None
    return LatentInputs(shape, l, x, W_router, bias, W_dn, W_up, W_gate_up, W_down, gamma, Ws_gate_up, Ws_down)


#: The Stable LatentMoE layer at the page's widths (d = 7168, l = 3584, 896
#: routed experts, 16 active, two shared experts); the expert widths are not
#: on the page: f = 512 for the routed experts (as in the other 896-expert
#: workloads) and fs = 2048 for the shared ones.
LATENT = {"shape": MoEShape("latent_prefill", 4096, 7168, 896, 16, 512, note="Stable LatentMoE"),
          "l": 3584, "S": 2, "fs": 2048}
