"""Benchmark of the MoE layer forward pass (route -> dispatch -> SwiGLU experts ->
combine) on B200, printing one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores
    python bench.py --mx-quant             # the MXFP8 / MXFP4 quantisers alone

A step is one moe_forward over one batch of T synthetic tokens with the
workload's weights resident in HBM. Timing: W untimed warm-up steps, then K
steps, each between CUDA events on the launching stream, with an L2 flush
(a write larger than L2) between steps outside the events; barrier and
synchronize on both sides; the max over ranks. Under torchrun every rank is an
independent replica with its own tokens (weak scaling, no data-path
collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_route_b200 import inputs as moe_inputs  # noqa: E402

METRIC = "moe_layer_tokens_per_s"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5.0:  # first sample before the timed region
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() in ("active", "1"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- algorithmic

def algorithmic(shape: moe_inputs.MoEShape, counts: np.ndarray):
    """F_alg and B_alg of one layer pass, plus the dominant kernel's bytes.

    F_alg = 2*T*d*E (router) + 6*T*k*d*f (experts)
    B_alg = 4*d*E (W_router) + 2*T*d*2 (x in, out) + n_touched*6*d*f (expert
            weights of experts with at least one row) + 4*E (bias, if any)
    gate/up GEMM kernel (the dominant one), per launch: the per-unit figure of
            that step, 2*d*f*2 bytes of gate and up weights per touched expert,
            times the experts one launch touches. The rows it reads and the h
            it writes (T*k*d*2 + T*k*f*2 bytes) are the materialised
            intermediates of this implementation, reported beside it.
    """
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    n_touched = int((counts > 0).sum())
    F = 2.0 * T * d * E + 6.0 * T * k * d * f
    B = 4.0 * d * E + 4.0 * T * d + n_touched * 6.0 * d * f + (4.0 * E if shape.bias else 0.0)
    gu_bytes = n_touched * 4.0 * d * f
    gu_impl_bytes = 2.0 * T * k * d + 2.0 * T * k * f
    gu_flops = 4.0 * T * k * d * f
    return {"F": F, "B": B, "n_touched": n_touched, "gu_bytes": gu_bytes, "gu_impl_bytes": gu_impl_bytes,
            "gu_flops": gu_flops, "ffn_bytes": n_touched * 6.0 * d * f, "ffn_flops": 6.0 * T * k * d * f}


# Steps of at most this many tokens run both expert GEMMs in one launch
# (the library's one-launch feed-forward): the gate/up stage then times both.
FUSED_FFN_MAX_TOKENS = 32
ONE_TOKEN_MAX_D = 8192  # one-token steps up to this width run the whole layer in one launch


def count_library_launches(step) -> int:
    """Kernels of this library (namespace moe::) that one step launches, counted
    with the torch profiler on an untimed step."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize()
    return sum(1 for ev in prof.events() if ev.device_type.name == "CUDA" and "moe::" in ev.name)


def kernel_source_digest() -> str:
    p = os.path.join(ROOT, "sparse_mixture_experts_route_b200", "csrc", "expert_gemm.cuh")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def profiled_traffic(workload: str):
    """dram read+write bytes per launch of the gate/up GEMM from a committed ncu
    summary, only if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "gemm_gate_up_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except ValueError:
        return None
    ent = d.get(workload)
    if not ent or ent.get("kernel_sha") != kernel_source_digest():
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------ CPU baseline

def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_pass(inp, shape, tokens, threads: int):
    """The oracle, as it stands, over the listed tokens: router and top-k,
    every selected (token, expert) row through the expert's SwiGLU block, and
    the weighted combine. Experts run on a pool of `threads` host threads in
    groups of `threads`; each group's weights are fetched from the device
    before its timed region, so only oracle arithmetic is timed. Returns
    (seconds, expert rows, expert FLOPs, expert seconds)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    d, k, f = shape.d, shape.k, shape.f
    xs = inp.x[torch.as_tensor(tokens, device=inp.x.device)].cpu()
    Wr = inp.W_router.cpu()
    b = inp.bias.cpu() if inp.bias is not None else None
    t0 = time.perf_counter()
    lg = oracle.router_logits(xs, Wr, b)
    idx, w = oracle.topk(lg, k)
    t_route = time.perf_counter() - t0
    n = len(tokens)
    y = np.zeros((n * k, d), dtype=np.float64)
    experts = np.unique(idx)
    t_ffn = 0.0
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for g0 in range(0, len(experts), threads):
            group = experts[g0:g0 + threads]
            wts = {int(e): (inp.W_gate_up[int(e)].cpu(), inp.W_down[int(e)].cpu()) for e in group}

            def one(e):
                rows = np.argwhere(idx == e)
                y[rows[:, 0] * k + rows[:, 1]] = oracle.expert_ffn(xs[torch.as_tensor(rows[:, 0])], *wts[int(e)])

            t1 = time.perf_counter()
            list(ex.map(one, group))
            t_ffn += time.perf_counter() - t1
            del wts
    t2 = time.perf_counter()
    oracle.combine(y, np.arange(n * k, dtype=np.int32).reshape(n, k), w)
    t_comb = time.perf_counter() - t2
    return t_route + t_ffn + t_comb, n * k, 6.0 * n * k * d * f, t_ffn


def sample_tokens(T: int, n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=min(n, T), replace=False))


def calibrate_tokens(inp, shape, budget_s: float, threads: int, cap: int = 1024) -> int:
    """Tokens per oracle pass so that one pass takes about budget_s: a first
    untimed pass over 8 tokens sets the per-token cost."""
    t8, _, _, _ = oracle_pass(inp, shape, sample_tokens(shape.T, 8, 99), threads)
    per_tok = t8 / min(8, shape.T)
    return int(max(1, min(shape.T, cap, budget_s / max(per_tok, 1e-9))))


def cpu_baseline(inp, shape, budget_s: float = 20.0, seed: int = 1):
    """The oracle on a bounded sample of the workload, on this host's cores:
    one complete pass over a seeded sample of tokens sized to take about
    budget_s; tokens/s = sampled tokens / oracle seconds."""
    import oracle
    threads = oracle.num_threads()
    n = calibrate_tokens(inp, shape, budget_s, threads)
    secs, rows, ffn_flops, ffn_s = oracle_pass(inp, shape, sample_tokens(shape.T, n, seed), threads)
    return {"value": n / secs, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"one oracle pass (router, top-k, {rows} expert rows, combine) over {n} seeded tokens "
                      f"of {shape.name}; tokens/s = {n} / oracle seconds (weights fetched to host untimed)",
            "seconds": secs, "tokens": n, "cpu_model": cpu_model(),
            "fp64_gflops": ffn_flops / ffn_s / 1e9 if ffn_s > 0 else None}


# ------------------------------------------------------------------ arms

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _collective_device():
    import torch.distributed as dist
    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time (a timing reduction, not a data-path collective)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=_collective_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_x_seed(rank: int) -> int:
    """Seed of a replica's tokens: rank 0 uses the workload's seed 0, every other
    rank its own stream, so replicas route different tokens (weak scaling)."""
    return 0 if rank == 0 else 1000 + rank


def aggregate_tokens_per_s(T: int, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * T * steps / (max_total_ms / 1e3)


class L2Flush:
    """Between timed steps: write a buffer twice the size of L2, then read
    another one, so the dirty lines are written back here and not inside the
    next timed step."""

    def __init__(self, dev):
        self.w = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self, s):
        self.w.fill_(float(s))
        self.r.amax()


def time_layer(_lib, shape, inp, steps: int, warmup: int, graph_on: bool, world: int, flush, local: int,
               count_launches: bool = False):
    """Times `steps` moe_forward steps of one workload (after `warmup`), each
    between CUDA events on the launching stream with an L2 flush outside the
    events; replays of one step captured as a CUDA graph when graph_on. The
    per-stage times (and so the dominant kernel's duration) come from eager
    moe_forward_timed steps, since events cannot time nodes inside a replay."""
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    ws = torch.empty(_lib.moe_forward_workspace_size(T, d, E, k, f), dtype=torch.uint8, device=inp.x.device)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=inp.x.device)
    stream = torch.cuda.current_stream()
    args = (inp.x, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k)

    # routing statistics of this batch (for the algorithmic byte counts)
    idx, _ = _lib.moe_route(inp.x, inp.W_router, inp.bias, k)
    offs, _, _, _ = _lib.moe_permute(None, idx, E, with_rows=False)
    counts = np.diff(offs.cpu().numpy())
    alg = algorithmic(shape, counts)

    nst = len(_lib.TIMED_STAGES)
    launches = count_library_launches(lambda: _lib.moe_forward(*args, out=out, workspace=ws)) \
        if count_launches else None
    for _ in range(warmup):
        flush(1)
        _lib.moe_forward(*args, out=out, workspace=ws)
    assert _lib.get_device_error() == 0, "device error during warm-up"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 + 2 * nst)] for _ in range(steps)]
    for row in evs:
        for ev in row:
            ev.record(stream)
    graph = None
    if graph_on:
        # one step captured as a CUDA graph (the library never allocates or
        # synchronises, so its launches capture as they are)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            _lib.moe_forward(*args, out=out, workspace=ws)
            with torch.cuda.graph(graph, stream=side):
                _lib.moe_forward(*args, out=out, workspace=ws)
        stream.wait_stream(side)
        for _ in range(warmup):
            flush(1)
            graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for s in range(steps):
        flush(s)                                  # L2 flush, outside the step's events
        evs[s][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            _lib.moe_forward_timed(*args, evs[s][2:], out, ws)
        evs[s][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    step_ms = [evs[s][0].elapsed_time(evs[s][1]) for s in range(steps)]
    if graph is not None:
        n_eager = min(steps, 5)
        _lib.moe_forward_timed(*args, evs[0][2:], out, ws)
        for s in range(n_eager):
            flush(s)
            _lib.moe_forward_timed(*args, evs[s][2:], out, ws)
        torch.cuda.synchronize()
        stage_steps = range(n_eager)
    else:
        stage_steps = range(steps)
    stage_ms = {name: [evs[s][2 + 2 * i].elapsed_time(evs[s][3 + 2 * i]) for s in stage_steps]
                for i, name in enumerate(_lib.TIMED_STAGES)}
    total_ms = max_over_ranks(sum(step_ms), world)
    assert _lib.get_device_error() == 0, "device error during timing"
    del graph
    return {"total_ms": total_ms, "step_ms": step_ms, "stage_ms": stage_ms, "alg": alg, "clocks": clk,
            "launches": launches, "out": out, "ws": ws, "counts": counts}


def layer_summary(shape, res, steps: int, world: int, peaks: dict) -> dict:
    """Throughput and roofline figures of one timed workload."""
    T, k, E = shape.T, shape.k, shape.E
    alg = res["alg"]
    ms_per_step = res["total_ms"] / steps
    t_step = ms_per_step / 1e3
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    gu_ms = statistics.mean(res["stage_ms"]["gemm_gate_up"])
    layer_roof_s = max(alg["F"] / (tc * 1e12), alg["B"] / (hbm * 1e9))
    if T == 1 and shape.d <= ONE_TOKEN_MAX_D:
        # the step is one launch (moe_one_token_kernel) plus an 8-byte memset;
        # the per-stage times above come from the three-launch form
        gu_ms = ms_per_step
        dom = {"kernel": "moe_one_token_kernel (router, top-k, both GEMMs and the combine, one launch)",
               "bytes": alg["B"], "flops": alg["F"],
               "rule": "the layer's bytes: W_router fp32 + touched experts x 6*d*f + x and out (per step, "
                       "which also holds the 8-byte memset of its barrier counts)"}
    elif T <= FUSED_FFN_MAX_TOKENS:
        dom = {"kernel": "grouped_ffn_fused_kernel (gate/up + SwiGLU + down, one launch)",
               "bytes": alg["ffn_bytes"], "flops": alg["ffn_flops"],
               "rule": "touched experts x 6*d*f (gate, up and down weights, bf16)"}
    else:
        dom = {"kernel": ("grouped_gemm_pair_kernel (CTA pairs)" if T * k > 128 * E else "grouped_gemm_kernel<2>")
                         + " (gate/up + SwiGLU)",
               "bytes": alg["gu_bytes"], "flops": alg["gu_flops"],
               "rule": "touched experts x 4*d*f (gate and up weights, bf16)"}
    return {
        "ms_per_step": ms_per_step,
        "tokens_per_s": aggregate_tokens_per_s(T, steps, world, res["total_ms"]),
        "tflops": alg["F"] / t_step / 1e12, "hbm_gbs": alg["B"] / t_step / 1e9,
        "F_alg": alg["F"], "B_alg": alg["B"], "n_touched": alg["n_touched"],
        "max_rows_per_expert": int(res["counts"].max()),
        "roofline_frac": layer_roof_s / t_step,
        "binding_roof": "hbm" if alg["B"] / hbm / 1e9 >= alg["F"] / tc / 1e12 else "tensor",
        "tensor_frac_of_peak": alg["F"] / t_step / 1e12 / tc,
        "hbm_frac_of_peak": alg["B"] / t_step / 1e9 / hbm,
        "stage_ms": {kname: statistics.mean(v) for kname, v in res["stage_ms"].items()},
        "dominant_kernel": {
            "kernel": dom["kernel"], "ms_per_launch": gu_ms, "alg_bytes_per_launch": dom["bytes"],
            "alg_bytes_rule": dom["rule"],
            "achieved_gbs": dom["bytes"] / (gu_ms / 1e3) / 1e9,
            "achieved_tflops": dom["flops"] / (gu_ms / 1e3) / 1e12},
        "clocks": res["clocks"],
    }


EXTRA_WORKLOADS = ("decode", "skewed") + tuple(f"sweep_T{t}" for t in moe_inputs.SWEEP_T)
# workloads also timed with the experts in the MX serving format
MX_WORKLOADS = ("decode",) + tuple(f"sweep_T{t}" for t in moe_inputs.SWEEP_T)


def time_layer_mx(_lib, shape, inp, experts, steps: int, warmup: int, graph_on: bool, world: int, flush,
                  local: int):
    """Times moe_forward_mx steps (MXFP4 expert weights packed once, MXFP8
    activations) like time_layer, without per-stage times."""
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    ws = torch.empty(_lib.raw.moe_forward_mx_workspace_size(T, d, E, k, f), dtype=torch.uint8, device=inp.x.device)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=inp.x.device)
    stream = torch.cuda.current_stream()

    def step():
        _lib.moe_forward_mx(inp.x, inp.W_router, inp.bias, experts, k, out=out, workspace=ws)

    idx, _ = _lib.moe_route(inp.x, inp.W_router, inp.bias, k)
    offs, _, _, _ = _lib.moe_permute(None, idx, E, with_rows=False)
    counts = np.diff(offs.cpu().numpy())
    for _ in range(warmup):
        flush(1)
        step()
    graph = None
    if graph_on:
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
            with torch.cuda.graph(graph, stream=side):
                step()
        stream.wait_stream(side)
        for _ in range(warmup):
            flush(1)
            graph.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for s_, (a, b) in enumerate(evs):
        flush(s_)
        a.record(stream)
        if graph is not None:
            graph.replay()
        else:
            step()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
    assert _lib.get_device_error() == 0, "device error during MX timing"
    del graph
    return total_ms, counts, clk


def time_latent(_lib, li, steps: int, warmup: int, graph_on: bool, world: int, flush, local: int):
    """Times moe_latent_forward steps like time_layer_mx (no per-stage times)."""
    k = li.shape.k
    args = (li.x, li.W_router, li.bias, li.W_dn, li.W_up, li.W_gate_up, li.W_down, li.gamma, li.Ws_gate_up,
            li.Ws_down, k)
    T, d, E, f = li.shape.T, li.shape.d, li.shape.E, li.shape.f
    S = li.Ws_down.shape[0] if li.Ws_down is not None else 0
    fs = li.Ws_down.shape[1] if li.Ws_down is not None else 0
    ws = torch.empty(_lib.raw.moe_latent_workspace_size(T, d, li.l, E, k, f, S, fs), dtype=torch.uint8,
                     device=li.x.device)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=li.x.device)
    stream = torch.cuda.current_stream()

    def step():
        _lib.moe_latent_forward(*args, out=out, workspace=ws)

    idx, _ = _lib.moe_route(li.x, li.W_router, li.bias, k)
    offs, _, _, _ = _lib.moe_permute(None, idx, E, with_rows=False)
    counts = np.diff(offs.cpu().numpy())
    for _ in range(warmup):
        flush(1)
        step()
    graph = None
    if graph_on:
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
            with torch.cuda.graph(graph, stream=side):
                step()
        stream.wait_stream(side)
        for _ in range(warmup):
            flush(1)
            graph.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for s_, (a, b) in enumerate(evs):
        flush(s_)
        a.record(stream)
        if graph is not None:
            graph.replay()
        else:
            step()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
    assert _lib.get_device_error() == 0, "device error during latent timing"
    del graph
    return total_ms, counts, clk, S, fs


def latent_summary(li, total_ms, counts, clk, S, fs, steps, world, peaks) -> dict:
    """Throughput and roofline of a Stable LatentMoE step. F_alg: router
    2 T d E, the two projections 2 * 2 T d l, routed experts 6 T k l f, shared
    experts 6 T S d fs. B_alg: W_router 4 d E, x in and out 4 T d, W_dn and W_up
    2 * 2 d l, the touched routed experts 6 l f each, the shared experts
    S * 6 d fs, gamma 4 l (+ 4 E with a bias)."""
    T, d, E, k, f = li.shape.T, li.shape.d, li.shape.E, li.shape.k, li.shape.f
    l = li.l
    n_touched = int((counts > 0).sum())
    F = 2.0 * T * d * E + 4.0 * T * d * l + 6.0 * T * k * l * f + 6.0 * T * S * d * fs
    B = (4.0 * d * E + 4.0 * T * d + 4.0 * d * l + n_touched * 6.0 * l * f + S * 6.0 * d * fs + 4.0 * l
         + (4.0 * E if li.bias is not None else 0.0))
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    ms = total_ms / steps
    t = ms / 1e3
    return {"T": T, "d": d, "l": l, "E": E, "k": k, "f": f, "S": S, "fs": fs, "steps": steps,
            "ms_per_step": ms, "tokens_per_s": aggregate_tokens_per_s(T, steps, world, total_ms),
            "F_alg": F, "B_alg": B, "n_touched": n_touched, "tflops": F / t / 1e12, "hbm_gbs": B / t / 1e9,
            "roofline_frac": max(F / (tc * 1e12), B / (hbm * 1e9)) / t,
            "binding_roof": "hbm" if B / hbm / 1e9 >= F / tc / 1e12 else "tensor",
            "glu": "SiTU-GLU beta1=4 beta2=25", "clocks": clk}


def mx_summary(shape, total_ms: float, counts, clk, steps: int, world: int, peaks: dict) -> dict:
    """Throughput and roofline of an MX step: expert weights at 4.25 bits
    (E2M1 codes plus one E8M0 scale per 32), the rest as in the bf16 layer."""
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    n_touched = int((counts > 0).sum())
    F = 2.0 * T * d * E + 6.0 * T * k * d * f
    B = 4.0 * d * E + 4.0 * T * d + n_touched * 3.0 * d * f * (0.5 + 1.0 / 32) + (4.0 * E if shape.bias else 0.0)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    ms = total_ms / steps
    t = ms / 1e3
    return {"ms_per_step": ms, "tokens_per_s": aggregate_tokens_per_s(T, steps, world, total_ms),
            "F_alg": F, "B_alg": B, "n_touched": n_touched, "hbm_gbs": B / t / 1e9,
            "roofline_frac": max(F / (tc * 1e12), B / (hbm * 1e9)) / t,
            "binding_roof": "hbm" if B / hbm / 1e9 >= F / tc / 1e12 else "tensor",
            "bytes_rule": "expert weights at 4.25 bits (E2M1 + E8M0 per 32); router fp32; x, out bf16",
            "clocks": clk}


def run_ours(args):
    from sparse_mixture_experts_route_b200 import _lib
    world, rank, local = dist_setup()
    shape = moe_inputs.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    flush = L2Flush(dev)

    log(f"[rank {rank}] generating {shape.name} on {dev}")
    inp = moe_inputs.make_inputs(shape, seed=0, device=dev)
    if rank != 0:  # each replica routes its own tokens
        inp.x = moe_inputs.make_x(shape, seed=replica_x_seed(rank), device=dev)
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    if args.mx:
        # the MX serving format alone, on this workload (for profiling runs)
        experts = _lib.moe_mx_pack_experts(inp.W_gate_up, inp.W_down)
        tm, cnt, clk = time_layer_mx(_lib, shape, inp, experts, args.steps, args.warmup, args.graph == "on", world,
                                     flush, local)
        if rank != 0:
            return None
        summ = mx_summary(shape, tm, cnt, clk, args.steps, world, peaks)
        return {"metric": METRIC + "_mx", "value": summ["tokens_per_s"], "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "dtype": "e4m3 x e2m1",
                "data": "synthetic", "config": {**shape.as_dict(), "experts": "MXFP4, activations MXFP8"}, **summ}
    res = time_layer(_lib, shape, inp, args.steps, args.warmup, args.graph == "on", world, flush, local,
                     count_launches=True)
    out = res["out"]
    stream = torch.cuda.current_stream()

    # end to end through the host-buffer call: every step copies x in from
    # pinned host memory, runs the pass and copies the result back, all inside
    # moe_forward_host. Steps alternate between two streams (two workspaces,
    # two output buffers), so one step's copies overlap the other's kernels,
    # as a serving loop would run it; the timed region spans from before the
    # first step's input copy to after the last step's output copy. Every
    # step streams its experts' weights (far more than L2), so no flush.
    x_host = inp.x.cpu().pin_memory()
    hws = _lib.moe_forward_host_workspace_size(T, d, E, k, f)
    e2e_streams = [stream, torch.cuda.Stream()]
    e2e_ws = [torch.empty(hws, dtype=torch.uint8, device="cuda") for _ in e2e_streams]
    e2e_out = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in e2e_streams]

    def e2e_steps(n):
        for s in range(n):
            j = s % 2
            _lib.moe_forward_host(x_host, inp.W_router, inp.bias, inp.W_gate_up, inp.W_down, k,
                                  out_host=e2e_out[j], workspace=e2e_ws[j], stream=e2e_streams[j])

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_streams[1].wait_event(e0)
    e2e_steps(args.steps)
    stream.wait_stream(e2e_streams[1])
    e1.record(stream)
    e1.synchronize()
    e2e_ms = [e0.elapsed_time(e1)]
    barrier(world)
    assert torch.equal(e2e_out[(args.steps - 1) % 2], out.cpu()), "host-buffer call disagrees with moe_forward"
    e2e_total = max_over_ranks(sum(e2e_ms), world)

    cpu_line = None
    if rank == 0 and not args.no_cpu_baseline:
        log("[rank 0] timing the CPU oracle on a bounded sample")
        cpu_line = cpu_baseline(inp, shape, budget_s=args.cpu_budget)
    head = layer_summary(shape, res, args.steps, world, peaks)
    launches, impl_bytes = res["launches"], res["alg"]["gu_impl_bytes"]
    del inp, res, e2e_ws, e2e_out, x_host
    torch.cuda.empty_cache()

    # the other workloads, one after another (every rank runs the same list,
    # so the timing barriers line up); skewed and the sweep share one set of
    # expert weights (same shapes and seeds), generated once
    extra = {}
    mx_packed = {}
    if not args.no_workloads:
        shared = None
        for name in EXTRA_WORKLOADS:
            ws_shape = moe_inputs.WORKLOADS[name]
            log(f"[rank {rank}] {name}")
            if shared is not None and shared.W_gate_up.shape == (ws_shape.E, ws_shape.d, 2 * ws_shape.f):
                x = moe_inputs.make_x(ws_shape, seed=replica_x_seed(rank), device=dev)
                bias = moe_inputs.zipf_bias(ws_shape.E).to(dev) if ws_shape.bias == "zipf" else None
                winp = type(shared)(ws_shape, x, shared.W_router, bias, shared.W_gate_up, shared.W_down)
            else:
                shared = None
                torch.cuda.empty_cache()
                winp = moe_inputs.make_inputs(ws_shape, seed=0, device=dev)
                if rank != 0:
                    winp.x = moe_inputs.make_x(ws_shape, seed=replica_x_seed(rank), device=dev)
                shared = winp
            steps = args.workload_steps
            r = time_layer(_lib, ws_shape, winp, steps, args.warmup, args.graph == "on", world, flush, local)
            extra[name] = {**{kk: v for kk, v in ws_shape.as_dict().items() if kk != "workload"},
                           "steps": steps, **layer_summary(ws_shape, r, steps, world, peaks)}
            del r
            if name in MX_WORKLOADS and not args.no_mx:
                if mx_packed.get("src") is not shared.W_gate_up:
                    mx_packed["experts"] = _lib.moe_mx_pack_experts(winp.W_gate_up, winp.W_down)
                    mx_packed["src"] = shared.W_gate_up
                tm, cnt, clk = time_layer_mx(_lib, ws_shape, winp, mx_packed["experts"], steps, args.warmup,
                                             args.graph == "on", world, flush, local)
                extra[name + "_mx"] = {**{kk: v for kk, v in ws_shape.as_dict().items() if kk != "workload"},
                                       "steps": steps, "experts": "MXFP4 (E2M1, E8M0 per 32), activations MXFP8",
                                       **mx_summary(ws_shape, tm, cnt, clk, steps, world, peaks)}
            del winp
        del shared
        mx_packed.clear()
        torch.cuda.empty_cache()
        if not args.no_latent:
            log(f"[rank {rank}] latent_prefill")
            lat = moe_inputs.LATENT
            li = moe_inputs.make_latent_inputs(lat["shape"], lat["l"], lat["S"], lat["fs"], seed=0, device=dev)
            if rank != 0:
                li.x = moe_inputs.make_x(lat["shape"], seed=replica_x_seed(rank), device=dev)
            tm, cnt, clk, S, fs = time_latent(_lib, li, args.workload_steps, args.warmup, args.graph == "on", world,
                                              flush, local)
            extra["latent_prefill"] = latent_summary(li, tm, cnt, clk, S, fs, args.workload_steps, world, peaks)
            del li
            torch.cuda.empty_cache()

    if rank != 0:
        return None
    n = world
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    dom = head["dominant_kernel"]
    line = {
        "metric": METRIC, "value": head["tokens_per_s"], "unit": UNIT, "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**shape.as_dict(), "seed": 0, "parallelism": f"replicas{n}",
                   "launch": "cuda_graph_replay" if args.graph == "on" else "eager",
                   "l2": "flushed between steps (2x L2 write, then 2x L2 read, outside the step events)",
                   "weights_gb": round(E * 6.0 * d * f / 1e9, 3)},
        "roofline": {"bound": "hbm", "kernel": dom["kernel"],
                     "achieved": dom["achieved_gbs"], "peak": hbm, "unit": "GB/s", "frac": dom["achieved_gbs"] / hbm,
                     "traffic": profiled_traffic(shape.name), "peak_source": f"{peak_src} hbm_gbs (burst copy)",
                     "alg_bytes_per_launch": dom["alg_bytes_per_launch"], "alg_bytes_rule": dom["alg_bytes_rule"],
                     "impl_bytes_per_launch": impl_bytes,
                     "ms_per_launch": dom["ms_per_launch"]},
        "layer": {kk: v for kk, v in head.items() if kk not in ("ms_per_step", "tokens_per_s", "clocks",
                                                                 "dominant_kernel")},
        "e2e": {"value": aggregate_tokens_per_s(T, args.steps, n, e2e_total), "unit": UNIT,
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2,
                "call": "moe_forward_host, steps alternating over 2 streams"},
        "gpu_launches": launches * args.steps,
        "clocks": head["clocks"],
    }
    if extra:
        line["workloads"] = extra
    if cpu_line is not None:
        line["cpu_baseline"] = cpu_line
    return line


def run_reference(args):
    """The oracle on the host cores, each step one oracle pass over a bounded,
    seeded sample of the workload's tokens (sized so the whole run takes about
    two and a half minutes)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    shape = moe_inputs.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = moe_inputs.make_inputs(shape, seed=0, device=dev)
    threads = oracle.num_threads()
    budget = max(1.0, min(args.cpu_budget, 150.0 / max(1, args.steps + args.warmup)))
    n = calibrate_tokens(inp, shape, budget, threads)
    for w_ in range(args.warmup):
        oracle_pass(inp, shape, sample_tokens(shape.T, n, 500 + w_), threads)
    secs, ffn = [], []
    for s in range(args.steps):
        t, rows, fl, fs = oracle_pass(inp, shape, sample_tokens(shape.T, n, 1 + s), threads)
        secs.append(t)
        ffn.append((fl, fs))
    ms_per_step = 1e3 * statistics.mean(secs)
    value = n * args.steps / sum(secs)
    cb = {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
          "sample": f"each step: one oracle pass (router, top-k, {n * shape.k} expert rows, combine) over {n} "
                    f"seeded tokens of {shape.name} (weights fetched to host untimed)",
          "tokens": n, "cpu_model": cpu_model(),
          "fp64_gflops": sum(a for a, _ in ffn) / max(sum(b for _, b in ffn), 1e-9) / 1e9}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**shape.as_dict(), "seed": 0, "parallelism": "host cores", "tokens_per_step": n},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_mx_quant(args):
    """Throughput of the MX quantisers (the MXFP8 activation and MXFP4 weight
    formats) on one GPU: the prefill activations widened to 16384 rows
    [16384, 7168] and 32 experts' W_gate_up [32, 7168, 4096]. Inputs are larger
    than L2, so no flush is needed; each launch is timed between CUDA events on
    its stream after W warm-up launches, and the mean over K is reported.
    Algorithmic bytes per element: 2 read + 1 code + 1/32 scale."""
    from sparse_mixture_experts_route_b200 import _lib
    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    x = torch.randn(16384, 7168, generator=g, device=dev).to(torch.bfloat16)
    w = torch.empty(32, 7168, 4096, dtype=torch.bfloat16, device=dev)
    for e in range(32):
        w[e].copy_(torch.randn(7168, 4096, generator=g, device=dev) / 84.66)
    cases = {
        "mxfp8_activations_16384x7168": (lambda c, s_: _lib.moe_mxfp8_quantize(x, codes=c, scales=s_),
                                        x.numel(), (16384, 7168), (16384, 7168 // 32)),
        "mxfp4_weights_32x7168x4096": (lambda c, s_: _lib.moe_mxfp4_quantize(w, codes=c, scales=s_),
                                      w.numel(), (32, 7168, 4096), (32, 7168 // 32, 4096)),
    }
    sampler = ClockSampler(0)
    out = {}
    sampler.start()
    for name, (fn, n_el, cshape, sshape) in cases.items():
        codes = torch.empty(cshape, dtype=torch.uint8, device=dev)
        scales = torch.empty(sshape, dtype=torch.uint8, device=dev)
        for _ in range(args.warmup):
            fn(codes, scales)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a, b in evs:
            a.record(stream)
            fn(codes, scales)
            b.record(stream)
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        gbs = n_el * (2 + 1 + 1 / 32) / (ms * 1e-3) / 1e9
        out[name] = {"ms_per_launch": ms, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]}
    clocks = sampler.stop()
    assert _lib.get_device_error() == 0
    return {"metric": "mx_quantize_bytes_per_s", "unit": "GB/s", "higher_is_better": True,
            "value": min(v["GB/s"] for v in out.values()), "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "dtype": "bf16->e4m3/e2m1", "data": "synthetic",
            "kernels": out, "peak": {"hbm_gbs": peaks["hbm_gbs"], "kind": peak_kind},
            "config": {"workload": "mx_quantize", "l2": "inputs larger than L2"}, "clocks": clocks}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=sorted(moe_inputs.WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only --workload (skip the decode, skewed and sweep entries of the line)")
    ap.add_argument("--no-mx", action="store_true", help="skip the MX-format entries of the workloads")
    ap.add_argument("--mx", action="store_true", help="time only moe_forward_mx on --workload (profiling runs)")
    ap.add_argument("--no-latent", action="store_true", help="skip the Stable LatentMoE entry of the workloads")
    ap.add_argument("--workload-steps", type=int, default=10,
                    help="timed steps of each of the other workloads")
    ap.add_argument("--graph", default="on", choices=["on", "off"],
                    help="time replays of one step captured as a CUDA graph (on) or eager calls (off)")
    ap.add_argument("--mx-quant", action="store_true",
                    help="time the MXFP8/MXFP4 quantisers instead of the layer (one GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.mx_quant:
        print(json.dumps(run_mx_quant(args)), flush=True)
        return
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and args.impl == "ours":
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
