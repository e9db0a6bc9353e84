"""CPU oracle for the sparse Mixture-of-Experts layer forward pass.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by ``bench.py``'s CPU-baseline leg. The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``moe_oracle.cpp`` (plain C++, fp64 except for the fp32
router whose summation order is stated there, and the Quantile Balancing
histogram's fp32-decision variant, pinned against its fp64 definition). This
module only builds that file and marshals numpy / torch CPU arrays into it.

Every function cites its passage in ``moe_oracle.cpp``. The oracle functions
here are pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_pins.py``
(brute-force sorts, closed forms, invariants, and library routines), with one
exception: SiTU-GLU's own formula (``glu_ffn`` / ``latent_forward`` with
``ACT_SITU``) is parity unpinned, because the page lost it; what is pinned
there is its stated bound, its SwiGLU limit for large caps, and the latent
layer's reductions to the pinned plain layer.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

CXXFLAGS = ["-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-mfma",
            "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.cpp`` into ``libmoe_oracle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["g++", *CXXFLAGS, _SRC, "-o", tmp], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int64
            lib.oracle_router_logits.argtypes = [P, P, P, I, I, I, P]
            lib.oracle_topk.argtypes = [P, I, I, I, P, P, P]
            lib.oracle_permute.argtypes = [P, I, I, I, P, P, P, P]
            lib.oracle_expert_ffn.argtypes = [P, I, P, P, I, I, P, P]
            lib.oracle_combine.argtypes = [P, P, P, I, I, I, P]
            lib.oracle_forward_tokens.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, P, P]
            lib.oracle_mxfp4_quantize.argtypes = [P, I, I, P, P]
            lib.oracle_mxfp4_dequantize.argtypes = [P, P, I, I, P]
            lib.oracle_mxfp8_quantize.argtypes = [P, I, I, P, P]
            lib.oracle_mxfp8_dequantize.argtypes = [P, P, I, I, P]
            lib.oracle_expert_ffn_mx.argtypes = [P, I, P, P, I, I, P, P]
            lib.oracle_qb_cutoffs.argtypes = [P, P, I, I, I, P]
            lib.oracle_qb_update.argtypes = [P, P, I, I, I, P]
            lib.oracle_qb_histogram.argtypes = [P, P, I, I, ctypes.c_double, ctypes.c_double, I, P]
            lib.oracle_qb_bias_from_histogram.argtypes = [P, I, I, ctypes.c_double, ctypes.c_double, I, I, P]
            lib.oracle_qb_histogram_f32.argtypes = [P, P, I, I, I, ctypes.c_float, ctypes.c_float, I, P, P]
            lib.oracle_qb_quantile_bins.argtypes = [P, I, I, I, I, P]
            D = ctypes.c_double
            lib.oracle_glu_ffn.argtypes = [P, I, P, P, I, I, I, ctypes.c_int, D, D, P, P]
            lib.oracle_rmsnorm.argtypes = [P, I, I, P, D, P]
            lib.oracle_latent_forward.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                                  ctypes.c_int, D, D, D, P, P]
            for fn in ("oracle_router_logits", "oracle_topk", "oracle_permute", "oracle_expert_ffn",
                       "oracle_combine", "oracle_forward_tokens", "oracle_num_threads", "oracle_version",
                       "oracle_mxfp4_quantize", "oracle_mxfp4_dequantize", "oracle_mxfp8_quantize",
                       "oracle_mxfp8_dequantize", "oracle_expert_ffn_mx", "oracle_qb_cutoffs", "oracle_qb_update",
                       "oracle_qb_histogram", "oracle_qb_bias_from_histogram", "oracle_qb_histogram_f32",
                       "oracle_qb_quantile_bins", "oracle_glu_ffn", "oracle_rmsnorm", "oracle_latent_forward"):
                getattr(lib, fn).restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ---------------------------------------------------------------- marshalling

def _bf16_bits(a) -> np.ndarray:
    """A bf16 torch tensor (CPU) or a uint16 numpy array -> contiguous uint16 bits."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16, a.dtype
            return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(a)
    assert a.dtype == np.uint16, a.dtype
    return np.ascontiguousarray(a)


def _bits_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16) -> fp64 values, exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f32(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return np.ascontiguousarray(a.detach().cpu().to(torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _check(st: int, what: str):
    if st == 1:
        raise ValueError(f"{what}: bad argument")
    if st == 2:
        raise FloatingPointError(f"{what}: non-finite input (outside the oracle's contract)")
    if st != 0:
        raise RuntimeError(f"{what}: status {st}")


# ------------------------------------------------------------------ the steps

def router_logits(x, W_router, bias=None) -> np.ndarray:
    """Step 1 of moe_oracle.cpp: fp32 logits [T, E] in the stated chunked order."""
    xb = _bf16_bits(x)
    Wr = _f32(W_router)
    T, d = xb.shape
    d2, E = Wr.shape
    assert d == d2
    b = _f32(bias) if bias is not None else None
    out = np.empty((T, E), dtype=np.float32)
    _check(_load().oracle_router_logits(_ptr(xb), _ptr(Wr), _ptr(b), T, d, E, _ptr(out)), "router_logits")
    return out


def topk(logits: np.ndarray, k: int, want_probs: bool = False):
    """Steps 2-3: (idx [T,k] int32, w [T,k] fp64[, probs [T,E] fp64])."""
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    probs = np.empty((T, E), dtype=np.float64) if want_probs else None
    _check(_load().oracle_topk(_ptr(lg), T, E, k, _ptr(idx), _ptr(w), _ptr(probs)), "topk")
    return (idx, w, probs) if want_probs else (idx, w)


def permute(idx: np.ndarray, E: int):
    """Step 4: (counts [E], offsets [E+1], perm_token [T*k], inv_perm [T,k]) int32."""
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = ix.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm_token = np.empty(T * k, dtype=np.int32)
    inv_perm = np.empty((T, k), dtype=np.int32)
    _check(_load().oracle_permute(_ptr(ix), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm_token),
                                  _ptr(inv_perm)), "permute")
    return counts, offsets, perm_token, inv_perm


def expert_ffn(x_rows, W_gate_up_e, W_down_e, want_h: bool = False):
    """Step 5 for one expert: y [n, d] fp64 (and h [n, f] fp64)."""
    xr = _bf16_bits(x_rows)
    Wg = _bf16_bits(W_gate_up_e)
    Wd = _bf16_bits(W_down_e)
    n, d = xr.shape
    d2, f2 = Wg.shape
    f, d3 = Wd.shape
    assert d == d2 == d3 and f2 == 2 * f
    y = np.empty((n, d), dtype=np.float64)
    h = np.empty((n, f), dtype=np.float64) if want_h else None
    _check(_load().oracle_expert_ffn(_ptr(xr), n, _ptr(Wg), _ptr(Wd), d, f, _ptr(y), _ptr(h)), "expert_ffn")
    return (y, h) if want_h else y


def combine(y_rows: np.ndarray, inv_perm: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Step 6: out [T, d] fp64."""
    y = np.ascontiguousarray(y_rows, dtype=np.float64)
    ip = np.ascontiguousarray(inv_perm, dtype=np.int32)
    ww = np.ascontiguousarray(w, dtype=np.float64)
    T, k = ip.shape
    d = y.shape[1]
    out = np.empty((T, d), dtype=np.float64)
    _check(_load().oracle_combine(_ptr(y), _ptr(ip), _ptr(ww), T, d, k, _ptr(out)), "combine")
    return out


def forward(x, W_router, bias, W_gate_up, W_down, k: int, tokens=None):
    """The whole layer (steps 1-6) for all tokens or the listed ones.

    Returns (out [n, d] fp64, idx [n, k] int32, w [n, k] fp64).
    """
    xb = _bf16_bits(x)
    Wr = _f32(W_router)
    b = _f32(bias) if bias is not None else None
    Wg = _bf16_bits(W_gate_up)
    Wd = _bf16_bits(W_down)
    T, d = xb.shape
    E = Wr.shape[1]
    f = Wd.shape[1]
    assert Wg.shape == (E, d, 2 * f) and Wd.shape == (E, f, d)
    tok = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
    n = T if tok is None else tok.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    idx = np.empty((n, k), dtype=np.int32)
    w = np.empty((n, k), dtype=np.float64)
    _check(_load().oracle_forward_tokens(_ptr(xb), _ptr(Wr), _ptr(b), _ptr(Wg), _ptr(Wd), T, d, E, k, f,
                                         _ptr(tok), n, _ptr(out), _ptr(idx), _ptr(w)), "forward")
    return out, idx, w


# ---------------------------------------------------------------- MXFP4 weights

def mxfp4_quantize(w):
    """MXFP4 of a weight matrix w [K, N] (bf16 tensor or uint16 bits, N
    contiguous, K % 32 == 0) with blocks of 32 along K (the reduction axis).
    Returns (codes uint8 [K, N]: one E2M1 code per byte, sign in bit 3;
    scales uint8 [K // 32, N]: E8M0 exponent codes, 2^(code - 127)).
    Definition and readings: ``oracle_mxfp4_quantize`` in moe_oracle.cpp."""
    wb = _bf16_bits(w)
    assert wb.ndim == 2, wb.shape
    K, N = wb.shape
    codes = np.empty((K, N), dtype=np.uint8)
    scales = np.empty((K // 32, N), dtype=np.uint8)
    st = _load().oracle_mxfp4_quantize(wb.ctypes.data, K, N, codes.ctypes.data, scales.ctypes.data)
    if st:
        raise ValueError(f"oracle_mxfp4_quantize: status {st}")
    return codes, scales


def mxfp4_dequantize(codes, scales) -> np.ndarray:
    """The MXFP4 values as bf16 bits (uint16 [K, N]; every value is exact in
    bf16): code c, scale code q -> (-1)^(c >> 3) * |E2M1(c & 7)| * 2^(q - 127)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    K, N = codes.shape
    assert scales.shape == (K // 32, N), (scales.shape, codes.shape)
    out = np.empty((K, N), dtype=np.uint16)
    st = _load().oracle_mxfp4_dequantize(codes.ctypes.data, scales.ctypes.data, K, N, out.ctypes.data)
    if st:
        raise ValueError(f"oracle_mxfp4_dequantize: status {st}")
    return out


def mxfp8_quantize(v):
    """MXFP8 (E4M3 elements, E8M0 scales) of v [rows, cols] (anything numpy
    converts to fp64, cols % 32 == 0) with blocks of 32 along each row.
    Returns (codes uint8 [rows, cols], scales uint8 [rows, cols // 32]).
    Definition and readings: ``oracle_mxfp8_quantize`` in moe_oracle.cpp."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    assert v.ndim == 2, v.shape
    R, C = v.shape
    codes = np.empty((R, C), dtype=np.uint8)
    scales = np.empty((R, C // 32), dtype=np.uint8)
    st = _load().oracle_mxfp8_quantize(v.ctypes.data, R, C, codes.ctypes.data, scales.ctypes.data)
    if st:
        raise ValueError(f"oracle_mxfp8_quantize: status {st}")
    return codes, scales


def mxfp8_dequantize(codes, scales) -> np.ndarray:
    """The MXFP8 values in fp64 [rows, cols]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, C = codes.shape
    assert scales.shape == (R, C // 32), (scales.shape, codes.shape)
    out = np.empty((R, C), dtype=np.float64)
    st = _load().oracle_mxfp8_dequantize(codes.ctypes.data, scales.ctypes.data, R, C, out.ctypes.data)
    if st:
        raise ValueError(f"oracle_mxfp8_dequantize: status {st}")
    return out


def expert_ffn_mx(x_rows, gu_codes, gu_scales, dn_codes, dn_scales, want_h: bool = False):
    """One expert's SwiGLU feed-forward in the MX serving format: the rows of x
    (bf16 [n, d]) take an MXFP8 round trip along d, the weights are the MXFP4
    codes/scales of W_gate_up [d, 2f] and W_down [f, d], h takes an MXFP8 round
    trip along f. Returns y [n, d] fp64 (and h' [n, f] with want_h)."""
    xb = _bf16_bits(x_rows)
    n, d = xb.shape
    x64 = np.ascontiguousarray(_bits_f64(xb))
    xq = mxfp8_dequantize(*mxfp8_quantize(x64)) if n > 0 else x64
    wgu = mxfp4_dequantize(gu_codes, gu_scales)
    wd = mxfp4_dequantize(dn_codes, dn_scales)
    assert wgu.shape[0] == d and wd.shape[1] == d, (wgu.shape, wd.shape)
    f = wd.shape[0]
    y = np.zeros((n, d), dtype=np.float64)
    h = np.zeros((n, f), dtype=np.float64)
    st = _load().oracle_expert_ffn_mx(xq.ctypes.data if n else None, n, wgu.ctypes.data, wd.ctypes.data, d, f,
                                      y.ctypes.data, h.ctypes.data)
    if st:
        raise ValueError(f"oracle_expert_ffn_mx: status {st}")
    return (y, h) if want_h else y


# ------------------------------------------------------ Quantile Balancing

def _f64c(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def qb_cutoffs(scores, k: int, bias=None) -> np.ndarray:
    """alpha [m]: each token's (k+1)-th largest biased score s + b (the cutoff
    of top-(k+1) routing). Definition and readings: oracle_qb_cutoffs in
    moe_oracle.cpp."""
    s = _f64c(scores)
    m, n = s.shape
    b = _f64c(bias) if bias is not None else None
    alpha = np.empty(m, dtype=np.float64)
    _check(_load().oracle_qb_cutoffs(s.ctypes.data, b.ctypes.data if b is not None else None, m, n, k,
                                     alpha.ctypes.data), "oracle_qb_cutoffs")
    return alpha


def qb_update(scores, k: int, bias=None) -> np.ndarray:
    """One Quantile Balancing step with exact quantiles: the new biases [n]."""
    s = _f64c(scores)
    m, n = s.shape
    b = _f64c(bias) if bias is not None else None
    out = np.empty(n, dtype=np.float64)
    _check(_load().oracle_qb_update(s.ctypes.data, b.ctypes.data if b is not None else None, m, n, k,
                                    out.ctypes.data), "oracle_qb_update")
    return out


def qb_histogram(scores, alpha, lo: float, hi: float, bins: int, H=None) -> np.ndarray:
    """Per-expert margin counts H [n, bins] int64 (added into H if given)."""
    s = _f64c(scores)
    m, n = s.shape
    a = _f64c(alpha)
    if H is None:
        H = np.zeros((n, bins), dtype=np.int64)
    assert H.dtype == np.int64 and H.shape == (n, bins) and H.flags.c_contiguous
    _check(_load().oracle_qb_histogram(s.ctypes.data, a.ctypes.data, m, n, float(lo), float(hi), bins,
                                       H.ctypes.data), "oracle_qb_histogram")
    return H


def qb_bias_from_histogram(H, lo: float, hi: float, m_total: int, k: int) -> np.ndarray:
    """The new biases [n] from (all-reduced) margin histograms."""
    H = np.ascontiguousarray(H, dtype=np.int64)
    n, bins = H.shape
    out = np.empty(n, dtype=np.float64)
    _check(_load().oracle_qb_bias_from_histogram(H.ctypes.data, n, bins, float(lo), float(hi), m_total, k,
                                                 out.ctypes.data), "oracle_qb_bias_from_histogram")
    return out


def qb_histogram_f32(scores, k: int, lo: float, hi: float, bins: int, bias=None, H=None):
    """The margin histogram with every decision in fp32 (scores and bias taken
    as fp32). Returns (alpha [m] fp32, H [n, bins] int64). Definition:
    oracle_qb_histogram_f32 in moe_oracle.cpp."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    m, n = s.shape
    b = np.ascontiguousarray(np.asarray(bias, dtype=np.float32)) if bias is not None else None
    if H is None:
        H = np.zeros((n, bins), dtype=np.int64)
    assert H.dtype == np.int64 and H.shape == (n, bins) and H.flags.c_contiguous
    alpha = np.empty(m, dtype=np.float32)
    _check(_load().oracle_qb_histogram_f32(s.ctypes.data, b.ctypes.data if b is not None else None, m, n, k,
                                           float(lo), float(hi), bins, alpha.ctypes.data, H.ctypes.data),
           "oracle_qb_histogram_f32")
    return alpha, H


def qb_quantile_bins(H, m_total: int, k: int) -> np.ndarray:
    """Per expert, the bin holding the ceil(m_total k / n)-th largest margin."""
    H = np.ascontiguousarray(H, dtype=np.int64)
    n, bins = H.shape
    out = np.empty(n, dtype=np.int64)
    _check(_load().oracle_qb_quantile_bins(H.ctypes.data, n, bins, m_total, k, out.ctypes.data),
           "oracle_qb_quantile_bins")
    return out


# ------------------------------------------------------ Stable LatentMoE

#: SiTU-GLU soft caps stated on the page (its bound is beta1 * beta2 = 100).
SITU_BETA1 = 4.0
SITU_BETA2 = 25.0
ACT_SWIGLU, ACT_SITU = 0, 1


def glu_ffn(x_rows, W_gu, W_d, act: int = ACT_SITU, beta1: float = SITU_BETA1, beta2: float = SITU_BETA2,
            want_h: bool = False):
    """One GLU feed-forward in fp64: x_rows [n, K] (anything numpy widens to
    fp64, or a bf16 tensor), W_gu [K, 2F] and W_d [F, N] bf16. act
    ACT_SWIGLU or ACT_SITU (SiTU-GLU with the given caps). Returns y [n, N]
    (and h [n, F] with want_h). Definition and readings: oracle_glu_ffn and the
    Stable LatentMoE notes in moe_oracle.cpp."""
    try:
        import torch
        if isinstance(x_rows, torch.Tensor) and x_rows.dtype == torch.bfloat16:
            x_rows = _bits_f64(_bf16_bits(x_rows))
    except ImportError:  # pragma: no cover
        pass
    x = _f64c(x_rows)
    n, K = x.shape
    wg = _bf16_bits(W_gu)
    wd = _bf16_bits(W_d)
    assert wg.shape[0] == K and wg.shape[1] % 2 == 0, (wg.shape, K)
    F = wg.shape[1] // 2
    N = wd.shape[1]
    assert wd.shape[0] == F, (wd.shape, F)
    y = np.zeros((n, N), dtype=np.float64)
    h = np.zeros((n, F), dtype=np.float64)
    _check(_load().oracle_glu_ffn(x.ctypes.data if n else None, n, wg.ctypes.data, wd.ctypes.data, K, F, N, act,
                                  float(beta1), float(beta2), y.ctypes.data, h.ctypes.data), "oracle_glu_ffn")
    return (y, h) if want_h else y


def rmsnorm(u, gamma=None, eps: float = 1e-6) -> np.ndarray:
    """gamma * u / sqrt(mean(u^2) + eps) per row, fp64 [n, l]."""
    u = _f64c(u)
    n, l = u.shape
    g = _f32(gamma) if gamma is not None else None
    out = np.empty_like(u)
    _check(_load().oracle_rmsnorm(u.ctypes.data if n else None, n, l, _ptr(g), float(eps), out.ctypes.data),
           "oracle_rmsnorm")
    return out


def latent_forward(x, W_router, bias, W_dn, W_up, W_gate_up, W_down, gamma, Ws_gate_up, Ws_down, k: int,
                   act: int = ACT_SITU, beta1: float = SITU_BETA1, beta2: float = SITU_BETA2, eps: float = 1e-6,
                   want_u: bool = False):
    """The Stable LatentMoE layer in fp64: out [T, d] (and the routed sum u
    [T, l] before the RMSNorm with want_u). x [T, d] bf16; W_router [d, E] fp32;
    bias [E] or None; W_dn [d, l], W_up [l, d]; routed W_gate_up [E, l, 2f],
    W_down [E, f, l]; gamma [l] or None; shared Ws_gate_up [S, d, 2fs],
    Ws_down [S, fs, d] (S may be 0, then both None). Definition and readings:
    oracle_latent_forward in moe_oracle.cpp."""
    xb = _bf16_bits(x)
    T, d = xb.shape
    Wr = _f32(W_router)
    E = Wr.shape[1]
    b = _f32(bias) if bias is not None else None
    wdn = _bf16_bits(W_dn)
    l = wdn.shape[1]
    wup = _bf16_bits(W_up)
    wgu = _bf16_bits(W_gate_up)
    wd = _bf16_bits(W_down)
    f = wd.shape[1]
    assert wgu.shape == (E, l, 2 * f) and wd.shape == (E, f, l) and wup.shape == (l, d), (wgu.shape, wd.shape)
    g = _f32(gamma) if gamma is not None else None
    if Ws_gate_up is not None:
        wsg = _bf16_bits(Ws_gate_up)
        wsd = _bf16_bits(Ws_down)
        S, fs = wsd.shape[0], wsd.shape[1]
    else:
        wsg = wsd = None
        S, fs = 0, 0
    out = np.zeros((T, d), dtype=np.float64)
    u = np.zeros((T, l), dtype=np.float64)
    _check(_load().oracle_latent_forward(xb.ctypes.data, Wr.ctypes.data, _ptr(b), wdn.ctypes.data, wup.ctypes.data,
                                         wgu.ctypes.data, wd.ctypes.data, _ptr(g), _ptr(wsg), _ptr(wsd), T, d, l, E,
                                         k, f, S, fs, act, float(beta1), float(beta2), float(eps), out.ctypes.data,
                                         u.ctypes.data), "oracle_latent_forward")
    return (out, u) if want_u else out
