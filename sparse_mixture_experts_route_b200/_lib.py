"""ctypes binding of ``libmoe.so`` (the C ABI in include/moe.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their ``data_ptr()`` and torch's current CUDA stream are passed to
the C entry point of the same name, and a non-OK status raises ``MoEError``.
Every step of the layer runs in the library's kernels. Importing this module
loads the library and raises if it is missing: there is no fallback.
MOE_LIBRARY=checks in the environment loads the index-checking build
``libmoe_checks.so`` instead (same entry points, see build.py).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_VARIANT = os.environ.get("MOE_LIBRARY", "")
if _VARIANT not in ("", "checks"):
    raise ImportError(f"MOE_LIBRARY={_VARIANT!r}: expected 'checks' or unset")
LIB_PATH = os.path.join(_HERE, "libmoe_checks.so" if _VARIANT == "checks" else "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                      f"python -m sparse_mixture_experts_route_b200.build{' --checks' if _VARIANT else ''}")

_lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I = ctypes.c_int
Z = ctypes.c_size_t

EXPORTS = {
    "moe_status_string": ([I], ctypes.c_char_p),
    "moe_version": ([], I),
    "moe_route_workspace_size": ([I, I, I], Z),
    "moe_route": ([P, P, P, I, I, I, I, P, P, P, Z, P], I),
    "moe_permute_workspace_size": ([I, I, I], Z),
    "moe_permute": ([P, P, I, I, I, I, P, P, P, P, P, Z, P], I),
    "moe_expert_ffn_workspace_size": ([I, I], Z),
    "moe_expert_ffn": ([P, P, P, P, I, I, I, I, P, P, P, Z, P], I),
    "moe_unpermute": ([P, P, P, I, I, I, P, P], I),
    "moe_forward_workspace_size": ([I, I, I, I, I], Z),
    "moe_forward": ([P, P, P, P, P, I, I, I, I, I, P, P, Z, P], I),
    "moe_mxfp8_quantize": ([P, I, I, P, P, P], I),
    "moe_mxfp4_quantize": ([P, I, I, P, P, P], I),
    "moe_mx_expert_bytes": ([I, I, I, ctypes.POINTER(Z), ctypes.POINTER(Z), ctypes.POINTER(Z),
                             ctypes.POINTER(Z)], I),
    "moe_mx_pack_experts": ([P, P, I, I, I, P, P, P, P, P], I),
    "moe_forward_mx_workspace_size": ([I, I, I, I, I], Z),
    "moe_forward_mx": ([P, P, P, P, P, P, P, I, I, I, I, I, P, P, Z, P], I),
    "moe_router_logits": ([P, P, P, I, I, I, P, P], I),
    "moe_qb_histogram": ([P, P, I, I, I, ctypes.c_float, ctypes.c_float, I, P, P, P], I),
    "moe_qb_bias": ([P, I, I, ctypes.c_float, ctypes.c_float, ctypes.c_int64, I, P, P, P], I),
    "moe_gather_rows": ([P, ctypes.c_int64, P, ctypes.c_int64, I, P, P], I),
    "moe_latent_workspace_size": ([I, I, I, I, I, I, I, I], Z),
    "moe_latent_forward": ([P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, ctypes.c_float,
                            ctypes.c_float, ctypes.c_float, P, P, Z, P], I),
    "moe_get_device_error": ([ctypes.POINTER(ctypes.c_uint32), I], I),
    "moe_selftest_wait_timeout": ([I, P], I),
}
for _name, (_args, _res) in EXPORTS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
DEVERR_SELFTEST_TIMEOUT = 4
DEVERR_BAD_ROUTE = 5
DEVERR_WAIT_TIMEOUT_DEPENDENCY = 7
DEVERR_INDEX_CHECK = 8  # index-checking build only


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _lib.moe_status_string(status).decode()
        super().__init__(f"{where}: {name}")


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _workspace(nbytes: int, device, stream=None) -> torch.Tensor:
    """Scratch for one call, allocated on the stream the call runs on: torch's
    caching allocator hands a freed block only to later allocations on the same
    stream, which run after this call's work, so a workspace freed when the
    binding returns is never reused by work that overlaps the call. (Blocks
    are 512-byte aligned.)"""
    if stream is None:
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    with torch.cuda.stream(stream):
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def version() -> int:
    return int(_lib.moe_version())


def route_workspace_size(T: int, d: int, E: int) -> int:
    return int(_lib.moe_route_workspace_size(T, d, E))


def permute_workspace_size(T: int, E: int, k: int) -> int:
    return int(_lib.moe_permute_workspace_size(T, E, k))


def expert_ffn_workspace_size(Tk: int, E: int) -> int:
    return int(_lib.moe_expert_ffn_workspace_size(Tk, E))


def moe_forward_workspace_size(T: int, d: int, E: int, k: int, f: int) -> int:
    return int(_lib.moe_forward_workspace_size(T, d, E, k, f))


def moe_route(x, W_router, router_bias, k: int, workspace=None, stream=None):
    """Steps 1-3. Returns (topk_idx [T,k] int32, topk_w [T,k] fp32)."""
    T, d = x.shape
    E = W_router.shape[1]
    _need(x, "x", torch.bfloat16, (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    ws = workspace if workspace is not None else _workspace(route_workspace_size(T, d, E), x.device, stream)
    _check(_lib.moe_route(_ptr(x), _ptr(W_router), _ptr(router_bias), T, d, E, k, _ptr(idx), _ptr(w),
                          _ptr(ws), ws.numel(), _stream(stream)), "moe_route")
    return idx, w


def moe_permute(x, topk_idx, E: int, with_rows: bool = True, workspace=None, stream=None):
    """Step 4. Returns (offsets [E+1], perm_token [T*k], inv_perm [T,k], x_perm [T*k,d] or None)."""
    T, k = topk_idx.shape
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    d = x.shape[1] if x is not None else 64
    if x is not None:
        _need(x, "x", torch.bfloat16, (T, d))
    dev = topk_idx.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv_perm = torch.empty(T, k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device=dev) if (with_rows and x is not None) else None
    ws = workspace if workspace is not None else _workspace(permute_workspace_size(T, E, k), dev, stream)
    _check(_lib.moe_permute(_ptr(x), _ptr(topk_idx), T, d, E, k, _ptr(offsets), _ptr(perm_token), _ptr(inv_perm),
                            _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return offsets, perm_token, inv_perm, x_perm


def moe_expert_ffn(x_perm, expert_offsets, W_gate_up, W_down, workspace=None, stream=None):
    """Step 5. Returns (h [Tk,f] bf16, y_perm [Tk,d] bf16)."""
    Tk, d = x_perm.shape
    E, d2, f2 = W_gate_up.shape
    f = f2 // 2
    _need(x_perm, "x_perm", torch.bfloat16, (Tk, d))
    _need(expert_offsets, "expert_offsets", torch.int32, (E + 1,))
    _need(W_gate_up, "W_gate_up", torch.bfloat16, (E, d, 2 * f))
    _need(W_down, "W_down", torch.bfloat16, (E, f, d))
    h = torch.empty(Tk, f, dtype=torch.bfloat16, device=x_perm.device)
    y = torch.empty(Tk, d, dtype=torch.bfloat16, device=x_perm.device)
    ws = workspace if workspace is not None else _workspace(expert_ffn_workspace_size(Tk, E), x_perm.device, stream)
    _check(_lib.moe_expert_ffn(_ptr(x_perm), _ptr(expert_offsets), _ptr(W_gate_up), _ptr(W_down), Tk, d, E, f,
                               _ptr(h), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_ffn")
    return h, y


def moe_unpermute(y_perm, inv_perm, topk_w, stream=None, out=None):
    """Step 6. Returns out [T,d] bf16."""
    T, k = inv_perm.shape
    d = y_perm.shape[1]
    _need(y_perm, "y_perm", torch.bfloat16, (T * k, d))
    _need(inv_perm, "inv_perm", torch.int32, (T, k))
    _need(topk_w, "topk_w", torch.float32, (T, k))
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=y_perm.device)
    _need(out, "out", torch.bfloat16, (T, d))
    _check(_lib.moe_unpermute(_ptr(y_perm), _ptr(inv_perm), _ptr(topk_w), T, d, k, _ptr(out), _stream(stream)),
           "moe_unpermute")
    return out


def moe_mxfp8_quantize(x, stream=None, codes=None, scales=None):
    """MXFP8 (E4M3) of x [rows, cols] bf16, blocks of 32 along each row.
    Returns (codes uint8 [rows, cols], scales uint8 [rows, cols // 32])."""
    rows, cols = x.shape
    _need(x, "x", torch.bfloat16, (rows, cols))
    if codes is None:
        codes = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device=x.device)
    _need(codes, "codes", torch.uint8, (rows, cols))
    _need(scales, "scales", torch.uint8, (rows, cols // 32))
    _check(_lib.moe_mxfp8_quantize(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_mxfp8_quantize")
    return codes, scales


def moe_mxfp4_quantize(w, stream=None, codes=None, scales=None):
    """MXFP4 (E2M1) of w [K, N] or a stack [E, K, N] bf16, blocks of 32 along K
    for each column. Returns (codes uint8 shaped like w, scales uint8 with K
    replaced by K // 32)."""
    if w.dim() not in (2, 3):
        raise ValueError("w must be [K, N] or [E, K, N]")
    K, N = w.shape[-2], w.shape[-1]
    rows = w.numel() // N
    _need(w, "w", torch.bfloat16, tuple(w.shape))
    sshape = tuple(w.shape[:-2]) + (K // 32, N)
    if codes is None:
        codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(sshape, dtype=torch.uint8, device=w.device)
    _need(codes, "codes", torch.uint8, tuple(w.shape))
    _need(scales, "scales", torch.uint8, sshape)
    _check(_lib.moe_mxfp4_quantize(_ptr(w), rows, N, _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_mxfp4_quantize")
    return codes, scales


class MxExperts:
    """The experts of one layer in the MX serving format (see moe_mx_pack_experts
    in include/moe.h): packed E2M1 codes and E8M0 scale atoms of W_gate_up and
    W_down, uint8 tensors on the device."""

    def __init__(self, wq_gate_up, sf_gate_up, wq_down, sf_down, E: int, d: int, f: int):
        self.wq_gate_up, self.sf_gate_up, self.wq_down, self.sf_down = wq_gate_up, sf_gate_up, wq_down, sf_down
        self.E, self.d, self.f = E, d, f


def moe_mx_expert_bytes(E: int, d: int, f: int):
    """Bytes of (wq_gate_up, sf_gate_up, wq_down, sf_down)."""
    vals = [ctypes.c_size_t(0) for _ in range(4)]
    _check(_lib.moe_mx_expert_bytes(E, d, f, *[ctypes.byref(v) for v in vals]), "moe_mx_expert_bytes")
    return tuple(v.value for v in vals)


def moe_mx_pack_experts(W_gate_up, W_down, stream=None) -> MxExperts:
    """Quantise and pack W_gate_up [E,d,2f] and W_down [E,f,d] (bf16) to MXFP4."""
    E, d, f2 = W_gate_up.shape
    f = f2 // 2
    _need(W_gate_up, "W_gate_up", torch.bfloat16, (E, d, 2 * f))
    _need(W_down, "W_down", torch.bfloat16, (E, f, d))
    sizes = moe_mx_expert_bytes(E, d, f)
    bufs = [torch.empty(n, dtype=torch.uint8, device=W_gate_up.device) for n in sizes]
    _check(_lib.moe_mx_pack_experts(_ptr(W_gate_up), _ptr(W_down), E, d, f, *[_ptr(b) for b in bufs],
                                    _stream(stream)), "moe_mx_pack_experts")
    return MxExperts(*bufs, E, d, f)


def moe_forward_mx(x, W_router, router_bias, experts: MxExperts, k: int, out=None, workspace=None, stream=None):
    """The whole layer with MX experts. Returns out [T,d] bf16."""
    T, d = x.shape
    E, f = experts.E, experts.f
    _need(x, "x", torch.bfloat16, (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    if d != experts.d:
        raise ValueError(f"x has width {d}, the experts {experts.d}")
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _need(out, "out", torch.bfloat16, (T, d))
    nbytes = _lib.moe_forward_mx_workspace_size(T, d, E, k, f)
    ws = workspace if workspace is not None else _workspace(nbytes, x.device, stream)
    _check(_lib.moe_forward_mx(_ptr(x), _ptr(W_router), _ptr(router_bias), _ptr(experts.wq_gate_up),
                               _ptr(experts.sf_gate_up), _ptr(experts.wq_down), _ptr(experts.sf_down), T, d, E, k,
                               f, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_forward_mx")
    return out


def moe_router_logits(x, W_router, router_bias=None, stream=None, out=None):
    """Router logits [T,E] fp32 for every expert, in the canonical order."""
    T, d = x.shape
    E = W_router.shape[1]
    _need(x, "x", torch.bfloat16, (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    if out is None:
        out = torch.empty(T, E, dtype=torch.float32, device=x.device)
    _need(out, "out", torch.float32, (T, E))
    _check(_lib.moe_router_logits(_ptr(x), _ptr(W_router), _ptr(router_bias), T, d, E, _ptr(out), _stream(stream)),
           "moe_router_logits")
    return out


def moe_qb_histogram(logits, bias, k: int, lo: float, hi: float, bins: int, H=None, stream=None):
    """Quantile Balancing, first half: cutoffs alpha [T] and the margin
    histogram H [E, bins] (int64 tensor; this batch's counts are added into H).
    All-reduce H over data-parallel ranks before moe_qb_bias."""
    T, E = logits.shape
    _need(logits, "logits", torch.float32, (T, E))
    if bias is not None:
        _need(bias, "bias", torch.float32, (E,))
    if H is None:
        H = torch.zeros(E, bins, dtype=torch.int64, device=logits.device)
    _need(H, "H", torch.int64, (E, bins))
    alpha = torch.empty(T, dtype=torch.float32, device=logits.device)
    _check(_lib.moe_qb_histogram(_ptr(logits), _ptr(bias), T, E, k, float(lo), float(hi), bins, _ptr(alpha), _ptr(H),
                                 _stream(stream)), "moe_qb_histogram")
    return alpha, H


def moe_qb_bias(H, lo: float, hi: float, m_total: int, k: int, stream=None):
    """Quantile Balancing, second half: (bins [E] int32, new biases [E] fp32)."""
    E, bins = H.shape
    _need(H, "H", torch.int64, (E, bins))
    bin_out = torch.empty(E, dtype=torch.int32, device=H.device)
    bias_out = torch.empty(E, dtype=torch.float32, device=H.device)
    _check(_lib.moe_qb_bias(_ptr(H), E, bins, float(lo), float(hi), int(m_total), k, _ptr(bin_out), _ptr(bias_out),
                            _stream(stream)), "moe_qb_bias")
    return bin_out, bias_out


def moe_forward(x, W_router, router_bias, W_gate_up, W_down, k: int, out=None, workspace=None, stream=None):
    """The whole layer. Returns out [T,d] bf16."""
    T, d = x.shape
    E = W_router.shape[1]
    f = W_down.shape[1]
    _need(x, "x", torch.bfloat16, (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    _need(W_gate_up, "W_gate_up", torch.bfloat16, (E, d, 2 * f))
    _need(W_down, "W_down", torch.bfloat16, (E, f, d))
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _need(out, "out", torch.bfloat16, (T, d))
    ws = workspace if workspace is not None else _workspace(moe_forward_workspace_size(T, d, E, k, f), x.device, stream)
    _check(_lib.moe_forward(_ptr(x), _ptr(W_router), _ptr(router_bias), _ptr(W_gate_up), _ptr(W_down),
                            T, d, E, k, f, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "moe_forward")
    return out


_lib.moe_forward_host_workspace_size.argtypes = [I, I, I, I, I]
_lib.moe_forward_host_workspace_size.restype = Z
_lib.moe_forward_host.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, P]
_lib.moe_forward_host.restype = I


def moe_forward_host_workspace_size(T: int, d: int, E: int, k: int, f: int) -> int:
    return int(_lib.moe_forward_host_workspace_size(T, d, E, k, f))


def _need_host(t: torch.Tensor, name: str, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be in host memory")
    if t.dtype != torch.bfloat16 or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 tensor of shape {tuple(shape)}")


def moe_forward_host(x_host, W_router, router_bias, W_gate_up, W_down, k: int, out_host=None, workspace=None,
                     stream=None):
    """The whole layer with x and the result in host memory: the library copies
    x in, runs the pass and copies the result back, all on ``stream``.
    out_host holds the result once the stream has run the call (pin both host
    tensors for asynchronous copies)."""
    T, d = x_host.shape
    E = W_router.shape[1]
    f = W_down.shape[1]
    _need_host(x_host, "x_host", (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    _need(W_gate_up, "W_gate_up", torch.bfloat16, (E, d, 2 * f))
    _need(W_down, "W_down", torch.bfloat16, (E, f, d))
    if out_host is None:
        out_host = torch.empty(T, d, dtype=torch.bfloat16).pin_memory()
    _need_host(out_host, "out_host", (T, d))
    ws = workspace if workspace is not None else _workspace(moe_forward_host_workspace_size(T, d, E, k, f),
                                                             W_router.device, stream)
    _check(_lib.moe_forward_host(_ptr(x_host), _ptr(W_router), _ptr(router_bias), _ptr(W_gate_up), _ptr(W_down),
                                 T, d, E, k, f, _ptr(out_host), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_forward_host")
    return out_host


def moe_gather_rows(src, rows, out=None, stream=None):
    """out[i] = src[rows[i]] (bf16 rows); rows[i] = -1 gives a zero row."""
    n_src, d = src.shape
    _need(src, "src", torch.bfloat16, (n_src, d))
    n_out = rows.shape[0]
    _need(rows, "rows", torch.int32, (n_out,))
    if out is None:
        out = torch.empty(n_out, d, dtype=torch.bfloat16, device=src.device)
    _need(out, "out", torch.bfloat16, (n_out, d))
    _check(_lib.moe_gather_rows(_ptr(src), n_src, _ptr(rows), n_out, d, _ptr(out), _stream(stream)),
           "moe_gather_rows")
    return out


ACT_SWIGLU, ACT_SITU = 0, 1
SITU_BETA1, SITU_BETA2 = 4.0, 25.0


def moe_latent_forward(x, W_router, router_bias, W_dn, W_up, W_gate_up, W_down, gamma, Ws_gate_up, Ws_down, k: int,
                       act: int = ACT_SITU, beta1: float = SITU_BETA1, beta2: float = SITU_BETA2, eps: float = 1e-6,
                       out=None, workspace=None, stream=None):
    """The Stable LatentMoE layer (include/moe.h, moe_latent_forward). Returns out [T, d] bf16."""
    T, d = x.shape
    E = W_router.shape[1]
    l = W_dn.shape[1]
    f = W_down.shape[1]
    _need(x, "x", torch.bfloat16, (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    _need(W_dn, "W_dn", torch.bfloat16, (d, l))
    _need(W_up, "W_up", torch.bfloat16, (l, d))
    _need(W_gate_up, "W_gate_up", torch.bfloat16, (E, l, 2 * f))
    _need(W_down, "W_down", torch.bfloat16, (E, f, l))
    if gamma is not None:
        _need(gamma, "gamma", torch.float32, (l,))
    if Ws_gate_up is not None:
        S, fs = Ws_down.shape[0], Ws_down.shape[1]
        _need(Ws_gate_up, "Ws_gate_up", torch.bfloat16, (S, d, 2 * fs))
        _need(Ws_down, "Ws_down", torch.bfloat16, (S, fs, d))
    else:
        S, fs = 0, 0
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _need(out, "out", torch.bfloat16, (T, d))
    nbytes = _lib.moe_latent_workspace_size(T, d, l, E, k, f, S, fs)
    if nbytes == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_latent_workspace_size")
    ws = workspace if workspace is not None else _workspace(nbytes, x.device, stream)
    _check(_lib.moe_latent_forward(_ptr(x), _ptr(W_router), _ptr(router_bias), _ptr(W_dn), _ptr(W_up),
                                   _ptr(W_gate_up), _ptr(W_down), _ptr(gamma), _ptr(Ws_gate_up), _ptr(Ws_down),
                                   T, d, l, E, k, f, S, fs, int(act), float(beta1), float(beta2), float(eps),
                                   _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_latent_forward")
    return out


def get_device_error(clear: bool = True) -> int:
    """Read (and clear) the current device's error word; synchronises the device."""
    code = ctypes.c_uint32(0)
    st = _lib.moe_get_device_error(ctypes.byref(code), 1 if clear else 0)
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoEError(st, "moe_get_device_error")
    return int(code.value)


def selftest_wait_timeout(timeout_us: int, stream=None):
    _check(_lib.moe_selftest_wait_timeout(int(timeout_us), _stream(stream)), "moe_selftest_wait_timeout")


# raw C entry points, for callers that hold device pointers themselves
raw = _lib

_lib.moe_forward_timed.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, P, P]
_lib.moe_forward_timed.restype = I
TIMED_STAGES = ("router", "dispatch", "gemm_gate_up", "gemm_down", "combine")


def moe_forward_timed(x, W_router, router_bias, W_gate_up, W_down, k: int, events, out, workspace, stream=None):
    """moe_forward that records ``events`` (2 * len(TIMED_STAGES) torch.cuda.Event
    with enable_timing=True) around its kernel groups on the launching stream."""
    T, d = x.shape
    E = W_router.shape[1]
    f = W_down.shape[1]
    assert len(events) == 2 * len(TIMED_STAGES)
    for ev in events:
        if ev.cuda_event == 0:  # torch creates the CUDA event on its first record
            ev.record(torch.cuda.current_stream() if stream is None else stream)
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(ev.cuda_event) for ev in events])
    _check(_lib.moe_forward_timed(_ptr(x), _ptr(W_router), _ptr(router_bias), _ptr(W_gate_up), _ptr(W_down),
                                  T, d, E, k, f, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream), arr),
           "moe_forward_timed")
    return out

_lib.moe_route_noalloc.argtypes = [P, P, P, I, I, I, I, P, P, P]
_lib.moe_route_noalloc.restype = I
ROUTE_NOALLOC_SCRATCH_BYTES = 4 << 20


def moe_route_noalloc(x, W_router, router_bias, k: int, topk_idx, topk_w, stream=None):
    """Steps 1-3 with the library's fixed device scratch instead of a workspace,
    for callers that cannot allocate device memory. Writes into the given
    topk_idx [T,k] int32 and topk_w [T,k] fp32; allocates nothing."""
    T, d = x.shape
    E = W_router.shape[1]
    _need(x, "x", torch.bfloat16, (T, d))
    _need(W_router, "W_router", torch.float32, (d, E))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    _need(topk_w, "topk_w", torch.float32, (T, k))
    _check(_lib.moe_route_noalloc(_ptr(x), _ptr(W_router), _ptr(router_bias), T, d, E, k, _ptr(topk_idx),
                                  _ptr(topk_w), _stream(stream)), "moe_route_noalloc")
    return topk_idx, topk_w
