"""The C-ABI library: it loads without a GPU, exports every entry point that
include/moe.h declares, sizes its workspaces consistently, and rejects bad
arguments on the host with the documented status before launching anything.
No test here launches a kernel."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_mixture_experts_route_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_unpermute", "moe_forward",
                     "moe_forward_workspace_size", "moe_status_string", "moe_get_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from sparse_mixture_experts_route_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_index_checking_build_exports_the_same_entry_points():
    from sparse_mixture_experts_route_b200 import build
    path = build.build(checks=True)
    assert "-DMOE_CHECKS" in build.flags(checks=True) and "-DMOE_CHECKS" not in build.flags()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    assert not [n for n in declared_functions() if n not in exported]


def test_library_is_sm100a_only_and_static_runtime(lib):
    from sparse_mixture_experts_route_b200 import build
    deps = subprocess.run(["ldd", build.LIB], capture_output=True, text=True).stdout
    assert "libcudart" not in deps  # runtime linked statically
    assert "libtorch" not in deps
    fl = build.flags()
    assert "arch=compute_100a,code=sm_100a" in fl


def _setup(lib):
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [I]
    for n in ("moe_route_workspace_size", "moe_permute_workspace_size", "moe_expert_ffn_workspace_size",
              "moe_forward_workspace_size"):
        getattr(lib, n).restype = Z
    lib.moe_route_workspace_size.argtypes = [I, I, I]
    lib.moe_permute_workspace_size.argtypes = [I, I, I]
    lib.moe_expert_ffn_workspace_size.argtypes = [I, I]
    lib.moe_forward_workspace_size.argtypes = [I, I, I, I, I]
    lib.moe_route.argtypes = [P, P, P, I, I, I, I, P, P, P, Z, P]
    lib.moe_permute.argtypes = [P, P, I, I, I, I, P, P, P, P, P, Z, P]
    lib.moe_expert_ffn.argtypes = [P, P, P, P, I, I, I, I, P, P, P, Z, P]
    lib.moe_unpermute.argtypes = [P, P, P, I, I, I, P, P]
    lib.moe_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, P]
    lib.moe_selftest_wait_timeout.argtypes = [I, P]
    lib.moe_forward_host_workspace_size.restype = Z
    lib.moe_forward_host_workspace_size.argtypes = [I, I, I, I, I]
    lib.moe_forward_host.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, P]
    return lib


def test_status_strings(lib):
    lib = _setup(lib)
    names = [lib.moe_status_string(i).decode() for i in range(6)]
    assert names == ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_WORKSPACE", "MOE_ERR_CUDA",
                     "MOE_ERR_DEVICE"]
    assert lib.moe_status_string(99).decode() == "MOE_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    lib = _setup(lib)
    for (T, d, E, k, f) in [(64, 128, 8, 2, 256), (4096, 7168, 384, 8, 2048), (128, 7168, 256, 4, 2048),
                            (8192, 7168, 896, 16, 512), (1, 7168, 896, 16, 512)]:
        fw = lib.moe_forward_workspace_size(T, d, E, k, f)
        rw = lib.moe_route_workspace_size(T, d, E)
        pw = lib.moe_permute_workspace_size(T, E, k)
        ew = lib.moe_expert_ffn_workspace_size(T * k, E)
        Tk = T * k
        inter = Tk * 4 * 4 + (E + 1) * 4 + Tk * d * 2 * 2 + Tk * f * 2
        # steps of <= 32 tokens run both GEMMs in one launch: a second set of
        # stream-K tickets (592 tiles x 8 epilogue warps), h_ready [E] and the chunk counter (int32), and 296
        # partial slots of 2 x 128 x 128 fp32
        a256 = lambda n: (n + 255) // 256 * 256
        fused = a256((592 * 8 + E + 1) * 4) + a256(296 * 2 * 128 * 128 * 4) if T <= 32 else 0
        assert fw >= rw + pw + ew + inter + fused
        assert fw % 256 == 0 and rw % 256 == 0 and pw % 256 == 0 and ew % 256 == 0
        assert rw >= T * E * 4
        assert fw < rw + pw + ew + inter + fused + 12 * 256
    assert lib.moe_forward_workspace_size(0, 128, 8, 2, 256) == 0


FAKE = 0x10000  # a 256-byte aligned non-null address; never dereferenced on these paths


def test_route_argument_checks(lib):
    lib = _setup(lib)
    p = ctypes.c_void_p(FAKE)
    ws = lib.moe_route_workspace_size(64, 128, 8)
    assert lib.moe_route(None, p, None, 64, 128, 8, 2, p, p, p, ws, None) == 1
    assert lib.moe_route(p, p, None, 0, 128, 8, 2, p, p, p, ws, None) == 1          # T = 0
    assert lib.moe_route(p, p, None, 64, 100, 8, 2, p, p, p, ws, None) == 1         # d % 64
    assert lib.moe_route(p, p, None, 64, 128, 8, 9, p, p, p, ws, None) == 1         # k > E
    assert lib.moe_route(p, p, None, 64, 128, 32, 17, p, p, p, 1 << 30, None) == 2  # k > 16
    assert lib.moe_route(p, p, None, 64, 128, 2048, 2, p, p, p, 1 << 30, None) == 2  # E > 1024
    assert lib.moe_route(p, p, None, 64, 128, 8, 2, p, p, p, ws - 1, None) == 3     # workspace too small
    assert lib.moe_route(p, p, None, 64, 128, 8, 2, p, p, None, ws, None) == 3      # no workspace
    assert lib.moe_route(p, p, None, 64, 128, 8, 2, p, p, ctypes.c_void_p(FAKE + 16), ws, None) == 3
    assert lib.moe_route(ctypes.c_void_p(FAKE + 2), p, None, 64, 128, 8, 2, p, p, p, ws, None) == 1  # x align


def test_other_argument_checks(lib):
    lib = _setup(lib)
    p = ctypes.c_void_p(FAKE)
    pw = lib.moe_permute_workspace_size(64, 8, 2)
    assert lib.moe_permute(p, None, 64, 128, 8, 2, p, p, p, p, p, pw, None) == 1
    assert lib.moe_permute(None, p, 64, 128, 8, 2, p, p, p, p, p, pw, None) == 1      # rows need x
    assert lib.moe_permute(p, p, 64, 128, 8, 2, p, p, p, p, p, pw - 256, None) == 3
    ew = lib.moe_expert_ffn_workspace_size(128, 8)
    assert lib.moe_expert_ffn(p, p, p, p, 128, 128, 8, 100, p, p, p, ew, None) == 1    # f % 64
    assert lib.moe_expert_ffn(p, p, p, p, 128, 128, 2000, 256, p, p, p, 1 << 20, None) == 2
    assert lib.moe_expert_ffn(p, p, p, p, 128, 128, 8, 256, p, p, p, 0, None) == 3
    assert lib.moe_unpermute(p, p, p, 64, 128, 17, p, None) == 2
    assert lib.moe_unpermute(p, p, p, 64, 120, 2, p, None) == 1
    fw = lib.moe_forward_workspace_size(64, 128, 8, 2, 256)
    assert lib.moe_forward(p, p, None, p, p, 64, 128, 8, 2, 256, None, p, fw, None) == 1
    assert lib.moe_forward(p, p, None, p, p, 64, 128, 8, 2, 250, p, p, fw, None) == 1
    assert lib.moe_forward(p, p, None, p, p, 64, 128, 8, 2, 256, p, p, fw - 256, None) == 3
    assert lib.moe_selftest_wait_timeout(0, None) == 1
    assert lib.moe_selftest_wait_timeout(2_000_000, None) == 1


def test_host_buffer_forward_checks(lib):
    """moe_forward_host: two 256-byte-rounded [T, d] bf16 staging buffers ahead
    of moe_forward's workspace; bad arguments are refused before any CUDA call."""
    lib = _setup(lib)
    for (T, d, E, k, f) in [(64, 128, 8, 2, 256), (4096, 7168, 384, 8, 2048), (3, 64, 8, 2, 64)]:
        stage = -(-T * d * 2 // 256) * 256
        assert lib.moe_forward_host_workspace_size(T, d, E, k, f) == 2 * stage + lib.moe_forward_workspace_size(
            T, d, E, k, f)
    assert lib.moe_forward_host_workspace_size(0, 128, 8, 2, 256) == 0
    p = ctypes.c_void_p(FAKE)
    hw = lib.moe_forward_host_workspace_size(64, 128, 8, 2, 256)
    assert lib.moe_forward_host(None, p, None, p, p, 64, 128, 8, 2, 256, p, p, hw, None) == 1    # no x
    assert lib.moe_forward_host(p, p, None, p, p, 64, 128, 8, 2, 256, None, p, hw, None) == 1    # no out
    assert lib.moe_forward_host(p, p, None, p, p, 64, 128, 8, 2, 250, p, p, hw, None) == 1       # f % 64
    assert lib.moe_forward_host(p, p, None, p, p, 64, 128, 8, 17, 256, p, p, hw, None) == 1      # k > E
    assert lib.moe_forward_host(p, p, None, p, p, 64, 128, 32, 17, 256, p, p, 1 << 30, None) == 2  # k > 16
    assert lib.moe_forward_host(p, p, None, p, p, 64, 128, 8, 2, 256, p, p, hw - 256, None) == 3
    assert lib.moe_forward_host(p, p, None, p, p, 64, 128, 8, 2, 256, p, ctypes.c_void_p(FAKE + 8), hw, None) == 3


def test_mx_quantize_checks(lib):
    """moe_mxfp8_quantize / moe_mxfp4_quantize refuse null pointers, a block
    axis that is not a multiple of 32, sizes out of range and misaligned
    16-byte operands before any CUDA call."""
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.moe_mxfp8_quantize.argtypes = [P, I, I, P, P, P]
    lib.moe_mxfp4_quantize.argtypes = [P, I, I, P, P, P]
    p = ctypes.c_void_p(FAKE)
    q8, q4 = lib.moe_mxfp8_quantize, lib.moe_mxfp4_quantize
    assert q8(None, 4, 64, p, p, None) == 1
    assert q8(p, 4, 64, None, p, None) == 1
    assert q8(p, 4, 64, p, None, None) == 1
    assert q8(p, 0, 64, p, p, None) == 1                          # rows = 0
    assert q8(p, 4, 48, p, p, None) == 1                          # cols % 32
    assert q8(p, 4, 16, p, p, None) == 1                          # cols < 32
    assert q8(p, 4, (1 << 20) + 32, p, p, None) == 1              # cols too large
    assert q8(ctypes.c_void_p(FAKE + 8), 4, 64, p, p, None) == 1  # x alignment
    assert q8(p, 4, 64, ctypes.c_void_p(FAKE + 4), p, None) == 1  # codes alignment
    assert q4(None, 64, 8, p, p, None) == 1
    assert q4(p, 64, 8, None, p, None) == 1
    assert q4(p, 64, 8, p, None, None) == 1
    assert q4(p, 40, 8, p, p, None) == 1                          # K % 32
    assert q4(p, 0, 8, p, p, None) == 1
    assert q4(p, 64, 0, p, p, None) == 1                          # N = 0
    assert q4(p, 64, (1 << 20) + 1, p, p, None) == 1              # N too large


def test_mx_expert_sizes_and_checks(lib):
    """MX experts: packed sizes (two E2M1 codes per byte, one E8M0 scale per 32
    codes), shape limits (d % 256, f % 128), and the host checks of
    moe_mx_pack_experts / moe_forward_mx, all before any CUDA call."""
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    ZP = ctypes.POINTER(Z)
    lib.moe_mx_expert_bytes.argtypes = [I, I, I, ZP, ZP, ZP, ZP]
    lib.moe_mx_pack_experts.argtypes = [P, P, I, I, I, P, P, P, P, P]
    lib.moe_forward_mx_workspace_size.argtypes = [I, I, I, I, I]
    lib.moe_forward_mx_workspace_size.restype = Z
    lib.moe_forward_mx.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P, P, Z, P]
    lib.moe_forward_workspace_size.argtypes = [I, I, I, I, I]
    lib.moe_forward_workspace_size.restype = Z
    v = [Z(0) for _ in range(4)]
    refs = [ctypes.byref(x) for x in v]
    assert lib.moe_mx_expert_bytes(384, 7168, 2048, *refs) == 0
    n = 384 * 7168 * 2048
    assert [x.value for x in v] == [n, n // 16, n // 2, n // 32]
    # bytes per expert parameter: 4 bits + 8 bits per 32 = 4.25 bits
    assert (v[0].value + v[1].value + v[2].value + v[3].value) * 8 == 3 * n * 4.25
    assert lib.moe_mx_expert_bytes(8, 7168 + 128, 512, *refs) == 1   # d % 256
    assert lib.moe_mx_expert_bytes(8, 7168, 576, *refs) == 1         # f % 128
    assert lib.moe_mx_expert_bytes(2048, 256, 128, *refs) == 2       # E > 1024
    assert lib.moe_mx_expert_bytes(8, 256, 128, None, *refs[1:]) == 1
    for (T, d, E, k, f) in [(1, 7168, 896, 16, 512), (4096, 7168, 384, 8, 2048), (100, 256, 8, 2, 128)]:
        mw = lib.moe_forward_mx_workspace_size(T, d, E, k, f)
        Tk = T * k
        tiles = -(-Tk // 112) + min(E, Tk)
        assert mw % 256 == 0
        # MXFP8 x and h rows, their scale atoms, bf16 y, routing tables
        assert mw >= Tk * d + Tk * f + tiles * (d // 128 + f // 128) * 512 + Tk * d * 2 + Tk * 16
    assert lib.moe_forward_mx_workspace_size(64, 7168 + 128, 8, 2, 256) == 0
    p = ctypes.c_void_p(FAKE)
    p16 = ctypes.c_void_p(FAKE + 16)   # 16- but not 32-byte aligned
    assert lib.moe_mx_pack_experts(None, p, 8, 256, 128, p, p, p, p, None) == 1
    assert lib.moe_mx_pack_experts(p, p, 8, 256, 128, p16, p, p, p, None) == 1     # wq alignment
    assert lib.moe_mx_pack_experts(p, p, 8, 256, 128, p, ctypes.c_void_p(FAKE + 8), p, p, None) == 1
    assert lib.moe_mx_pack_experts(p, p, 8, 384, 128, p, p, p, p, None) == 1      # d % 256
    mw = lib.moe_forward_mx_workspace_size(64, 256, 8, 2, 128)
    args = [p, p, None, p, p, p, p, 64, 256, 8, 2, 128, p, p, mw, None]
    assert lib.moe_forward_mx(*args[:3], p16, *args[4:]) == 1                     # wq alignment
    assert lib.moe_forward_mx(*args[:7], 64, 256, 8, 9, 128, *args[12:]) == 1     # k > E
    assert lib.moe_forward_mx(*args[:7], 64, 256, 32, 17, 128, *args[12:]) == 2   # k > 16
    assert lib.moe_forward_mx(*args[:11], 192, *args[12:]) == 1                   # f % 128
    assert lib.moe_forward_mx(*args[:14], mw - 256, None) == 3                    # workspace
    assert lib.moe_forward_mx(*args[:13], ctypes.c_void_p(FAKE + 64), mw, None) == 3


def test_qb_and_router_logits_checks(lib):
    """moe_router_logits / moe_qb_histogram / moe_qb_bias refuse bad arguments
    before any CUDA call."""
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.moe_router_logits.argtypes = [P, P, P, I, I, I, P, P]
    lib.moe_qb_histogram.argtypes = [P, P, I, I, I, F, F, I, P, P, P]
    lib.moe_qb_bias.argtypes = [P, I, I, F, F, ctypes.c_int64, I, P, P, P]
    p = ctypes.c_void_p(FAKE)
    rl, qh, qbias = lib.moe_router_logits, lib.moe_qb_histogram, lib.moe_qb_bias
    assert rl(None, p, None, 64, 128, 8, p, None) == 1
    assert rl(p, p, None, 64, 100, 8, p, None) == 1                   # d % 64
    assert rl(ctypes.c_void_p(FAKE + 2), p, None, 64, 128, 8, p, None) == 1
    assert rl(p, p, None, 64, 128, 2048, p, None) == 2                # E > 1024
    assert rl(p, p, None, 64 * 65535 + 1, 128, 8, p, None) == 2       # grid rows
    assert qh(None, None, 64, 8, 2, -4.0, 4.0, 1000, p, p, None) == 1
    assert qh(p, None, 64, 8, 8, -4.0, 4.0, 1000, p, p, None) == 1    # k >= E
    assert qh(p, None, 64, 8, 2, 4.0, -4.0, 1000, p, p, None) == 1    # hi <= lo
    assert qh(p, None, 64, 8, 2, -4.0, float("inf"), 1000, p, p, None) == 1
    assert qh(p, None, 64, 8, 2, -4.0, 4.0, 0, p, p, None) == 1       # no bins
    assert qh(p, None, 64, 8, 2, -4.0, 4.0, 2000, p, p, None) == 2    # > 1536 bins
    assert qh(p, None, 64, 64, 17, -4.0, 4.0, 1000, p, p, None) == 2  # k > 16
    assert qbias(None, 8, 1000, -4.0, 4.0, 64, 2, p, p, None) == 1
    assert qbias(p, 8, 1000, -4.0, 4.0, 0, 2, p, p, None) == 1        # no tokens
    assert qbias(p, 8, 1000, -4.0, 4.0, 64, 8, p, p, None) == 1       # k >= E
    assert qbias(p, 8, 1000, -4.0, 4.0, 64, 2, p, None, None) == 1


def test_gather_rows_checks(lib):
    """moe_gather_rows refuses bad sizes and pointers on the host; n_out = 0
    enqueues nothing and succeeds."""
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.moe_gather_rows.argtypes = [P, I64, P, I64, I, P, P]
    lib.moe_gather_rows.restype = I
    p = ctypes.c_void_p(FAKE)
    assert lib.moe_gather_rows(p, 10, p, 0, 64, p, None) == 0          # nothing to do
    assert lib.moe_gather_rows(p, 10, p, 5, 60, p, None) == 1          # d % 8
    assert lib.moe_gather_rows(p, 10, None, 5, 64, p, None) == 1       # no row list
    assert lib.moe_gather_rows(p, 10, p, 5, 64, None, None) == 1       # no output
    assert lib.moe_gather_rows(p, -1, p, 5, 64, p, None) == 1
    assert lib.moe_gather_rows(ctypes.c_void_p(FAKE + 2), 10, p, 5, 64, p, None) == 1   # unaligned rows
