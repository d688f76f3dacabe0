"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "w4a8.h")


def declared_symbols():
    text = open(HEADER).read()
    return [n for n in re.findall(r"^W4A8_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, re.M)]


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    for must in ("w4_quantize_pack", "a8_quantize_rows", "w4a8_linear", "w4a8_linear_q",
                 "w4a8_workspace_size", "w4a8_packed_ld", "w4a8_get_device_status",
                 "w4a8_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol():
    from w4a8_quantized_gemm_channel_b200 import native
    raw = ctypes.CDLL(native.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), name
        assert name in native.SIGNATURES, name


def header_defines():
    """#define NAME value (integer literals) and the status enum of the header."""
    text = open(HEADER).read()
    out = {}
    pat = r"^#define\s+(W[48]A8_\w+)\s+\(?\s*(0x[0-9a-fA-F]+|\d+)u?(?:\s*<<\s*(\d+))?"
    for name, val, shift in re.findall(pat, text, re.M):
        out[name] = int(val, 0) << (int(shift) if shift else 0)
    for name, val in re.findall(r"^\s+(W4A8_(?:OK|ERR_\w+))\s*=\s*(\d+)", text, re.M):
        out[name] = int(val)
    return out


def test_binding_constants_match_the_header():
    """The binding's flag, path and status values and size limits are the
    header's (a drift would make the Python side ask for another kernel)."""
    from w4a8_quantized_gemm_channel_b200 import native
    d = header_defines()
    pairs = {"RELU": "W4A8_RELU", "OUT_F32": "W4A8_OUT_F32", "OUT_BF16": "W4A8_OUT_BF16",
             "OUT_S32": "W4A8_OUT_S32", "STATIC_WEIGHTS": "W4A8_STATIC_WEIGHTS",
             "PATH_AUTO": "W4A8_PATH_AUTO", "PATH_GENERIC": "W4A8_PATH_GENERIC",
             "PATH_DECODE": "W4A8_PATH_DECODE", "PATH_TC": "W4A8_PATH_TC",
             "PATH_DECODE_RING": "W4A8_PATH_DECODE_RING", "PATH_DECODE_REGS": "W4A8_PATH_DECODE_REGS",
             "PATH_DECODE_SPLIT": "W4A8_PATH_DECODE_SPLIT", "PATH_TC_PAIR": "W4A8_PATH_TC_PAIR",
             "MAX_K": "W4A8_MAX_K", "OK": "W4A8_OK", "ERR_INVALID_ARG": "W4A8_ERR_INVALID_ARG",
             "ERR_UNSUPPORTED": "W4A8_ERR_UNSUPPORTED", "ERR_WORKSPACE": "W4A8_ERR_WORKSPACE",
             "ERR_CUDA": "W4A8_ERR_CUDA", "ERR_TIMEOUT": "W4A8_ERR_TIMEOUT"}
    for py, c in pairs.items():
        assert c in d, c
        assert getattr(native, py) == d[c], (py, getattr(native, py), d[c])
    # the no-allocation scratch size, as the library reports it
    assert native.NOALLOC_SCRATCH_BYTES == d["W4A8_NOALLOC_SCRATCH_BYTES"]
    assert native.lib.w4a8_noalloc_scratch_bytes() == d["W4A8_NOALLOC_SCRATCH_BYTES"]
    # every forced path value fits the path mask
    for name in pairs.values():
        if name.startswith("W4A8_PATH_"):
            assert d[name] & ~d["W4A8_PATH_MASK"] == 0


def test_size_queries():
    from w4a8_quantized_gemm_channel_b200 import native
    import oracle
    for k in (1, 2, 10, 31, 32, 33, 4096, 28672):
        assert native.packed_ld(k) == oracle.packed_ld(k)
        assert native.act_ld(k) % 16 == 0 and native.act_ld(k) >= k
    assert native.packed_ld(0) == -1
    assert native.workspace_size(0, 8) > 0
    assert native.workspace_size(-1, 8) == 0
    assert native.workspace_size(16, 4096) >= 16 * 4096 + 16 * 4


def test_status_strings():
    from w4a8_quantized_gemm_channel_b200 import native
    for s in range(6):
        assert native.lib.w4a8_status_string(s) != b"unknown status"
    assert native.lib.w4a8_status_string(6) == b"unknown status"
    assert native.lib.w4a8_status_string(99) == b"unknown status"


def _linear(lib, **kw):
    a = dict(X=16, M=4, K=64, ldx=64, Wp=4096, ldp=32, sw=8192, N=8, bias=None, flags=0,
             Y=12288, ldy=8, ws=16384, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.w4a8_linear(a["X"], a["M"], a["K"], a["ldx"], a["Wp"], a["ldp"], a["sw"], a["N"],
                           a["bias"], a["flags"], a["Y"], a["ldy"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(K=0), 1), (dict(N=0), 1), (dict(M=-1), 1), (dict(K=2097153), 1),
    (dict(ldp=16), 1),            # ldp < ceil(K/2)
    (dict(ldp=40), 1),            # not a multiple of 16
    (dict(Wp=4100), 1),           # Wp not 16-byte aligned
    (dict(ldx=63), 1), (dict(ldy=7), 1),
    (dict(Y=None), 1), (dict(sw=None), 1),
    (dict(flags=0x04 | 0x01), 1),  # S32 output with ReLU
    (dict(flags=0x04, bias=64), 1),  # S32 output with a bias
    (dict(flags=0x06), 1),         # two output formats
    (dict(flags=0x100), 1),        # unknown flag bit
    (dict(ws=None), 3), (dict(wsb=10), 3), (dict(ws=16392), 3),
    (dict(M=0), 0),                # no rows: a no-op
])
def test_linear_argument_checks(kw, want):
    """Rejected before any device work (these run without a GPU)."""
    from w4a8_quantized_gemm_channel_b200 import native
    assert _linear(native.lib, **kw) == want


def test_quantize_argument_checks():
    from w4a8_quantized_gemm_channel_b200 import native
    lib = native.lib
    assert lib.w4_quantize_pack(16, 0, 8, 8, 4096, 16, 64, None) == 1
    assert lib.w4_quantize_pack(16, 64, 8, 7, 4096, 32, 64, None) == 1   # ldw < N
    assert lib.w4_quantize_pack(16, 64, 8, 8, 4096, 16, 64, None) == 1   # ldp too small
    assert lib.w4_quantize_pack(16, 64, 8, 8, 4104, 32, 64, None) == 1   # Wp misaligned
    assert lib.a8_quantize_rows(16, 0, 64, 64, 4096, 64, 64, None) == 0  # M = 0: no-op
    assert lib.a8_quantize_rows(16, 2, 64, 64, 4096, 72, 64, None) == 1  # ldq % 16
    assert lib.a8_quantize_rows(16, 2, 64, 60, 4096, 64, 64, None) == 1  # ldx < K
    assert lib.w4a8_linear_q(24, 2, 64, 64, 64, 4096, 32, 64, 8, None, 0, 8192, 8, None) == 1  # Xq misaligned


def _linear8(lib, **kw):
    a = dict(X=16, M=4, K=64, ldx=64, Wq=4096, ldw8=64, sw=8192, N=8, bias=None, flags=0,
             Y=12288, ldy=8, ws=16384, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.w8a8_linear(a["X"], a["M"], a["K"], a["ldx"], a["Wq"], a["ldw8"], a["sw"], a["N"],
                           a["bias"], a["flags"], a["Y"], a["ldy"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(K=0), 1), (dict(N=0), 1), (dict(M=-1), 1),
    (dict(K=133145, ldx=133145, ldw8=133152), 1),  # past W8A8_MAX_K
    (dict(ldw8=48), 1),           # ldw8 < K
    (dict(ldw8=72), 1),           # not a multiple of 16
    (dict(Wq=4100), 1),           # Wq not 16-byte aligned
    (dict(ldx=63), 1), (dict(ldy=7), 1), (dict(Y=None), 1), (dict(sw=None), 1),
    (dict(flags=0x04 | 0x01), 1), (dict(flags=0x100), 1),
    (dict(ws=None), 3), (dict(wsb=10), 3),
    (dict(M=0), 0),
])
def test_w8a8_argument_checks(kw, want):
    """The W8A8 calls reject bad arguments before any device work."""
    from w4a8_quantized_gemm_channel_b200 import native
    assert _linear8(native.lib, **kw) == want


def test_w8a8_sizes_and_quantize_checks():
    from w4a8_quantized_gemm_channel_b200 import native
    import oracle
    for k in (1, 15, 16, 17, 4096, 28672):
        assert native.w8a8_ld(k) == oracle.w8_ld(k)
    assert native.w8a8_ld(0) == -1
    lib = native.lib
    assert lib.w8_quantize(16, 0, 8, 8, 4096, 16, 64, None) == 1          # K = 0
    assert lib.w8_quantize(16, 64, 8, 7, 4096, 64, 64, None) == 1         # ldw < N
    assert lib.w8_quantize(16, 64, 8, 8, 4096, 48, 64, None) == 1         # ldw8 < K
    assert lib.w8_quantize(16, 64, 8, 8, 4104, 64, 64, None) == 1         # Wq misaligned
    assert lib.w8a8_linear_q(16, 0, 64, 64, 64, 4096, 64, 64, 8, None, 0, 8192, 8, None) == 0  # M = 0
    assert lib.w8a8_linear_q(24, 2, 64, 64, 64, 4096, 64, 64, 8, None, 0, 8192, 8, None) == 1  # Xq misaligned


def test_no_device_means_unsupported_not_a_crash():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    from w4a8_quantized_gemm_channel_b200 import native
    assert _linear(native.lib) == 2


def test_last_launch_count_starts_at_zero_per_thread():
    import threading
    from w4a8_quantized_gemm_channel_b200 import native
    seen = []
    t = threading.Thread(target=lambda: seen.append((native.last_launch_count(), native.last_kernel())))
    t.start()
    t.join()
    assert seen == [(0, "")]


def test_selftest_timeout_rejects_bad_limits():
    from w4a8_quantized_gemm_channel_b200 import native
    assert native.lib.w4a8_selftest_timeout(10, None) == native.ERR_INVALID_ARG
    assert native.lib.w4a8_selftest_timeout(10 ** 12, None) == native.ERR_INVALID_ARG


def test_grouped_rejects_bad_arguments_before_the_device():
    import ctypes as ct
    from w4a8_quantized_gemm_channel_b200 import native
    P = native.Problem
    assert native.lib.w4a8_linear_grouped(None, 0, 0, None) == native.OK        # nothing to do
    assert native.lib.w4a8_linear_grouped(None, 1, 0, None) == native.ERR_INVALID_ARG
    arr = (P * 1)(P(16, 4096, 8192, None, 12288, 5, 64, 64, 32, 8, 8))     # M = 5 > 4
    assert native.lib.w4a8_linear_grouped(arr, 1, 0, None) == native.ERR_INVALID_ARG
    arr = (P * 1)(P(16, 4096, 8192, None, 12288, 2, 64, 64, 32, 8, 8))
    assert native.lib.w4a8_linear_grouped(arr, 1, native.PATH_TC, None) == native.ERR_INVALID_ARG
    assert ct.sizeof(P) == 64


def test_zero_point_calls_check_arguments_before_the_device():
    """The zero-point entry points reject bad arguments (and report the
    workspace size) without touching a device."""
    from w4a8_quantized_gemm_channel_b200 import native
    lib = native.lib
    m, k, n = 4, 64, 8
    need = lib.w4z_workspace_size(m, k, n)
    # INT8 rows + scales + row sums + INT32 accumulators, each 256-aligned, + slack
    assert need >= m * 64 + 4 * m + 4 * m + 4 * m * n
    assert lib.w4z_workspace_size(-1, k, n) == 0 and lib.w4z_workspace_size(m, 0, n) == 0
    assert lib.w4z_workspace_size(m, k, 0) == 0
    args = dict(X=16, M=m, K=k, ldx=k, Wp=4096, ldp=32, sa=8192, zp=8448, N=n, bias=None, flags=0,
                Y=12288, ldy=n, ws=16384, wsb=need, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.w4z_linear(a["X"], a["M"], a["K"], a["ldx"], a["Wp"], a["ldp"], a["sa"], a["zp"], a["N"],
                              a["bias"], a["flags"], a["Y"], a["ldy"], a["ws"], a["wsb"], a["stream"])
    assert call(zp=None) == 1            # zero points missing
    assert call(zp=8450) == 1            # misaligned zero points
    assert call(ldp=16) == 1             # ldp < ceil(K/2)
    assert call(K=0) == 1
    assert call(ws=None) == 3 and call(wsb=need - 1) == 3
    assert call(M=0) == 0                # no rows: a no-op
    assert lib.w4z_quantize_pack(16, k, n, n, 4096, 32, 64, None, None) == 1   # zp missing
    assert lib.w4z_quantize_pack(16, k, n, n - 1, 4096, 32, 64, 128, None) == 1  # ldw < N
    assert lib.w4z_linear_q(24, 2, k, k, 64, 4096, 32, 64, 128, n, None, 0, 8192, n, 16384, need, None) == 1


def test_group_wise_calls_check_arguments_before_the_device():
    from w4a8_quantized_gemm_channel_b200 import native
    lib = native.lib
    assert lib.w4g_groups(1) == 1 and lib.w4g_groups(128) == 1 and lib.w4g_groups(129) == 2
    assert lib.w4g_groups(0) == -1
    m, k, n = 4, 300, 8
    a = dict(X=16, M=m, K=k, ldx=k, Wp=4096, ldp=160, sa=8192, zp=8448, N=n, bias=None, flags=0,
             Y=12288, ldy=n, ws=16384, wsb=1 << 20, stream=None)

    def call(**kw):
        b = dict(a, **kw)
        return lib.w4g_linear(b["X"], b["M"], b["K"], b["ldx"], b["Wp"], b["ldp"], b["sa"], b["zp"], b["N"],
                              b["bias"], b["flags"], b["Y"], b["ldy"], b["ws"], b["wsb"], b["stream"])
    assert call(flags=0x04) == 1      # INT32 output: no single accumulator in this form
    assert call(zp=None) == 1 and call(ldp=144) == 1 and call(ws=None) == 3
    assert call(M=0) == 0
    assert lib.w4g_quantize_pack(16, k, n, n, 4096, 160, 64, None, None) == 1


def test_no_multicast_bulk_loads_in_the_kernels():
    """No TMA or bulk copy in the kernel sources multicasts across a cluster:
    every load lands in the issuing CTA's own shared memory (the CTA-pair
    GEMM multicasts only its tcgen05.commit mbarrier arrives)."""
    csrc = os.path.join(ROOT, "w4a8_quantized_gemm_channel_b200", "csrc")
    bad = []
    for name in sorted(os.listdir(csrc)):
        if not name.endswith((".cu", ".cuh")):
            continue
        for i, line in enumerate(open(os.path.join(csrc, name)), 1):
            if "cp.async.bulk" in line and "multicast" in line:
                bad.append(f"{name}:{i}")
    assert not bad, bad
