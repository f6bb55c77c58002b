"""Host-side checks of the C ABI: no GPU needed, no compute launched.

* the shared library loads and exports every function ``include/esa.h`` declares;
* workspace sizing follows the documented layout;
* argument, alignment and workspace errors are reported before any CUDA call;
* on a machine without a CUDA device a well-formed call reports ESA_ERR_DEVICE
  (it never falls back to a CPU path).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "esa.h")


@pytest.fixture(scope="module")
def lib():
    from gated_linear_recurrence_b200 import build
    build.build()
    from gated_linear_recurrence_b200 import esa
    return esa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(esa_[a-z_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("esa_scan_fwd", "esa_scan_bwd", "esa_step", "esa_workspace_size", "esa_workspace_init",
              "esa_check", "esa_strerror", "esa_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/esa.h but not exported"


def test_exports_are_c_linkage():
    import subprocess
    from gated_linear_recurrence_b200 import esa
    out = subprocess.run(["nm", "-D", "--defined-only", esa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(esa_[a-z_]+)\b", out))
    assert set(declared_functions()) <= exported


def test_version_and_strerror(lib):
    from gated_linear_recurrence_b200 import esa
    assert esa.esa_version() == 100
    for code in range(-7, 1):
        assert esa.esa_strerror(code)
    assert "unknown" in esa.esa_strerror(-99)


@pytest.mark.parametrize("dtype,L", [(0, 32), (1, 64), (2, 64)])
def test_workspace_size_layout(lib, dtype, L):
    B, T, H, D = 3, 1000, 5, 64          # C = 320 -> 5 channel tiles of 64
    words = B * 5 * -(-T // L) * 64

    def up(x):
        return -(-x // 256) * 256
    expect = 256
    expect = up(expect + 8 * words)      # forward chunk-end states
    expect = up(expect + 8 * words)      # backward chunk carries
    expect = up(expect + 16 * words)     # chunk maps
    assert lib.esa_workspace_size(B, T, H, D, dtype) == expect
    assert lib.esa_workspace_size(B, T, H, 256, dtype) == up(up(up(256 + 8 * B * -(-T // L) * 5 * 256)
                                                                 + 8 * B * -(-T // L) * 5 * 256)
                                                              + 16 * B * -(-T // L) * 5 * 256)


def test_workspace_size_rejects_bad_shapes(lib):
    assert lib.esa_workspace_size(1, 10, 2, 24, 1) == 0     # D not supported
    assert lib.esa_workspace_size(-1, 10, 2, 32, 1) == 0
    assert lib.esa_workspace_size(1, 10, 0, 32, 1) == 0
    assert lib.esa_workspace_size(1, 10, 2, 32, 7) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def _fwd(lib, a=0x1000, v=0x2000, q=0x3000, y=0x4000, Ef=0, B=2, T=8, H=2, D=32, mode=1, Ei=0,
         dtype=1, ws=0x10000, wsb=1 << 30):
    return lib.esa_scan_fwd(_fake(a), _fake(v), _fake(q), _fake(y), _fake(Ef) if Ef else None, B, T, H, D,
                            mode, _fake(Ei) if Ei else None, dtype, _fake(ws) if ws else None, wsb, None)


def test_fwd_argument_errors(lib):
    from gated_linear_recurrence_b200 import esa
    assert _fwd(lib, mode=2) == esa.ESA_ERR_ARG
    assert _fwd(lib, dtype=4) == esa.ESA_ERR_ARG
    assert _fwd(lib, B=-1) == esa.ESA_ERR_ARG
    assert _fwd(lib, H=0) == esa.ESA_ERR_ARG
    assert _fwd(lib, D=24) == esa.ESA_ERR_UNSUPPORTED
    assert _fwd(lib, D=512) == esa.ESA_ERR_UNSUPPORTED
    assert _fwd(lib, a=0) == esa.ESA_ERR_ARG
    assert _fwd(lib, y=0) == esa.ESA_ERR_ARG
    assert _fwd(lib, q=0x3008) == esa.ESA_ERR_ALIGN
    assert _fwd(lib, Ef=0x5004) == esa.ESA_ERR_ALIGN
    assert _fwd(lib, ws=0) == esa.ESA_ERR_WORKSPACE
    assert _fwd(lib, wsb=64) == esa.ESA_ERR_WORKSPACE


def test_bwd_and_step_argument_errors(lib):
    from gated_linear_recurrence_b200 import esa
    P = _fake
    rc = lib.esa_scan_bwd(P(0x1000), P(0x2000), P(0x3000), None, None, P(0x5000), P(0x6000), P(0x7000),
                          None, 2, 8, 2, 32, 1, None, 1, P(0x10000), 1 << 30, None)
    assert rc == esa.ESA_ERR_ARG                                   # dy missing
    rc = lib.esa_scan_bwd(P(0x1000), P(0x2000), P(0x3000), P(0x4000), None, P(0x5000), P(0x6000),
                          P(0x7001), None, 2, 8, 2, 32, 1, None, 1, P(0x10000), 1 << 30, None)
    assert rc == esa.ESA_ERR_ALIGN                                 # dq misaligned
    rc = lib.esa_step(P(0x1000), P(0x2000), P(0x3000), None, P(0x5000), 2, 2, 32, 1, 1, None)
    assert rc == esa.ESA_ERR_ARG                                   # E missing
    rc = lib.esa_step(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), 2, 2, 40, 1, 1, None)
    assert rc == esa.ESA_ERR_UNSUPPORTED


def test_no_device_is_an_error_not_a_fallback(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present; this checks the device-less path")
    from gated_linear_recurrence_b200 import esa
    assert _fwd(lib) == esa.ESA_ERR_DEVICE
    assert lib.esa_workspace_init(_fake(0x10000), 4096, None) == esa.ESA_ERR_DEVICE
    assert lib.esa_workspace_init(None, 4096, None) == esa.ESA_ERR_ARG
    assert lib.esa_workspace_init(_fake(0x10004), 4096, None) == esa.ESA_ERR_ALIGN
    assert lib.esa_step(_fake(0x1000), _fake(0x2000), _fake(0x3000), _fake(0x4000), _fake(0x5000),
                        2, 2, 32, 1, 1, None) == esa.ESA_ERR_DEVICE


def test_binding_rejects_cpu_tensors(lib):
    import torch
    from gated_linear_recurrence_b200 import esa
    x = torch.zeros(1, 4, 2, 32, dtype=torch.float16)
    with pytest.raises(TypeError):
        esa.esa_scan_fwd(x, x, x)
    with pytest.raises(TypeError):
        esa.esa_step(x[:, 0], x[:, 0], x[:, 0], torch.zeros(1, 2, 32))


def test_segment_map_argument_errors(lib):
    from gated_linear_recurrence_b200 import esa
    P = _fake
    # esa_scan_map(a, v, P, S, B, T, H, D, mode, dtype, ws, wsb, stream)
    assert lib.esa_scan_map(P(0x1000), P(0x2000), None, P(0x4000), 2, 8, 2, 32, 1, 1, P(0x10000), 1 << 30,
                            None) == esa.ESA_ERR_ARG                 # P missing
    assert lib.esa_scan_map(None, P(0x2000), P(0x3000), P(0x4000), 2, 8, 2, 32, 1, 1, P(0x10000), 1 << 30,
                            None) == esa.ESA_ERR_ARG                 # a missing
    assert lib.esa_scan_map(P(0x1000), P(0x2000), P(0x3004), P(0x4000), 2, 8, 2, 32, 1, 1, P(0x10000),
                            1 << 30, None) == esa.ESA_ERR_ALIGN
    assert lib.esa_scan_map(P(0x1000), P(0x2000), P(0x3000), P(0x4000), 2, 8, 2, 24, 1, 1, P(0x10000),
                            1 << 30, None) == esa.ESA_ERR_UNSUPPORTED
    assert lib.esa_scan_map(P(0x1000), P(0x2000), P(0x3000), P(0x4000), 2, 8, 2, 32, 1, 1, P(0x10000), 64,
                            None) == esa.ESA_ERR_WORKSPACE
    # esa_scan_bwd_map(a, v, q, dy, P, S, B, T, H, D, mode, E_init, dtype, ws, wsb, stream)
    assert lib.esa_scan_bwd_map(P(0x1000), P(0x2000), P(0x3000), None, P(0x5000), P(0x6000), 2, 8, 2, 32, 1,
                                None, 1, P(0x10000), 1 << 30, None) == esa.ESA_ERR_ARG   # dy missing
    assert lib.esa_scan_bwd_map(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), P(0x6000), 2, 8, 2, 32,
                                3, None, 1, P(0x10000), 1 << 30, None) == esa.ESA_ERR_ARG   # mode
    assert lib.esa_scan_bwd_map(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), P(0x6000), 2, 8, 2, 32,
                                1, P(0x7008), 1, P(0x10000), 1 << 30, None) == esa.ESA_ERR_ALIGN
    # esa_compose(P, S, n, count, reverse, x0, x, stream)
    assert lib.esa_compose(P(0x1000), P(0x2000), -1, 16, 0, None, P(0x3000), None) == esa.ESA_ERR_ARG
    assert lib.esa_compose(P(0x1000), P(0x2000), 2, 16, 2, None, P(0x3000), None) == esa.ESA_ERR_ARG
    assert lib.esa_compose(None, P(0x2000), 2, 16, 0, None, P(0x3000), None) == esa.ESA_ERR_ARG
    assert lib.esa_compose(P(0x1000), P(0x2000), 2, 16, 0, None, None, None) == esa.ESA_ERR_ARG
    assert lib.esa_compose(P(0x1000), P(0x2004), 2, 16, 0, None, P(0x3000), None) == esa.ESA_ERR_ALIGN


def test_segment_map_calls_need_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present; this checks the device-less path")
    from gated_linear_recurrence_b200 import esa
    P = _fake
    assert lib.esa_scan_map(P(0x1000), P(0x2000), P(0x3000), P(0x4000), 2, 8, 2, 32, 1, 1, P(0x10000), 1 << 30,
                            None) == esa.ESA_ERR_DEVICE
    assert lib.esa_scan_bwd_map(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), P(0x6000), 2, 8, 2, 32,
                                1, None, 1, P(0x10000), 1 << 30, None) == esa.ESA_ERR_DEVICE
    assert lib.esa_compose(P(0x1000), P(0x2000), 2, 16, 0, None, P(0x3000), None) == esa.ESA_ERR_DEVICE


def test_fused_forward_argument_errors(lib):
    from gated_linear_recurrence_b200 import esa
    P = _fake

    def call(x=0x1000, W=0x2000, y=0x3000, a=None, v=None, q=None, B=2, T=8, H=2, D=32, cin=128, dtype=1, wsb=1 << 30):
        return lib.esa_fused_fwd(P(x) if x else None, P(W) if W else None, P(y) if y else None, None,
                                 P(a) if a else None, P(v) if v else None, P(q) if q else None, B, T, H, D, cin, 1,
                                 None, dtype, P(0x10000), wsb, None)
    assert call(cin=96) == esa.ESA_ERR_UNSUPPORTED           # input width
    assert call(D=128) == esa.ESA_ERR_UNSUPPORTED            # head dimension above 64
    assert call(dtype=0) == esa.ESA_ERR_UNSUPPORTED          # float32 I/O
    assert call(W=0) == esa.ESA_ERR_ARG
    assert call(a=0x4000) == esa.ESA_ERR_ARG                 # a without v and q
    assert call(x=0x1008) == esa.ESA_ERR_ALIGN
    assert call(wsb=64) == esa.ESA_ERR_WORKSPACE
    if not __import__("torch").cuda.is_available():
        assert call() == esa.ESA_ERR_DEVICE
        assert call(a=0x4000, v=0x5000, q=0x6000) == esa.ESA_ERR_DEVICE


def test_fused_layer_forward_argument_errors(lib):
    from gated_linear_recurrence_b200 import esa
    P = _fake
    lib.esa_fused_layer_fwd.restype = __import__("ctypes").c_int

    def call(x=0x1000, W=0x2000, W_O=0x3000, z=0x4000, y=None, B=2, T=8, H=2, D=32, cin=64, dtype=1, wsb=1 << 30):
        return lib.esa_fused_layer_fwd(P(x) if x else None, P(W) if W else None, P(W_O) if W_O else None,
                                       P(z) if z else None, P(y) if y else None, None, B, T, H, D, cin, 1, None,
                                       dtype, P(0x10000), wsb, None)
    assert call(H=4) == esa.ESA_ERR_UNSUPPORTED              # C = 128: a row spans two channel tiles
    assert call(cin=256) == esa.ESA_ERR_UNSUPPORTED          # input width beyond the output-projection kernels
    assert call(dtype=0) == esa.ESA_ERR_UNSUPPORTED          # float32 I/O
    assert call(W_O=0) == esa.ESA_ERR_ARG
    assert call(z=0) == esa.ESA_ERR_ARG
    assert call(z=0x4008) == esa.ESA_ERR_ALIGN
    assert call(W_O=0x3004) == esa.ESA_ERR_ALIGN
    assert call(wsb=64) == esa.ESA_ERR_WORKSPACE
    if not __import__("torch").cuda.is_available():
        assert call() == esa.ESA_ERR_DEVICE                  # y may be NULL
        assert call(y=0x5000, H=1, D=64, cin=128) == esa.ESA_ERR_DEVICE


def test_fp8_inputs_are_a_scan_dtype(lib):
    import torch
    from gated_linear_recurrence_b200 import esa
    P = _fake
    # e4m3 inputs: 1-byte a, v, q; the workspace is sized like the 16-bit one (64-row slots)
    assert lib.esa_workspace_size(2, 1000, 4, 32, 3) == lib.esa_workspace_size(2, 1000, 4, 32, 1)
    rc = lib.esa_fused_fwd(P(0x1000), P(0x2000), P(0x3000), None, None, None, None, 2, 8, 2, 32, 128, 1, None, 3,
                           P(0x10000), 1 << 30, None)
    assert rc == esa.ESA_ERR_UNSUPPORTED
    if not torch.cuda.is_available():   # the scans accept it: they get as far as the device check
        rc = lib.esa_scan_bwd(P(0x1000), P(0x2000), P(0x3000), P(0x4000), None, P(0x5000), P(0x6000), P(0x7000),
                              None, 2, 8, 2, 32, 1, None, 3, P(0x10000), 1 << 30, None)
        assert rc == esa.ESA_ERR_DEVICE
        rc = lib.esa_step(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), 2, 2, 32, 1, 3, None)
        assert rc == esa.ESA_ERR_DEVICE


def test_row_strided_entry_points_check_their_strides(lib):
    """esa_scan_fwd_ld / esa_scan_bwd_ld: a row stride below C is an argument
    error, one that is not a whole number of 16-byte units an alignment
    error; a well-formed call on a machine without a device reports that."""
    from gated_linear_recurrence_b200 import esa
    P = _fake
    C = 64   # H = 2, D = 32

    def fwd(ld, dtype=1):
        return lib.esa_scan_fwd_ld(P(0x1000), P(0x2000), P(0x3000), ld, P(0x4000), None, 2, 8, 2, 32, 1, None,
                                   dtype, P(0x10000), 1 << 30, None)

    def bwd(ld_in, ld_g, dtype=1):
        return lib.esa_scan_bwd_ld(P(0x1000), P(0x2000), P(0x3000), ld_in, P(0x4000), None, P(0x5000),
                                   P(0x6000), P(0x7000), ld_g, None, 2, 8, 2, 32, 1, None, dtype, P(0x10000),
                                   1 << 30, None)

    assert fwd(0) == esa.ESA_ERR_ARG
    assert fwd(C - 8) == esa.ESA_ERR_ARG
    assert fwd(3 * C + 1) == esa.ESA_ERR_ALIGN       # 16-bit: 386 bytes
    assert fwd(3 * C + 2, dtype=0) == esa.ESA_ERR_ALIGN   # fp32: 776 bytes
    assert fwd(3 * C + 8, dtype=3) == esa.ESA_ERR_ALIGN   # e4m3: 200 bytes
    assert bwd(3 * C, C - 1) == esa.ESA_ERR_ARG
    assert bwd(3 * C, 3 * C + 4) == esa.ESA_ERR_ALIGN
    import torch
    if not torch.cuda.is_available():
        assert fwd(3 * C) == esa.ESA_ERR_DEVICE
        assert bwd(3 * C, 3 * C) == esa.ESA_ERR_DEVICE
        assert bwd(3 * C, 3 * C + 8, dtype=3) == esa.ESA_ERR_DEVICE   # e4m3 grads are fp16: 400-byte rows


def test_row_stride_of_views():
    import torch
    from gated_linear_recurrence_b200.esa import row_stride
    B, T, H, D = 2, 5, 4, 8
    C = H * D
    P = torch.empty(B, T, 3 * C)
    a, v, q = P.view(B, T, 3, H, D).unbind(2)
    assert row_stride(a) == row_stride(q) == 3 * C
    assert row_stride(torch.empty(B, T, H, D)) == C
    assert row_stride(torch.empty(B, T, D, H).transpose(2, 3)) is None          # channels not contiguous
    assert row_stride(torch.empty(T, B, H, D).transpose(0, 1)) is None          # batch inside time
    assert row_stride(torch.empty(1, 1, H, D)) == C
    assert row_stride(P.view(B, T, 3, H, D)[:, :1].unbind(2)[1]) == T * 3 * C   # T = 1: rows are batch rows
