"""The C ABI on a machine without a GPU: the library loads, exports every
entry point include/s4dplr.h declares, and rejects bad arguments on the host
before any CUDA call (no kernel is launched by these tests)."""
import ctypes
import os
import re

import pytest

from structured_state_space_dplr_b200 import _lib
from structured_state_space_dplr_b200 import build as s4build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s4dplr.h")

FAKE = 0x7f0000000000          # 256-byte aligned, never dereferenced
FAKE2 = 0x7f1000000000


@pytest.fixture(scope="module")
def lib():
    s4build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|s4_status|int)\s*\**\s*(s4\w+)\s*\(", text, re.M)))


def test_header_declares_the_expected_calls():
    names = declared_functions()
    for must in ("s4_kernel_dplr", "s4_fft_conv", "s4d_kernel_vandermonde", "s4_recurrent_step"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings(lib):
    assert _lib.status_string(0) == "S4_OK"
    assert _lib.status_string(3) == "S4_ERR_WORKSPACE"
    assert lib.s4_version() == 1


def p(v):
    return ctypes.c_void_p(v)


def kdplr(lib, H=4, Nh=32, L=1024, ptrs=None, K=FAKE2):
    ptrs = ptrs or [FAKE + 0x10000 * i for i in range(6)]
    return lib.s4_kernel_dplr(*(p(x) for x in ptrs), H, Nh, L, p(K), p(0), p(0))


def test_kernel_dplr_rejects_bad_arguments(lib):
    assert kdplr(lib, ptrs=[0, FAKE, FAKE, FAKE, FAKE, FAKE]) == _lib.S4_ERR_INVALID_ARG
    assert kdplr(lib, K=0) == _lib.S4_ERR_INVALID_ARG
    assert kdplr(lib, H=0) == _lib.S4_ERR_INVALID_ARG
    assert kdplr(lib, Nh=0) == _lib.S4_ERR_INVALID_ARG
    assert kdplr(lib, Nh=257) == _lib.S4_ERR_UNSUPPORTED
    assert kdplr(lib, H=65536) == _lib.S4_ERR_UNSUPPORTED
    for L in (0, 8, 1000, 3 * 1024, 131072, -16):
        assert kdplr(lib, L=L) == _lib.S4_ERR_UNSUPPORTED
    assert kdplr(lib, K=FAKE2 + 4) == _lib.S4_ERR_INVALID_ARG          # K not 16-byte aligned
    assert kdplr(lib, ptrs=[FAKE + 4] + [FAKE] * 5) == _lib.S4_ERR_INVALID_ARG   # complex not 8-aligned
    assert kdplr(lib, K=FAKE) == _lib.S4_ERR_INVALID_ARG               # K overlaps Lambda


def test_workspace_size(lib):
    n = ctypes.c_size_t()
    assert lib.s4_fft_conv_workspace_size(256, 4096, ctypes.byref(n)) == 0
    assert n.value >= 256 * 2 * 4096 * 8 and n.value % 256 == 0
    assert lib.s4_fft_conv_workspace_size(256, 1000, ctypes.byref(n)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_fft_conv_workspace_size(0, 1024, ctypes.byref(n)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_fft_conv_workspace_size(4, 1024, None) == _lib.S4_ERR_INVALID_ARG
    # the workspace is the spectrum alone at every length: H x 2L complex floats
    for H in (1, 3, 256):
        for lg in range(4, 17):
            L = 1 << lg
            assert lib.s4_fft_conv_workspace_size(H, L, ctypes.byref(n)) == 0
            assert n.value == (H * 2 * L * 8 + 255) // 256 * 256


def conv(lib, u=FAKE, K=FAKE + 0x10000000, D=FAKE + 0x20000000, Bt=2, H=4, L=1024, y=FAKE2,
         ws=FAKE + 0x30000000, wsb=None):
    if wsb is None:
        n = ctypes.c_size_t()
        lib.s4_fft_conv_workspace_size(H, L, ctypes.byref(n))
        wsb = n.value
    return lib.s4_fft_conv(p(u), p(K), p(D), Bt, H, L, p(y), p(ws), wsb, p(0))


def test_fft_conv_rejects_bad_arguments(lib):
    assert conv(lib, u=0) == _lib.S4_ERR_INVALID_ARG
    assert conv(lib, y=0) == _lib.S4_ERR_INVALID_ARG
    assert conv(lib, ws=0) == _lib.S4_ERR_INVALID_ARG
    assert conv(lib, Bt=0) == _lib.S4_ERR_INVALID_ARG
    assert conv(lib, L=12) == _lib.S4_ERR_UNSUPPORTED
    assert conv(lib, wsb=1024) == _lib.S4_ERR_WORKSPACE
    assert conv(lib, ws=FAKE + 0x30000000 + 64) == _lib.S4_ERR_WORKSPACE   # not 256-aligned
    assert conv(lib, u=FAKE + 8) == _lib.S4_ERR_INVALID_ARG                # u not 16-aligned
    assert conv(lib, y=FAKE + 4096) == _lib.S4_ERR_INVALID_ARG             # y overlaps u
    assert conv(lib, Bt=1 << 20, H=1 << 10, L=1 << 16) == _lib.S4_ERR_INVALID_ARG  # >= 2^40 elements


def test_steps_reject_bad_arguments(lib):
    args = [p(FAKE), p(FAKE + 0x1000000), p(FAKE + 0x2000000), p(FAKE + 0x3000000)]
    x, u, y = p(FAKE + 0x4000000), p(FAKE + 0x5000000), p(FAKE + 0x6000000)
    assert lib.s4_recurrent_step(7, *args, 2, 4, 64, x, u, y, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_recurrent_step(0, *args, 2, 4, 1024, x, u, y, p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_recurrent_step(0, *args, 2, 4, 256, x, u, y, p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_recurrent_step(1, *args, 2, 4, 300, x, u, y, p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_recurrent_step(1, *args, 0, 4, 32, x, u, y, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_recurrent_scan(1, *args, 2, 4, 32, 0, x, u, y, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_recurrent_step(1, *args, 2, 4, 32, x, u, u, p(0)) == _lib.S4_ERR_INVALID_ARG  # y aliases u
    assert lib.s4_recurrent_step(2, *args, 2, 4, 257, x, u, y, p(0)) == _lib.S4_ERR_UNSUPPORTED   # structured, Nh > 256
    assert lib.s4_recurrent_scan(2, *args, 2, 4, 32, 0, x, u, y, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_recurrent_step(2, p(FAKE + 4), *args[1:], 2, 4, 32, x, u, y, p(0)) == _lib.S4_ERR_INVALID_ARG


def test_vandermonde_and_discretize_reject_bad_arguments(lib):
    a = [p(FAKE + 0x100000 * i) for i in range(4)]
    assert lib.s4d_kernel_vandermonde(*a, 4, 32, 1000, p(FAKE2), p(0), p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4d_kernel_vandermonde(p(0), *a[1:], 4, 32, 1024, p(FAKE2), p(0), p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4d_discretize_zoh(*a[:3], 4, 300, p(FAKE2), p(FAKE2 + 0x100000), p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_dplr_discretize(*(p(FAKE + 0x100000 * i) for i in range(6)), 0, 32,
                                  p(FAKE2), p(FAKE2 + 0x100000), p(FAKE2 + 0x200000), p(0)) == _lib.S4_ERR_INVALID_ARG
    five = [p(FAKE + 0x100000 * i) for i in range(5)]
    out = [p(FAKE2), p(FAKE2 + 0x100000)]
    assert lib.s4_dplr_discretize_structured(*five, 4, 257, *out, p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_dplr_discretize_structured(*five, 0, 32, *out, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_dplr_discretize_structured(*five[:4], p(0), 4, 32, *out, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_dplr_discretize_structured(*five, 4, 32, p(FAKE2 + 4), out[1], p(0)) == _lib.S4_ERR_INVALID_ARG


def test_backward_entries_reject_bad_arguments(lib):
    n = ctypes.c_size_t()
    assert lib.s4_fft_conv_kernel_grad_workspace_size(4, 1000, ctypes.byref(n)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_fft_conv_kernel_grad_workspace_size(4, 16384, ctypes.byref(n)) == _lib.S4_OK
    assert n.value >= 4 * 2 * 16384 * 8 + 4 * 16384 * 4   # spectrum of (H, L) + one row of shares
    assert lib.s4_fft_conv_kernel_grad_workspace_size(4, 4096, ctypes.byref(n)) == _lib.S4_OK
    assert n.value == 2 * 4 * 2 * 4096 * 8
    u, dy, dK, dD = p(FAKE), p(FAKE + 0x10000000), p(FAKE2), p(FAKE2 + 0x10000000)
    ws, wsb = p(FAKE + 0x40000000), n.value
    assert lib.s4_fft_conv_kernel_grad(p(0), dy, 2, 4, 4096, dK, dD, ws, wsb, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_fft_conv_kernel_grad(u, dy, 2, 4, 1000, dK, dD, ws, wsb, p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert lib.s4_fft_conv_kernel_grad(u, dy, 2, 4, 4096, dK, dD, ws, wsb - 1, p(0)) == _lib.S4_ERR_WORKSPACE
    assert lib.s4_fft_conv_kernel_grad(u, dy, 2, 4, 4096, p(FAKE + 4096), dD, ws, wsb, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_fft_conv_apply_adjoint(p(0), ws, 2, 4, 4096, dK, wsb, p(0)) == _lib.S4_ERR_INVALID_ARG


def test_block_entries_reject_bad_arguments(lib):
    n = ctypes.c_size_t()
    assert lib.s4_glu_projection_workspace_size(0, ctypes.byref(n)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_glu_projection_workspace_size(8193, ctypes.byref(n)) == _lib.S4_ERR_INVALID_ARG
    assert lib.s4_glu_projection_workspace_size(256, ctypes.byref(n)) == _lib.S4_OK
    assert n.value == 8 * 2 * 2 * 16384         # (H/32 chunks) x (H/128 row blocks) x hi/lo x 16 KB
    assert lib.s4_glu_projection_workspace_size(100, ctypes.byref(n)) == _lib.S4_OK
    assert n.value == 4 * 1 * 2 * 16384         # ragged H rounds both counts up
    x, z, g, b = p(FAKE), p(FAKE + 0x10000000), p(FAKE2), p(FAKE2 + 0x1000)
    ln = lib.s4_layernorm_channels
    assert ln(p(0), g, b, 1e-5, 2, 4, 64, z, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert ln(x, g, b, 0.0, 2, 4, 64, z, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert ln(x, g, b, float("nan"), 2, 4, 64, z, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert ln(x, g, b, 1e-5, 2, 4, 48, z, p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert ln(x, g, b, 1e-5, 0, 4, 64, z, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert ln(x, g, b, 1e-5, 2, 4, 64, p(FAKE + 64), p(0)) == _lib.S4_ERR_INVALID_ARG   # partial overlap
    assert ln(x, g, b, 1e-5, 2, 4, 64, p(FAKE + 0x10000004), p(0)) == _lib.S4_ERR_INVALID_ARG   # misaligned
    ws, wsb = p(FAKE2 + 0x100000), 4 * 8 * 2 * 8192
    assert lib.s4_glu_projection_prepare(p(FAKE), 256, ws, wsb - 1, p(0)) == _lib.S4_ERR_WORKSPACE
    assert lib.s4_glu_projection_prepare(p(FAKE), 256, p(FAKE2 + 0x100010), wsb, p(0)) == _lib.S4_ERR_WORKSPACE
    assert lib.s4_glu_projection_prepare(p(0), 256, ws, wsb, p(0)) == _lib.S4_ERR_INVALID_ARG
    y, out, bias = p(FAKE + 0x20000000), p(FAKE + 0x30000000), p(FAKE2 + 0x2000)
    gl = lib.s4_glu_projection_residual
    assert gl(y, x, bias, ws, wsb, 2, 256, 4096, y, p(0), p(0)) == _lib.S4_ERR_INVALID_ARG       # out = y
    assert gl(y, x, bias, ws, wsb - 1, 2, 256, 4096, out, p(0), p(0)) == _lib.S4_ERR_WORKSPACE
    assert gl(y, x, bias, ws, wsb, 2, 256, 1000, out, p(0), p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert gl(y, x, p(0), ws, wsb, 2, 256, 4096, out, p(0), p(0)) == _lib.S4_ERR_INVALID_ARG
    assert gl(y, x, bias, ws, wsb, 2, 256, 4096, p(FAKE + 4096), p(0), p(0)) == _lib.S4_ERR_INVALID_ARG
    cws = p(FAKE2 + 0x40000000)
    bf = lib.s4_block_forward
    assert bf(x, g, b, 1e-5, cws, 1 << 30, bias, ws, wsb, 2, 256, 4096, x, y, out, p(0), p(0)) == \
        _lib.S4_ERR_INVALID_ARG                                                                  # z = x
    assert bf(x, g, b, 1e-5, cws, 16, bias, ws, wsb, 2, 256, 4096, z, y, out, p(0), p(0)) == _lib.S4_ERR_WORKSPACE


def test_kernel_backward_workspace(lib):
    n = ctypes.c_size_t()
    assert lib.s4_kernel_dplr_backward_workspace_size(4, 16384, ctypes.byref(n)) == _lib.S4_OK and n.value == 0
    assert lib.s4_kernel_dplr_backward_workspace_size(4, 65536, ctypes.byref(n)) == _lib.S4_OK
    # four-step intermediate, G_hat (rounded to 256 bytes), and the partial sums of
    # 64 frequency slices per channel (16 floats per mode + 1, for up to 256 modes)
    assert n.value == 4 * 65536 * 8 + 1048832 + 4 * 64 * (16 * 256 + 1) * 4
    five = [p(FAKE + 0x10000 * i) for i in range(5)]
    outs = [p(FAKE2 + 0x10000 * i) for i in range(5)]
    ldt, dK, dl = p(FAKE + 0x60000), p(FAKE + 0x1000000), p(FAKE2 + 0x60000)
    ws = p(FAKE2 + 0x10000000)
    kb = lib.s4_kernel_dplr_backward
    assert kb(*five, ldt, dK, 4, 5, 65536, *outs, dl, p(0)) == _lib.S4_ERR_UNSUPPORTED   # needs the _ws form
    kw = lib.s4_kernel_dplr_backward_ws
    assert kw(*five, ldt, dK, 4, 5, 65536, *outs, dl, p(0), 0, p(0)) == _lib.S4_ERR_WORKSPACE
    assert kw(*five, ldt, dK, 4, 5, 65536, *outs, dl, ws, n.value - 1, p(0)) == _lib.S4_ERR_WORKSPACE
    assert kw(*five, ldt, dK, 4, 5, 65536, *outs, dl, p(FAKE2 + 0x10000010), n.value, p(0)) == \
        _lib.S4_ERR_WORKSPACE                                                              # misaligned


def test_zoh_entries_reject_bad_arguments(lib):
    five = [p(FAKE + 0x10000 * i) for i in range(5)]
    ldt = p(FAKE + 0x60000)
    out = [p(FAKE2), p(FAKE2 + 0x100000), p(FAKE2 + 0x200000)]
    dz = lib.s4_dplr_discretize_zoh
    assert dz(*five, ldt, 4, 33, *out, p(0)) == _lib.S4_ERR_UNSUPPORTED          # Nh > 32
    assert dz(*five, ldt, 4, 0, *out, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert dz(p(0), *five[1:], ldt, 4, 32, *out, p(0)) == _lib.S4_ERR_INVALID_ARG
    assert dz(*five, ldt, 4, 32, out[0], out[0], out[2], p(0)) == _lib.S4_ERR_INVALID_ARG   # Abar overlaps Bbar
    kz = lib.s4_kernel_dplr_zoh
    assert kz(*five, ldt, 4, 33, 1024, p(FAKE2), p(0), p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert kz(*five, ldt, 4, 32, 1000, p(FAKE2), p(0), p(0)) == _lib.S4_ERR_UNSUPPORTED
    assert kz(*five, ldt, 4, 32, 1024, p(FAKE2 + 8), p(0), p(0)) == _lib.S4_ERR_INVALID_ARG   # K misaligned
    assert kz(*five, ldt, 4, 32, 1024, p(0), p(0), p(0)) == _lib.S4_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    import structured_state_space_dplr_b200 as s4
    u = torch.zeros(2, 2, 64)
    with pytest.raises(TypeError):
        s4.fft_conv(u, torch.zeros(2, 64), torch.zeros(2))
