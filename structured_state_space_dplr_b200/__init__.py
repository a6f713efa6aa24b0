"""B200 (sm_100a) S4 DPLR kernel generation and FFT convolution.

Thin Python binding over libs4dplr.so (C ABI in include/s4dplr.h). Each
function only marshals torch CUDA tensors into device pointers and the
current CUDA stream; all arithmetic runs in the library's CUDA kernels.
PyTorch provides device memory and streams.

Complex parameters are [H, Nh] complex64 tensors (or [H, Nh, 2] float32, the
real (..., 2) storage) holding the Nh stored modes of a conjugate-closed
system (N = 2 Nh).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (S4_FLAG_NONFINITE, S4_FLAG_UNSTABLE, S4_STEP_DENSE, S4_STEP_DIAG, S4_STEP_DPLR,  # noqa: F401
                   S4Error)

__all__ = [
    "kernel_dplr", "kernel_dplr_prepare", "kernel_dplr_zoh", "dplr_discretize_zoh", "layernorm_channels", "glu_projection_workspace_size", "glu_projection_prepare", "glu_projection_residual", "block_forward", "forward_dplr", "dplr_spectrum", "irfft_packed", "fft_conv", "fft_conv_workspace_size", "fft_conv_prepare", "fft_conv_apply",
    "fft_conv_static",
    "s4d_kernel_vandermonde", "dplr_discretize", "s4d_discretize_zoh", "recurrent_step",
    "recurrent_scan", "S4Error", "S4_FLAG_UNSTABLE", "S4_FLAG_NONFINITE", "S4_STEP_DENSE",
    "S4_STEP_DIAG", "S4_STEP_DPLR", "dplr_discretize_structured", "dplr_ctilde", "forward_dplr_host",
    "fft_conv_host", "fft_conv_apply_adjoint", "fft_conv_kernel_grad", "fft_conv_kernel_grad_workspace_size",
    "kernel_dplr_backward", "kernel_dplr_backward_workspace_size", "s4d_kernel_vandermonde_backward", "load",
]


def load():
    """Load libs4dplr.so now (raises if it is missing)."""
    return _lib.lib()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _cuda(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    # the library launches on the current device's current stream (and the
    # static-scratch entry point uses that device's scratch), so every
    # operand must live there: a pointer of another device would be an
    # illegal address on this one
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()} (use torch.cuda.device({t.device}))")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _cplx(t, name):
    """[H, Nh] complex64, or [H, Nh, 2] float32 viewed as complex."""
    if isinstance(t, torch.Tensor) and t.dtype == torch.float32 and t.dim() >= 1 and t.shape[-1] == 2:
        t = torch.view_as_complex(t)
    return _cuda(t, name, torch.complex64)


def _flags_ptr(flags):
    if flags is None:
        return ctypes.c_void_p(0)
    _cuda(flags, "flags", torch.int32)
    return _ptr(flags)


def kernel_dplr(Lambda, P, Q, B, C, log_dt, L, *, out=None, flags=None):
    """Aliased bilinear DPLR kernel K [H, L] (s4_kernel_dplr)."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    for x in (P, Q, B, C):
        if tuple(x.shape) != (H, Nh):
            raise ValueError("parameter shapes differ")
    if out is None:
        out = torch.empty(H, L, device=Lambda.device, dtype=torch.float32)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_kernel_dplr", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              H, Nh, int(L), _ptr(out), _flags_ptr(flags), _stream())
    return out


def dplr_spectrum(Lambda, P, Q, B, C, log_dt, L, *, out=None, flags=None):
    """Packed half spectrum of the DPLR kernel, times 1/L (s4_dplr_spectrum)."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    if out is None:
        out = torch.empty(H, L, device=Lambda.device, dtype=torch.float32)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_dplr_spectrum", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              H, Nh, int(L), _ptr(out), _flags_ptr(flags), _stream())
    return out


def irfft_packed(K):
    """In place: packed half spectrum [H, L] -> real kernel (s4_irfft_packed)."""
    K = _cuda(K, "K", torch.float32)
    H, L = K.shape
    _lib.call("s4_irfft_packed", _ptr(K), H, L, _stream())
    return K


def fft_conv_kernel_grad_workspace_size(H, L) -> int:
    """Bytes of workspace fft_conv_kernel_grad needs."""
    n = ctypes.c_size_t()
    _lib.call("s4_fft_conv_kernel_grad_workspace_size", int(H), int(L), ctypes.byref(n))
    return n.value


def fft_conv_workspace_size(H, L) -> int:
    n = ctypes.c_size_t(0)
    _lib.call("s4_fft_conv_workspace_size", int(H), int(L), ctypes.byref(n))
    return n.value


def _workspace(H, L, device, workspace):
    need = fft_conv_workspace_size(H, L)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    _cuda(workspace, "workspace", torch.uint8)
    return workspace


def fft_conv(u, K, D, *, out=None, workspace=None):
    """y = K * u + D u (causal, zero-padded FFT convolution; s4_fft_conv).

    u: [Bt, H, L] float32; K: [H, L] float32; D: [H] float32."""
    u = _cuda(u, "u", torch.float32)
    K = _cuda(K, "K", torch.float32)
    D = _cuda(D, "D", torch.float32)
    Bt, H, L = u.shape
    if tuple(K.shape) != (H, L) or tuple(D.shape) != (H,):
        raise ValueError("shape mismatch between u, K and D")
    workspace = _workspace(H, L, u.device, workspace)
    if out is None:
        out = torch.empty_like(u)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_fft_conv", _ptr(u), _ptr(K), _ptr(D), Bt, H, L, _ptr(out), _ptr(workspace),
              workspace.numel(), _stream())
    return out


def fft_conv_static(u, K, D, *, out=None):
    """s4_fft_conv with the library's own device scratch (s4_fft_conv_static),
    for callers that cannot allocate device memory. Calls that overlap on the
    GPU share that scratch and must be serialised by the caller."""
    u = _cuda(u, "u", torch.float32)
    K = _cuda(K, "K", torch.float32)
    D = _cuda(D, "D", torch.float32)
    Bt, H, L = u.shape
    if tuple(K.shape) != (H, L) or tuple(D.shape) != (H,):
        raise ValueError("shape mismatch between u, K and D")
    if out is None:
        out = torch.empty_like(u)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_fft_conv_static", _ptr(u), _ptr(K), _ptr(D), Bt, H, L, _ptr(out), _stream())
    return out


def fft_conv_prepare(K, D=None, workspace=None):
    """Spectrum of the zero-padded K + D delta_0 into a workspace
    (s4_fft_conv_prepare); D None means no feed-through term."""
    K = _cuda(K, "K", torch.float32)
    H, L = K.shape
    if D is not None:
        D = _cuda(D, "D", torch.float32)
        if tuple(D.shape) != (H,):
            raise ValueError("D must be [H]")
    workspace = _workspace(H, L, K.device, workspace)
    _lib.call("s4_fft_conv_prepare", _ptr(K), _ptr(D), H, L, _ptr(workspace), workspace.numel(), _stream())
    return workspace


def fft_conv_apply(u, workspace, *, out=None):
    """Convolution with a prepared spectrum (s4_fft_conv_apply)."""
    u = _cuda(u, "u", torch.float32)
    _cuda(workspace, "workspace", torch.uint8)
    Bt, H, L = u.shape
    if out is None:
        out = torch.empty_like(u)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_fft_conv_apply", _ptr(u), _ptr(workspace), Bt, H, L, _ptr(out), workspace.numel(),
              _stream())
    return out


# ------------------------------------------------------------ S4Block ----
def layernorm_channels(x, gamma, beta, eps=1e-5, *, out=None):
    """Layer norm over the H channels at each (b, t) of x [Bt, H, L]
    (s4_layernorm_channels); out may be x."""
    x = _cuda(x, "x", torch.float32)
    gamma = _cuda(gamma, "gamma", torch.float32)
    beta = _cuda(beta, "beta", torch.float32)
    Bt, H, L = x.shape
    if out is None:
        out = torch.empty_like(x)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_layernorm_channels", _ptr(x), _ptr(gamma), _ptr(beta), float(eps), Bt, H, L, _ptr(out),
              _stream())
    return out


def glu_projection_workspace_size(H) -> int:
    n = ctypes.c_size_t(0)
    _lib.call("s4_glu_projection_workspace_size", int(H), ctypes.byref(n))
    return n.value


def glu_projection_prepare(W, *, workspace=None):
    """Split W [2H, H] into the projection's tensor-core operand images
    (s4_glu_projection_prepare); returns the workspace."""
    W = _cuda(W, "W", torch.float32)
    H = W.shape[1]
    if tuple(W.shape) != (2 * H, H):
        raise ValueError("W must be [2H, H]")
    need = glu_projection_workspace_size(H)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    _cuda(workspace, "workspace", torch.uint8)
    _lib.call("s4_glu_projection_prepare", _ptr(W), H, _ptr(workspace), workspace.numel(), _stream())
    return workspace


def glu_projection_residual(y, x, bias, workspace, *, out=None, flags=None):
    """out = x + p[:H] * sigmoid(p[H:]), p = W y + bias at each (b, t)
    (s4_glu_projection_residual); out may be x."""
    y = _cuda(y, "y", torch.float32)
    x = _cuda(x, "x", torch.float32)
    bias = _cuda(bias, "bias", torch.float32)
    _cuda(workspace, "workspace", torch.uint8)
    Bt, H, L = y.shape
    if tuple(x.shape) != (Bt, H, L) or tuple(bias.shape) != (2 * H,):
        raise ValueError("shapes: y, x [Bt, H, L], bias [2H]")
    if out is None:
        out = torch.empty_like(x)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_glu_projection_residual", _ptr(y), _ptr(x), _ptr(bias), _ptr(workspace), workspace.numel(),
              Bt, H, L, _ptr(out), _flags_ptr(flags), _stream())
    return out


def block_forward(x, gamma, beta, eps, conv_workspace, bias, glu_workspace, *, z=None, y=None, out=None,
                  flags=None):
    """The S4Block: out = x + GLU(W S4(LN(x)) + bias) (s4_block_forward).
    conv_workspace holds the layer's prepared spectrum (fft_conv_prepare or
    kernel_dplr_prepare); glu_workspace comes from glu_projection_prepare.
    Returns (out, z, y): z = LN(x) and y = S4(z) are kept for a backward pass."""
    x = _cuda(x, "x", torch.float32)
    for t, n in ((gamma, "gamma"), (beta, "beta"), (bias, "bias")):
        _cuda(t, n, torch.float32)
    _cuda(conv_workspace, "conv_workspace", torch.uint8)
    _cuda(glu_workspace, "glu_workspace", torch.uint8)
    Bt, H, L = x.shape
    z = torch.empty_like(x) if z is None else _cuda(z, "z", torch.float32)
    y = torch.empty_like(x) if y is None else _cuda(y, "y", torch.float32)
    out = torch.empty_like(x) if out is None else _cuda(out, "out", torch.float32)
    _lib.call("s4_block_forward", _ptr(x), _ptr(gamma), _ptr(beta), float(eps), _ptr(conv_workspace),
              conv_workspace.numel(), _ptr(bias), _ptr(glu_workspace), glu_workspace.numel(), Bt, H, L,
              _ptr(z), _ptr(y), _ptr(out), _flags_ptr(flags), _stream())
    return out, z, y


def fft_conv_apply_adjoint(dy, workspace, *, out=None):
    """Backward of fft_conv_apply in u: du = sum_{t>=s} K[t-s] dy[t] + D dy[s]
    with the same prepared spectrum (s4_fft_conv_apply_adjoint)."""
    dy = _cuda(dy, "dy", torch.float32)
    _cuda(workspace, "workspace", torch.uint8)
    Bt, H, L = dy.shape
    if out is None:
        out = torch.empty_like(dy)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_fft_conv_apply_adjoint", _ptr(dy), _ptr(workspace), Bt, H, L, _ptr(out), workspace.numel(),
              _stream())
    return out


def fft_conv_kernel_grad(u, dy, *, dK=None, dD=None, workspace=None):
    """Backward of the convolution in K and D (s4_fft_conv_kernel_grad):
    (dK [H, L], dD [H]) for the batch u, dy [Bt, H, L]."""
    u = _cuda(u, "u", torch.float32)
    dy = _cuda(dy, "dy", torch.float32)
    Bt, H, L = u.shape
    if dK is None:
        dK = torch.empty(H, L, device=u.device, dtype=torch.float32)
    if dD is None:
        dD = torch.empty(H, device=u.device, dtype=torch.float32)
    _cuda(dK, "dK", torch.float32)
    _cuda(dD, "dD", torch.float32)
    if workspace is None:
        workspace = torch.empty(fft_conv_kernel_grad_workspace_size(H, L), dtype=torch.uint8, device=u.device)
    _cuda(workspace, "workspace", torch.uint8)
    _lib.call("s4_fft_conv_kernel_grad", _ptr(u), _ptr(dy), Bt, H, L, _ptr(dK), _ptr(dD), _ptr(workspace),
              workspace.numel(), _stream())
    return dK, dD


def kernel_dplr_backward(Lambda, P, Q, B, C, log_dt, dK, *, workspace=None):
    """Gradient through the DPLR kernel (s4_kernel_dplr_backward_ws): given
    dK = dLoss/dK [H, L], returns dict(Lambda, P, Q, B, C -> complex64
    [H, Nh] as dLoss/dRe + i dLoss/dIm; log_dt -> float32 [H]). For
    L > 16384 a workspace of kernel_dplr_backward_workspace_size(H, L) bytes
    is used (allocated here when not given)."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    dK = _cuda(dK, "dK", torch.float32)
    H, Nh = Lambda.shape
    L = dK.shape[-1]
    out = {k: torch.empty_like(Lambda) for k in ("Lambda", "P", "Q", "B", "C")}
    out["log_dt"] = torch.empty_like(log_dt)
    need = kernel_dplr_backward_workspace_size(H, L)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=Lambda.device)
    nbytes = 0
    if workspace is not None:
        _cuda(workspace, "workspace", torch.uint8)
        nbytes = workspace.numel()
    _lib.call("s4_kernel_dplr_backward_ws", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              _ptr(dK), H, Nh, L, _ptr(out["Lambda"]), _ptr(out["P"]), _ptr(out["Q"]), _ptr(out["B"]),
              _ptr(out["C"]), _ptr(out["log_dt"]), _ptr(workspace), nbytes, _stream())
    return out


def s4d_kernel_vandermonde_backward(A, B, C, log_dt, dK):
    """Gradient through the S4D kernel (s4d_kernel_vandermonde_backward): given
    dK [H, L], returns dict(A, B, C -> complex64 [H, Nh] as dLoss/dRe +
    i dLoss/dIm; log_dt -> float32 [H])."""
    A, B, C = (_cplx(x, n) for x, n in zip((A, B, C), "A B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    dK = _cuda(dK, "dK", torch.float32)
    H, Nh = A.shape
    L = dK.shape[-1]
    out = {k: torch.empty_like(A) for k in ("A", "B", "C")}
    out["log_dt"] = torch.empty_like(log_dt)
    _lib.call("s4d_kernel_vandermonde_backward", _ptr(A), _ptr(B), _ptr(C), _ptr(log_dt), _ptr(dK), H, Nh, L,
              _ptr(out["A"]), _ptr(out["B"]), _ptr(out["C"]), _ptr(out["log_dt"]), _stream())
    return out


def kernel_dplr_backward_workspace_size(H, L) -> int:
    """Bytes of workspace kernel_dplr_backward needs (0 for L <= 16384)."""
    n = ctypes.c_size_t(0)
    _lib.call("s4_kernel_dplr_backward_workspace_size", int(H), int(L), ctypes.byref(n))
    return n.value


def kernel_dplr_prepare(Lambda, P, Q, B, C, log_dt, D, L, *, K=None, workspace=None, flags=None):
    """K and the convolution spectrum of K + D delta_0 (s4_kernel_dplr_prepare).
    Returns (K, workspace); the workspace feeds fft_conv_apply."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    if D is not None:
        D = _cuda(D, "D", torch.float32)
    if K is None:
        K = torch.empty(H, L, device=Lambda.device, dtype=torch.float32)
    _cuda(K, "K", torch.float32)
    workspace = _workspace(H, L, Lambda.device, workspace)
    _lib.call("s4_kernel_dplr_prepare", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              _ptr(D), H, Nh, int(L), _ptr(K), _ptr(workspace), workspace.numel(), _flags_ptr(flags),
              _stream())
    return K, workspace


def forward_dplr(u, Lambda, P, Q, B, C, log_dt, D, *, out=None, K=None, workspace=None, flags=None):
    """y = K * u + D u with K the DPLR kernel, in one call (s4_forward_dplr)."""
    u = _cuda(u, "u", torch.float32)
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    D = _cuda(D, "D", torch.float32)
    Bt, H, L = u.shape
    Nh = Lambda.shape[1]
    if K is None:
        K = torch.empty(H, L, device=u.device, dtype=torch.float32)
    if out is None:
        out = torch.empty_like(u)
    _cuda(out, "out", torch.float32)
    workspace = _workspace(H, L, u.device, workspace)
    _lib.call("s4_forward_dplr", _ptr(u), _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              _ptr(D), Bt, H, Nh, L, _ptr(K), _ptr(out), _ptr(workspace), workspace.numel(),
              _flags_ptr(flags), _stream())
    return out


_copy_streams = {}


def _host(t, name):
    if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.float32:
        raise TypeError(f"{name} must be a float32 CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _host_call_buffers(u_host, y_host, u_dev, y_dev, dev):
    u_host = _host(u_host, "u_host")
    if y_host is None:
        y_host = torch.empty(u_host.shape, dtype=torch.float32, pin_memory=u_host.is_pinned())
    _host(y_host, "y_host")
    if u_dev is None:
        u_dev = torch.empty(u_host.shape, dtype=torch.float32, device=dev)
    if y_dev is None:
        y_dev = torch.empty(u_host.shape, dtype=torch.float32, device=dev)
    _cuda(u_dev, "u_dev", torch.float32)
    _cuda(y_dev, "y_dev", torch.float32)
    key = torch.cuda.current_device()
    if key not in _copy_streams:   # one upload and one download stream per device
        _copy_streams[key] = (torch.cuda.Stream(), torch.cuda.Stream())
    h2d, d2h = _copy_streams[key]
    return y_host, u_dev, y_dev, ctypes.c_void_p(h2d.cuda_stream), ctypes.c_void_p(d2h.cuda_stream)


def forward_dplr_host(u_host, Lambda, P, Q, B, C, log_dt, D, *, y_host=None, K=None, u_dev=None, y_dev=None,
                      workspace=None, flags=None, chunks=4):
    """forward_dplr with u and y in host memory (s4_forward_dplr_host): the
    uploads, convolutions and downloads of `chunks` row-pair chunks overlap.
    u_host: float32 CPU tensor [Bt, H, L] (pinned memory for overlap).
    Returns y_host, complete once torch's current stream is synchronised."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    D = _cuda(D, "D", torch.float32)
    dev = Lambda.device
    y_host, u_dev, y_dev, h2d, d2h = _host_call_buffers(u_host, y_host, u_dev, y_dev, dev)
    Bt, H, L = u_host.shape
    Nh = Lambda.shape[1]
    if K is None:
        K = torch.empty(H, L, device=dev, dtype=torch.float32)
    workspace = _workspace(H, L, dev, workspace)
    _lib.call("s4_forward_dplr_host", _ptr(u_host), _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C),
              _ptr(log_dt), _ptr(D), Bt, H, Nh, L, _ptr(y_host), _ptr(K), _ptr(u_dev), _ptr(y_dev),
              _ptr(workspace), workspace.numel(), _flags_ptr(flags), int(chunks), _stream(), h2d, d2h)
    return y_host


def fft_conv_host(u_host, K, D, *, y_host=None, u_dev=None, y_dev=None, workspace=None, chunks=4):
    """fft_conv with u and y in host memory (s4_fft_conv_host); K, D on the
    device. Returns y_host, complete once torch's current stream is
    synchronised."""
    K = _cuda(K, "K", torch.float32)
    D = _cuda(D, "D", torch.float32)
    y_host, u_dev, y_dev, h2d, d2h = _host_call_buffers(u_host, y_host, u_dev, y_dev, K.device)
    Bt, H, L = u_host.shape
    workspace = _workspace(H, L, K.device, workspace)
    _lib.call("s4_fft_conv_host", _ptr(u_host), _ptr(K), _ptr(D), Bt, H, L, _ptr(y_host), _ptr(u_dev),
              _ptr(y_dev), _ptr(workspace), workspace.numel(), int(chunks), _stream(), h2d, d2h)
    return y_host


def s4d_kernel_vandermonde(A, B, C, log_dt, L, *, out=None, flags=None):
    """S4D ZOH truncated kernel K [H, L] (s4d_kernel_vandermonde)."""
    A, B, C = (_cplx(x, n) for x, n in zip((A, B, C), "A B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = A.shape
    if out is None:
        out = torch.empty(H, L, device=A.device, dtype=torch.float32)
    _cuda(out, "out", torch.float32)
    _lib.call("s4d_kernel_vandermonde", _ptr(A), _ptr(B), _ptr(C), _ptr(log_dt), H, Nh, int(L),
              _ptr(out), _flags_ptr(flags), _stream())
    return out


def dplr_discretize(Lambda, P, Q, B, C, log_dt):
    """Dense bilinear (Abar [H,N,N], Bbar [H,N], Cfull [H,N]) complex64, N = 2 Nh."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    N = 2 * Nh
    dev = Lambda.device
    Ab = torch.empty(H, N, N, dtype=torch.complex64, device=dev)
    Bb = torch.empty(H, N, dtype=torch.complex64, device=dev)
    Cf = torch.empty(H, N, dtype=torch.complex64, device=dev)
    _lib.call("s4_dplr_discretize", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              H, Nh, _ptr(Ab), _ptr(Bb), _ptr(Cf), _stream())
    return Ab, Bb, Cf


def dplr_discretize_zoh(Lambda, P, Q, B, C, log_dt):
    """Zero-order hold of the full DPLR system (s4_dplr_discretize_zoh):
    (Abar = exp(dt A) [H,N,N], Bbar [H,N], Cfull [H,N]) complex64, N = 2 Nh,
    Nh <= 32; the dense recurrent step runs it unchanged."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    N = 2 * Nh
    dev = Lambda.device
    Ab = torch.empty(H, N, N, dtype=torch.complex64, device=dev)
    Bb = torch.empty(H, N, dtype=torch.complex64, device=dev)
    Cf = torch.empty(H, N, dtype=torch.complex64, device=dev)
    _lib.call("s4_dplr_discretize_zoh", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              H, Nh, _ptr(Ab), _ptr(Bb), _ptr(Cf), _stream())
    return Ab, Bb, Cf


def kernel_dplr_zoh(Lambda, P, Q, B, C, log_dt, L, *, out=None, flags=None):
    """Truncated kernel of the ZOH-discretised DPLR system K [H, L]
    (s4_kernel_dplr_zoh), Nh <= 32."""
    Lambda, P, Q, B, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B, C), "Lambda P Q B C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    if out is None:
        out = torch.empty(H, L, device=Lambda.device, dtype=torch.float32)
    _cuda(out, "out", torch.float32)
    _lib.call("s4_kernel_dplr_zoh", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(C), _ptr(log_dt),
              H, Nh, int(L), _ptr(out), _flags_ptr(flags), _stream())
    return out


def dplr_discretize_structured(Lambda, P, Q, B, log_dt):
    """Bilinear DPLR transition in diagonal-plus-rank-1 form for the O(Nh)
    step: (Astr [H, Nh, 3] = {a, g, beta}, Bbar [H, Nh]) complex64."""
    Lambda, P, Q, B = (_cplx(x, n) for x, n in zip((Lambda, P, Q, B), "Lambda P Q B".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    dev = Lambda.device
    Astr = torch.empty(H, Nh, 3, dtype=torch.complex64, device=dev)
    Bb = torch.empty(H, Nh, dtype=torch.complex64, device=dev)
    _lib.call("s4_dplr_discretize_structured", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(B), _ptr(log_dt),
              H, Nh, _ptr(Astr), _ptr(Bb), _stream())
    return Astr, Bb


def dplr_ctilde(Lambda, P, Q, C, log_dt, L):
    """Ctilde = C (I - Abar^L) [H, Nh] complex64: used in place of C, the
    generated kernel is the truncated one (Cbar Abar^k Bbar, k < L)."""
    Lambda, P, Q, C = (_cplx(x, n) for x, n in zip((Lambda, P, Q, C), "Lambda P Q C".split()))
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = Lambda.shape
    Ct = torch.empty_like(C)
    _lib.call("s4_dplr_ctilde", _ptr(Lambda), _ptr(P), _ptr(Q), _ptr(C), _ptr(log_dt), H, Nh, int(L),
              _ptr(Ct), _stream())
    return Ct


def s4d_discretize_zoh(A, B, log_dt):
    """Diagonal ZOH (Abar, Bbar) [H, Nh] complex64."""
    A, B = _cplx(A, "A"), _cplx(B, "B")
    log_dt = _cuda(log_dt, "log_dt", torch.float32)
    H, Nh = A.shape
    Ab = torch.empty_like(A)
    Bb = torch.empty_like(A)
    _lib.call("s4d_discretize_zoh", _ptr(A), _ptr(B), _ptr(log_dt), H, Nh, _ptr(Ab), _ptr(Bb), _stream())
    return Ab, Bb


def _step_args(Abar, Bbar, C, D, x, mode):
    Abar, Bbar, C, x = (_cplx(t, n) for t, n in zip((Abar, Bbar, C, x), "Abar Bbar C x".split()))
    D = _cuda(D, "D", torch.float32)
    Bt, H, Ns = x.shape
    if mode is None:   # from the shape of Abar
        dense = Abar.dim() == 3 and tuple(Abar.shape[1:]) == (Ns, Ns)
        struct = Abar.dim() == 3 and tuple(Abar.shape[1:]) == (Ns, 3)
        if dense and struct:
            raise ValueError("Abar [H, 3, 3] is ambiguous: pass mode=S4_STEP_DENSE or S4_STEP_DPLR")
        mode = S4_STEP_DENSE if dense else (S4_STEP_DPLR if struct else S4_STEP_DIAG)
    return mode, Abar, Bbar, C, D, x, Bt, H, Ns


def recurrent_step(Abar, Bbar, C, D, x, u_t, *, out=None, mode=None):
    """One token: x <- Abar x + Bbar u_t (in place), returns y_t [Bt, H].
    Dense if Abar is [H, N, N], structured DPLR if Abar is [H, Nh, 3]
    (from dplr_discretize_structured), diagonal (S4D) if Abar is [H, Nh]."""
    mode, Abar, Bbar, C, D, x, Bt, H, Ns = _step_args(Abar, Bbar, C, D, x, mode)
    u_t = _cuda(u_t, "u_t", torch.float32)
    if out is None:
        out = torch.empty_like(u_t)
    _lib.call("s4_recurrent_step", mode, _ptr(Abar), _ptr(Bbar), _ptr(C), _ptr(D), Bt, H, Ns,
              _ptr(x), _ptr(u_t), _ptr(out), _stream())
    return out


def recurrent_scan(Abar, Bbar, C, D, x, u, *, out=None, mode=None):
    """T tokens in one launch: u [Bt, H, T] -> y [Bt, H, T]; x updated in place."""
    mode, Abar, Bbar, C, D, x, Bt, H, Ns = _step_args(Abar, Bbar, C, D, x, mode)
    u = _cuda(u, "u", torch.float32)
    T = u.shape[-1]
    if out is None:
        out = torch.empty_like(u)
    _lib.call("s4_recurrent_scan", mode, _ptr(Abar), _ptr(Bbar), _ptr(C), _ptr(D), Bt, H, Ns, T,
              _ptr(x), _ptr(u), _ptr(out), _stream())
    return out
