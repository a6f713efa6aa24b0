"""ctypes access to libs4dplr.so (the C ABI declared in include/s4dplr.h).

Loading fails loudly if the library has not been built: there is no other
implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs4dplr.so")

S4_OK, S4_ERR_INVALID_ARG, S4_ERR_UNSUPPORTED, S4_ERR_WORKSPACE, S4_ERR_CUDA = range(5)
S4_FLAG_UNSTABLE = 1
S4_FLAG_NONFINITE = 2
S4_FLAG_TIMEOUT = 4
S4_STEP_DENSE, S4_STEP_DIAG, S4_STEP_DPLR = 0, 1, 2

_p = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

# name -> (restype, argtypes)
SIGNATURES = {
    "s4_status_string": (ctypes.c_char_p, [_i]),
    "s4_last_cuda_error": (_i, []),
    "s4_version": (_i, []),
    "s4_kernel_dplr": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p]),
    "s4_dplr_spectrum": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p]),
    "s4_irfft_packed": (_i, [_p, _i, _i, _p]),
    "s4_fft_conv_workspace_size": (_i, [_i, _i, ctypes.POINTER(_sz)]),
    "s4_dplr_discretize_zoh": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _p, _p, _p, _p]),
    "s4_kernel_dplr_zoh": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p]),
    "s4d_kernel_vandermonde_backward": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p, _p, _p]),
    "s4_layernorm_channels": (_i, [_p, _p, _p, ctypes.c_float, _i, _i, _i, _p, _p]),
    "s4_glu_projection_workspace_size": (_i, [_i, ctypes.POINTER(_sz)]),
    "s4_glu_projection_prepare": (_i, [_p, _i, _p, _sz, _p]),
    "s4_glu_projection_residual": (_i, [_p, _p, _p, _p, _sz, _i, _i, _i, _p, _p, _p]),
    "s4_block_forward": (_i, [_p, _p, _p, ctypes.c_float, _p, _sz, _p, _p, _sz, _i, _i, _i, _p, _p, _p, _p, _p]),
    "s4_fft_conv": (_i, [_p, _p, _p, _i, _i, _i, _p, _p, _sz, _p]),
    "s4_fft_conv_prepare": (_i, [_p, _p, _i, _i, _p, _sz, _p]),
    "s4_fft_conv_apply": (_i, [_p, _p, _i, _i, _i, _p, _sz, _p]),
    "s4_fft_conv_apply_adjoint": (_i, [_p, _p, _i, _i, _i, _p, _sz, _p]),
    "s4_fft_conv_kernel_grad_workspace_size": (_i, [_i, _i, ctypes.POINTER(ctypes.c_size_t)]),
    "s4_fft_conv_kernel_grad": (_i, [_p, _p, _i, _i, _i, _p, _p, _p, _sz, _p]),
    "s4_kernel_dplr_backward": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "s4_kernel_dplr_backward_workspace_size": (_i, [_i, _i, ctypes.POINTER(_sz)]),
    "s4_kernel_dplr_backward_ws": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p,
                                        _sz, _p]),
    "s4_fft_conv_static": (_i, [_p, _p, _p, _i, _i, _i, _p, _p]),
    "s4_kernel_dplr_prepare": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _p, _sz, _p, _p]),
    "s4_forward_dplr": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _sz, _p, _p]),
    "s4d_kernel_vandermonde": (_i, [_p, _p, _p, _p, _i, _i, _i, _p, _p, _p]),
    "s4_dplr_discretize": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _p, _p, _p, _p]),
    "s4_dplr_discretize_structured": (_i, [_p, _p, _p, _p, _p, _i, _i, _p, _p, _p]),
    "s4_dplr_ctilde": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "s4_fft_conv_host": (_i, [_p, _p, _p, _i, _i, _i, _p, _p, _p, _p, _sz, _i, _p, _p, _p]),
    "s4_forward_dplr_host": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _sz, _p,
                                  _i, _p, _p, _p]),
    "s4d_discretize_zoh": (_i, [_p, _p, _p, _i, _i, _p, _p, _p]),
    "s4_recurrent_step": (_i, [_i, _p, _p, _p, _p, _i, _i, _i, _p, _p, _p, _p]),
    "s4_recurrent_scan": (_i, [_i, _p, _p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _p]),
}

_lib = None


class S4Error(RuntimeError):
    def __init__(self, fn, status, cuda_err=0):
        self.status = status
        self.cuda_error = cuda_err
        msg = f"{fn} returned {status_string(status)}"
        if status == S4_ERR_CUDA:
            msg += f" (cudaError {cuda_err})"
        super().__init__(msg)


def lib():
    """The loaded library (raises OSError if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with "
                          "`python -m structured_state_space_dplr_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().s4_status_string(int(s)).decode()


def call(name: str, *args) -> None:
    """Call an entry point and raise S4Error on any status other than S4_OK."""
    st = getattr(lib(), name)(*args)
    if st != S4_OK:
        raise S4Error(name, st, lib().s4_last_cuda_error() if st == S4_ERR_CUDA else 0)
