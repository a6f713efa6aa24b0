"""Shared helpers for the GPU parity tests (CUDA path vs the fp64 oracle)."""
import numpy as np
import pytest

K_TOL = 1e-4   # per channel: max_k |K_gpu - K_ref| / max_k |K_ref|
Y_TOL = 2e-4   # whole tensor (or sample): ||y_gpu - y_ref||_2 / ||y_ref||_2


def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test run without a CUDA device")
    return torch


def to_dev(inp, keys=None):
    torch = torch_cuda()
    out = {}
    for k, v in inp.items():
        if isinstance(v, np.ndarray) and (keys is None or k in keys):
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).cuda()
    return out


def kernel_err(Kg, Kref):
    """max over channels of max|dK| / max|K_ref| (per-channel reading)."""
    Kg = np.asarray(Kg, np.float64)
    Kref = np.asarray(Kref, np.float64)
    return max(np.abs(Kg[i] - Kref[i]).max() / np.abs(Kref[i]).max() for i in range(Kref.shape[0]))


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def sample_times(L, n=48, seed=0):
    """Sampled output times: both ends, tile boundaries and random points."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2, 15, 16, 31, L // 4, L // 2 - 1, L // 2, L - 2, L - 1]
    t = np.unique(np.concatenate([[x for x in fixed if 0 <= x < L], rng.integers(0, L, n)]))
    return t
