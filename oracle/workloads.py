"""Oracle drivers over the seeded workloads (fp64; test infrastructure only).

They take the float32 / complex64 arrays that ``s4inputs`` hands to the CUDA
path, promote them to fp64, and apply the definitions in ``oracle.ssm``.
"""
from __future__ import annotations

import numpy as np

from . import ssm


def _f64(x):
    return np.asarray(x).astype(np.complex128 if np.iscomplexobj(x) else np.float64)


def dplr_channel_system(inp, h):
    """Full conjugate-closed (A, B_f, C_f) and dt of channel h."""
    A, Bf, Cf = ssm.full_system(_f64(inp["Lambda"][h]), _f64(inp["P"][h]), _f64(inp["Q"][h]),
                                _f64(inp["B"][h]), _f64(inp["C"][h]))
    dt = float(np.exp(np.float64(inp["log_dt"][h])))
    return A, Bf, Cf, dt


def dplr_discretized(inp, h):
    """Bilinear (Abar, Bbar, Cbar = C_f) of channel h ("The S4 kernel, from
    scratch", §3)."""
    A, Bf, Cf, dt = dplr_channel_system(inp, h)
    Ab, Bb = ssm.bilinear(A, Bf, dt)
    return Ab, Bb, Cf


def dplr_zoh_discretized(inp, h):
    """Zero-order-hold (Abar, Bbar, Cbar = C_f) of channel h's full DPLR
    system ("The S4 kernel, from scratch", §3, ZOH rule on the dense A)."""
    A, Bf, Cf, dt = dplr_channel_system(inp, h)
    Ab, Bb = ssm.zoh_dense(A, Bf, dt)
    return Ab, Bb, Cf


def dplr_zoh_kernel(inp, channels=None, imag_tol=1e-10):
    """Truncated ZOH DPLR kernel K[h, k] = Re(C_f Abar^k Bbar), k < L, by dense
    powers (no aliasing: the generating-function shortcut is bilinear only)."""
    L = inp["L"]
    channels = range(inp["H"]) if channels is None else channels
    out = []
    for h in channels:
        Ab, Bb, Cf = dplr_zoh_discretized(inp, h)
        K = ssm.truncated_kernel(Ab, Bb, Cf, L)
        kmax = np.max(np.abs(K.real))
        if np.max(np.abs(K.imag)) > imag_tol * max(kmax, 1e-300):
            raise AssertionError(f"channel {h}: kernel not real (|Im K| = {np.max(np.abs(K.imag))})")
        out.append(K.real)
    return np.array(out)


def dplr_kernel(inp, channels=None, method="closed", imag_tol=1e-10):
    """Aliased bilinear DPLR kernel K[h, 0..L-1] (fp64, real) for the given
    channels, by dense powers ("closed": one period from (I - Abar^L)^-1 Bbar;
    "brute": many periods from Bbar). Asserts max|Im K| <= imag_tol max|K|."""
    L = inp["L"]
    channels = range(inp["H"]) if channels is None else channels
    out = []
    for h in channels:
        Ab, Bb, Cf = dplr_discretized(inp, h)
        if method == "closed":
            K = ssm.aliased_kernel_closed(Ab, Bb, Cf, L)
        else:
            K, _ = ssm.aliased_kernel_bruteforce(Ab, Bb, Cf, L)
        kmax = np.max(np.abs(K.real))
        if np.max(np.abs(K.imag)) > imag_tol * max(kmax, 1e-300):
            raise AssertionError(f"channel {h}: kernel not real (|Im K| = {np.max(np.abs(K.imag))})")
        out.append(K.real)
    return np.array(out)


def s4d_params(inp, channels=None):
    """ZOH (Abar, Bbar) [len, Nh] of an S4D workload, fp64."""
    channels = list(range(inp["H"]) if channels is None else channels)
    a = _f64(inp["A"])[channels]
    B = _f64(inp["B"])[channels]
    dt = np.exp(_f64(inp["log_dt"])[channels])
    Ab = np.empty_like(a); Bb = np.empty_like(a)
    for i in range(len(channels)):
        Ab[i], Bb[i] = ssm.zoh_diag(a[i], B[i], float(dt[i]))
    return Ab, Bb


def s4d_kernel(inp, channels=None):
    channels = list(range(inp["H"]) if channels is None else channels)
    dt = np.exp(_f64(inp["log_dt"])[channels])
    return ssm.s4d_kernel(_f64(inp["A"])[channels], _f64(inp["B"])[channels],
                          _f64(inp["C"])[channels], dt, inp["L"])


def conv_full(inp, K):
    """y = K * u + D u for the whole batch (direct O(L^2) sum)."""
    return ssm.causal_conv(inp["u"], K, _f64(inp["D"]))


def conv_rows_at(inp, K_rows, rows, ts):
    """Direct sum for sampled rows (list of (b, h)) at sampled times ts.

    K_rows[i] is the kernel of rows[i]'s channel; returns [len(rows), len(ts)]."""
    u = np.stack([inp["u"][b, h] for b, h in rows]).astype(np.float64)
    D = np.array([float(inp["D"][h]) for _, h in rows])
    return ssm.causal_conv_rows_at(u, np.arange(len(rows)), np.asarray(K_rows, np.float64), D,
                                   np.asarray(ts, np.int64))


# ---------------------------------------------------------------- gradients --
def fd_gradient(fun, params, keys, eps=1e-6):
    """Central-difference gradient of the real scalar fun(params) in fp64.

    params: dict of fp64 arrays (not modified); keys: which of them to
    differentiate. For a complex entry theta the result is
    d fun / d Re(theta) + i d fun / d Im(theta); for a real entry, the
    derivative. Steps are eps * max(1, |entry|)."""
    out = {}
    for key in keys:
        base = np.asarray(params[key])
        g = np.zeros(base.shape, dtype=base.dtype)
        for idx in np.ndindex(base.shape):
            step = eps * max(1.0, abs(base[idx]))
            dirs = (1.0, 1j) if np.iscomplexobj(base) else (1.0,)
            for d in dirs:
                vals = []
                for sgn in (1.0, -1.0):
                    p = dict(params)
                    arr = base.copy()
                    arr[idx] = arr[idx] + sgn * step * d
                    p[key] = arr
                    vals.append(fun(p))
                deriv = (vals[0] - vals[1]) / (2.0 * step)
                g[idx] += deriv if d == 1.0 else 1j * deriv
        out[key] = g
    return out


def dplr_kernel_param_grad(inp, dK, channels=None, eps=1e-6):
    """Gradient of <K, dK> (K = dplr_kernel, the aliased bilinear kernel of
    "The S4 kernel, from scratch" §3-§4) with respect to each channel's
    Lambda, P, Q, B, C (complex: d/dRe + i d/dIm) and log_dt, by central
    differences of the dense fp64 definition. dK: [len(channels), L].
    Returns a dict of arrays [len(channels), Nh] (log_dt: [len(channels)])."""
    channels = list(range(inp["H"]) if channels is None else channels)
    keys = ("Lambda", "P", "Q", "B", "C", "log_dt")
    res = {k: [] for k in keys}
    for i, h in enumerate(channels):
        params = {k: _f64(inp[k])[h:h + 1] for k in keys}
        dKh = np.asarray(dK[i], np.float64)

        def fun(p):
            sub = dict(H=1, L=inp["L"], **{k: p[k] for k in keys})
            return float(np.dot(dplr_kernel(sub, [0])[0], dKh))

        g = fd_gradient(fun, params, keys, eps)
        for k in keys:
            res[k].append(g[k][0])
    return {k: np.array(v) for k, v in res.items()}


def s4d_kernel_param_grad(inp, dK, channels=None, eps=1e-6):
    """Gradient of <K, dK> (K = the S4D ZOH kernel of the "S4" wiki page,
    section "S4D": 2 Re sum_n C_n Bbar_n Abar_n^k) with respect to each
    channel's A, B, C (complex: d/dRe + i d/dIm) and log_dt, by central
    differences of ssm.s4d_kernel in fp64. dK: [len(channels), L]. Returns a
    dict of arrays [len(channels), Nh] (log_dt: [len(channels)])."""
    channels = list(range(inp["H"]) if channels is None else channels)
    keys = ("A", "B", "C", "log_dt")
    res = {k: [] for k in keys}
    for i, h in enumerate(channels):
        params = {k: _f64(inp[k])[h:h + 1] for k in keys}
        dKh = np.asarray(dK[i], np.float64)

        def fun(p):
            K = ssm.s4d_kernel(p["A"], p["B"], p["C"], np.exp(p["log_dt"]), inp["L"])
            return float(np.dot(K[0], dKh))

        g = fd_gradient(fun, params, keys, eps)
        for k in keys:
            res[k].append(g[k][0])
    return {k: np.array(v) for k, v in res.items()}
