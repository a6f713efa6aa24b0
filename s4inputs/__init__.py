"""Seeded synthetic inputs for the S4 DPLR / S4D hot path.

This module is shared by the tests, the benchmark and the oracle. It holds
NO arithmetic of the method: it only draws random numbers, loads the stored
HiPPO-LegS DPLR parameters (a data file written by ``oracle/write_fixtures.py``
from the fp64 oracle) and writes down the S4D-Lin initial values, which are an
input to the method, not a result of it.

Every array handed out is float32 (complex parameters as complex64, i.e.
interleaved (re, im) float32 pairs) so that the CUDA path and the oracle read
exactly the same numbers; the oracle promotes them to float64.

Workloads (one per entry of ``CONFIGS``):

1. S4 DPLR bilinear, H=4, N=64 (32 stored conjugate pairs), L=1024, batch 2.
2. Same parameter law, H=256, L=4096, batch 16.
3. Long sequence, H=256, L=16384, batch 8, u a flattened 128x128 binary image
   with 5 % ones (a synthetic stand-in for the Path-X sequence length named on
   the "S4" wiki page, section on the Long Range Arena).
4. Audio length, H=64, L=65536, batch 4, u = three sinusoids + N(0, 0.1^2)
   noise, log-step in [log 1e-4, log 1e-2] (stand-in for raw audio).
5. S4D-Lin diagonal ZOH, a_n = -1/2 + i*pi*n, H=1024, L=8192, batch 32.

Draw order (numpy PCG64, ``default_rng(seed)``): log_dt[H]; Re C [H,Nh];
Im C [H,Nh] (each N(0,1) scaled by 0.5/sqrt(2), so E|C|^2 = 0.25); D[H]; u.
"""
from __future__ import annotations

import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HIPPO_FIXTURE = os.path.join(_HERE, "hippo_legs_dplr_n64.txt")

CONFIGS = {
    1: dict(name="s4_dplr_bilinear_h4_n64_l1024_b2", kind="dplr", H=4, N=64, L=1024,
            Bt=2, dt_min=1e-3, dt_max=1e-1, u="normal"),
    2: dict(name="s4_dplr_bilinear_h256_n64_l4096_b16", kind="dplr", H=256, N=64, L=4096,
            Bt=16, dt_min=1e-3, dt_max=1e-1, u="normal"),
    3: dict(name="s4_dplr_bilinear_h256_n64_l16384_b8_binary", kind="dplr", H=256, N=64,
            L=16384, Bt=8, dt_min=1e-3, dt_max=1e-1, u="bernoulli"),
    4: dict(name="s4_dplr_bilinear_h64_n64_l65536_b4_audio", kind="dplr", H=64, N=64,
            L=65536, Bt=4, dt_min=1e-4, dt_max=1e-2, u="sines"),
    5: dict(name="s4d_lin_zoh_h1024_n64_l8192_b32", kind="s4d", H=1024, N=64, L=8192,
            Bt=32, dt_min=1e-3, dt_max=1e-1, u="normal"),
}


def load_hippo_dplr(N: int = 64):
    """Stored HiPPO-LegS DPLR modes (Lambda, P, B) for state size N, float64.

    The file holds the Nh = N/2 stored modes (positive imaginary part); the
    other Nh are their complex conjugates. Q = P for HiPPO-LegS.
    """
    if N != 64:
        raise ValueError("only the N=64 HiPPO-LegS fixture is stored")
    rows = []
    with open(HIPPO_FIXTURE) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([float(v) for v in line.split()])
    a = np.asarray(rows, dtype=np.float64)
    if a.shape != (N // 2, 6):
        raise ValueError(f"bad HiPPO fixture shape {a.shape}")
    lam = a[:, 0] + 1j * a[:, 1]
    p = a[:, 2] + 1j * a[:, 3]
    b = a[:, 4] + 1j * a[:, 5]
    return lam, p, b


def s4d_lin_init(Nh: int):
    """S4D-Lin initial values a_n = -1/2 + i*pi*n, B_n = 1 (the "S4" wiki page,
    section "S4D", list of initializations)."""
    n = np.arange(Nh, dtype=np.float64)
    return -0.5 + 1j * math.pi * n, np.ones(Nh, dtype=np.complex128)


def _draw_u(rng, kind, Bt, H, L):
    if kind == "normal":
        return rng.standard_normal((Bt, H, L), dtype=np.float32)
    if kind == "bernoulli":
        return (rng.random((Bt, H, L), dtype=np.float32) < 0.05).astype(np.float32)
    if kind == "sines":
        f = rng.uniform(0.001, 0.2, size=(Bt, H, 3))
        ph = rng.uniform(0.0, 2.0 * math.pi, size=(Bt, H, 3))
        t = np.arange(L, dtype=np.float64)
        u = np.zeros((Bt, H, L), dtype=np.float32)
        for i in range(3):
            u += np.sin(2.0 * math.pi * f[:, :, i, None] * t + ph[:, :, i, None]).astype(np.float32)
        u += (0.1 * rng.standard_normal((Bt, H, L), dtype=np.float32))
        return u
    if kind == "impulse":
        u = np.zeros((Bt, H, L), dtype=np.float32)
        u[:, :, 0] = 1.0
        return u
    raise ValueError(kind)


def make_inputs(cfg: int, seed: int = 0, *, H=None, Bt=None, L=None, with_u=True,
                u_kind=None):
    """Seeded inputs of workload ``cfg``; H, Bt, L may be overridden (same laws).

    Returns a dict of float32 / complex64 numpy arrays:
      dplr: Lambda, P, Q, B, C  [H, Nh] complex64; log_dt, D [H]; u [Bt, H, L]
      s4d:  A, B, C [H, Nh] complex64; log_dt, D [H]; u [Bt, H, L]
    """
    c = dict(CONFIGS[cfg])
    H = c["H"] if H is None else H
    Bt = c["Bt"] if Bt is None else Bt
    L = c["L"] if L is None else L
    Nh = c["N"] // 2
    rng = np.random.default_rng(seed)
    log_dt = rng.uniform(math.log(c["dt_min"]), math.log(c["dt_max"]), size=H)
    s = 0.5 / math.sqrt(2.0)
    c_re = rng.standard_normal((H, Nh)) * s
    c_im = rng.standard_normal((H, Nh)) * s
    D = rng.standard_normal(H)
    out = dict(cfg=cfg, H=H, Bt=Bt, L=L, Nh=Nh, kind=c["kind"],
               log_dt=log_dt.astype(np.float32), D=D.astype(np.float32),
               C=(c_re + 1j * c_im).astype(np.complex64))
    if c["kind"] == "dplr":
        lam, p, b = load_hippo_dplr(c["N"])
        out["Lambda"] = np.tile(lam, (H, 1)).astype(np.complex64)
        out["P"] = np.tile(p, (H, 1)).astype(np.complex64)
        out["Q"] = out["P"].copy()
        out["B"] = np.tile(b, (H, 1)).astype(np.complex64)
    else:
        a, b = s4d_lin_init(Nh)
        out["A"] = np.tile(a, (H, 1)).astype(np.complex64)
        out["B"] = np.tile(b, (H, 1)).astype(np.complex64)
    if with_u:
        out["u"] = _draw_u(rng, u_kind or c["u"], Bt, H, L)
    return out


def block_params(seed: int, H: int):
    """Seeded S4Block parameters around an H-channel S4 layer.

    Drawn from ``default_rng([seed, 7])`` (independent of the layer's own
    draws), in this order: gamma = 1 + 0.1 N(0,1) [H]; beta = 0.1 N(0,1) [H];
    W = N(0, 1/H) [2H, H] (rows [0, H) project to the GLU value, [H, 2H) to the
    gate); bias = 0.1 N(0,1) [2H]. eps = 1e-5. All float32.
    """
    rng = np.random.default_rng([seed, 7])
    gamma = 1.0 + 0.1 * rng.standard_normal(H)
    beta = 0.1 * rng.standard_normal(H)
    W = rng.standard_normal((2 * H, H)) / math.sqrt(H)
    bias = 0.1 * rng.standard_normal(2 * H)
    return dict(gamma=gamma.astype(np.float32), beta=beta.astype(np.float32),
                W=W.astype(np.float32), bias=bias.astype(np.float32), eps=1e-5)


def random_dplr(seed: int, H: int, Nh: int, L: int, Bt: int, *, dt_min=1e-3, dt_max=1e-1,
                re_min=-2.0, re_max=-0.1, im_max=60.0, lowrank=1.0):
    """Random (non-HiPPO) DPLR systems for generality cases.

    Re(Lambda) uniform in [re_min, re_max] (strictly negative), Im(Lambda)
    uniform in [0, im_max]; P complex normal, Q = P plus an independent
    complex-normal perturbation (so P != Q), both scaled by ``lowrank``
    (lowrank=0 gives the purely diagonal case); B and C complex normal.
    """
    rng = np.random.default_rng(seed)
    def cn(shape, scale=1.0):
        return (rng.standard_normal(shape) + 1j * rng.standard_normal(shape)) * (scale / math.sqrt(2.0))
    lam = rng.uniform(re_min, re_max, size=(H, Nh)) + 1j * rng.uniform(0.0, im_max, size=(H, Nh))
    P = cn((H, Nh), lowrank * 0.5)
    Q = P + cn((H, Nh), lowrank * 0.15)
    B = cn((H, Nh))
    C = cn((H, Nh), 0.5)
    log_dt = rng.uniform(math.log(dt_min), math.log(dt_max), size=H)
    D = rng.standard_normal(H)
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    return dict(kind="dplr", H=H, Bt=Bt, L=L, Nh=Nh,
                Lambda=lam.astype(np.complex64), P=P.astype(np.complex64),
                Q=Q.astype(np.complex64), B=B.astype(np.complex64), C=C.astype(np.complex64),
                log_dt=log_dt.astype(np.float32), D=D.astype(np.float32), u=u)
