"""Plain fp64 definitions of what the S4 hot path computes (oracle).

Test infrastructure only. Every function is the definition on the pages,
written out with dense linear algebra, so it can be checked by eye:

* "The S4 kernel, from scratch" (p1) -- §1 the SSM, §3 discretisation,
  §4 kernel via the generating function (+ "Aliasing"), §5 the two views;
* "S4" wiki page (p2), section "S4D" -- the diagonal variant;
* glossary page "Structured state-space sequence model and S4" (p4) --
  recurrence/convolution duality and the scalar ZOH worked example.

Readings of points the pages leave open (listed in the design notes):
* the stored Nh modes are half of a conjugate-closed system of N = 2 Nh modes
  (the partner of mode n is its complex conjugate, C included), so K is real;
* bilinear: Abar = (I - dt/2 A)^-1 (I + dt/2 A), Bbar = (I - dt/2 A)^-1 dt B,
  Cbar = C -- the unique choice that reproduces the generating function
  (2/(1+z)) C (g(z) I - A)^-1 B printed in §4;
* K is the aliased kernel sum_p K_{k+pL} (§4 "Aliasing");
* roots of unity z_j = exp(-2 pi i j / L) (K_hat is the forward DFT of K);
* y[t] includes K[0] u[t] (the kernel starts at C Bbar, §4) and D u[t] (§1).
"""
from __future__ import annotations

import numpy as np
import scipy.linalg

from . import _cloops


# ---------------------------------------------------------------- systems --
def full_system(Lambda, P, Q, B, C):
    """Conjugate-closed full-N DPLR system from Nh stored modes.

    A = diag(Lambda_f) - P_f Q_f^*  ("The S4 kernel, from scratch", §2), with
    X_f = [X, conj(X)] for X in Lambda, P, Q, B, C. Returns (A [N,N], B_f, C_f).
    """
    cat = lambda x: np.concatenate([np.asarray(x, np.complex128),
                                    np.conj(np.asarray(x, np.complex128))])
    Lf, Pf, Qf, Bf, Cf = cat(Lambda), cat(P), cat(Q), cat(B), cat(C)
    A = np.diag(Lf) - np.outer(Pf, Qf.conj())
    return A, Bf, Cf


def bilinear(A, B, dt):
    """Bilinear (Tustin) discretisation ("The S4 kernel, from scratch", §3).

    Abar = (I - dt/2 A)^-1 (I + dt/2 A);  Bbar = (I - dt/2 A)^-1 dt B.
    For a scalar a this is the printed (1 + dt a/2)/(1 - dt a/2).
    """
    A = np.atleast_2d(np.asarray(A, np.complex128))
    N = A.shape[0]
    I = np.eye(N)
    M = I - (dt / 2.0) * A
    Ab = np.linalg.solve(M, I + (dt / 2.0) * A)
    Bb = np.linalg.solve(M, dt * np.asarray(B, np.complex128).reshape(N, -1)).reshape(np.shape(B))
    return Ab, Bb


def zoh_diag(a, B, dt):
    """Zero-order hold for a diagonal system ("The S4 kernel, from scratch",
    §3): Abar = exp(dt a), Bbar = (exp(dt a) - 1)/a * B, with the Taylor
    series dt (1 + x/2 + x^2/6 + x^3/24 + x^4/120), x = dt a, when |x| < 1e-4
    (the "Taylor fallback near a -> 0")."""
    a = np.asarray(a, np.complex128)
    x = dt * a
    Ab = np.exp(x)
    ratio = np.empty_like(x)
    small = np.abs(x) < 1e-4
    xs = x[small]
    ratio[small] = dt * (1 + xs / 2 + xs ** 2 / 6 + xs ** 3 / 24 + xs ** 4 / 120)
    big = ~small
    ratio[big] = (Ab[big] - 1.0) / a[big]
    return Ab, ratio * np.asarray(B, np.complex128)


def zoh_dense(A, B, dt):
    """Zero-order hold for a dense (non-diagonal) system, the rule of "The S4
    kernel, from scratch", §3 applied to the full DPLR matrix:
    Abar = exp(dt A), Bbar = (integral_0^dt exp(A s) ds) B. Both come from one
    matrix exponential (scipy.linalg.expm) of the augmented matrix
    [[dt A, dt B], [0, 0]]: its top-left block is Abar and its top-right column
    is Bbar. No inverse of A is needed, so a singular A is fine."""
    A = np.atleast_2d(np.asarray(A, np.complex128))
    N = A.shape[0]
    X = np.zeros((N + 1, N + 1), np.complex128)
    X[:N, :N] = dt * A
    X[:N, N] = dt * np.asarray(B, np.complex128).reshape(N)
    E = scipy.linalg.expm(X)
    return E[:N, :N], E[:N, N]


# ------------------------------------------------------- generating function --
def roots_of_unity(L):
    """z_j = exp(-2 pi i j / L), j = 0..L-1 (reading of "L-th roots of unity")."""
    return np.exp(-2j * np.pi * np.arange(L) / L)


def generating_function_discrete(Ab, Bb, C, z):
    """K_hat(z) = sum_{k>=0} Cbar Abar^k Bbar z^k = Cbar (I - z Abar)^-1 Bbar
    (the infinite generating function of §4), by dense solves."""
    N = Ab.shape[0]
    I = np.eye(N)
    return np.array([C @ np.linalg.solve(I - zz * Ab, Bb) for zz in np.atleast_1d(z)])


def generating_function_continuous(A, B, C, dt, z):
    """(2/(1+z)) C (g(z) I - A)^-1 B with g(z) = (2/dt)(1-z)/(1+z)
    ("The S4 kernel, from scratch", §4), by dense solves (z != -1)."""
    N = A.shape[0]
    I = np.eye(N)
    out = []
    for zz in np.atleast_1d(z):
        g = (2.0 / dt) * (1 - zz) / (1 + zz)
        out.append((2.0 / (1 + zz)) * (C @ np.linalg.solve(g * I - A, B)))
    return np.array(out)


def cauchy_woodbury(Lf, Pf, Qf, Bf, Cf, dt, z):
    """The pages' DPLR formula over all N modes ("The S4 kernel, from
    scratch", §4): with g = (2/dt)(1-z)/(1+z) and r_n = 1/(g - Lambda_n),
      k00 = sum C B r, k01 = sum C P r, k10 = sum conj(Q) B r, k11 = sum conj(Q) P r,
      K_hat = (2/(1+z)) (k00 - k01 k10 / (1 + k11)).
    Inputs are the full conjugate-closed vectors; z != -1."""
    z = np.atleast_1d(np.asarray(z, np.complex128))
    g = (2.0 / dt) * (1 - z) / (1 + z)
    r = 1.0 / (g[:, None] - np.asarray(Lf)[None, :])
    k00 = r @ (Cf * Bf)
    k01 = r @ (Cf * Pf)
    k10 = r @ (np.conj(Qf) * Bf)
    k11 = r @ (np.conj(Qf) * Pf)
    return (2.0 / (1 + z)) * (k00 - k01 * k10 / (1 + k11))


# ------------------------------------------------------------------ kernels --
def aliased_kernel_bruteforce(Ab, Bb, C, L, max_periods=100000, rel_tol=1e-17):
    """sum_{p>=0} Cbar Abar^(k+pL) Bbar for k < L by iterating v <- Abar v over
    whole periods until a period adds less than rel_tol * max|K| (§4
    "Aliasing"). Returns (K complex [L], periods used)."""
    Kr, Ki, per = _cloops.power_kernel(Ab[None], np.asarray(Bb)[None], np.asarray(C)[None],
                                       L, max_periods, rel_tol)
    return Kr[0] + 1j * Ki[0], int(per[0])


def aliased_kernel_closed(Ab, Bb, C, L):
    """The same infinite sum in closed form: K[k] = Cbar Abar^k (I - Abar^L)^-1 Bbar,
    then one period of dense powers (k = 0..L-1)."""
    N = Ab.shape[0]
    AL = np.linalg.matrix_power(Ab, L)
    w = np.linalg.solve(np.eye(N) - AL, Bb)
    Kr, Ki, _ = _cloops.power_kernel(Ab[None], w[None], np.asarray(C)[None], L, 1, 0.0)
    return Kr[0] + 1j * Ki[0]


def truncated_kernel(Ab, Bb, C, L):
    """K[k] = Cbar Abar^k Bbar, k < L (§4, the kernel before aliasing)."""
    Kr, Ki, _ = _cloops.power_kernel(Ab[None], np.asarray(Bb)[None], np.asarray(C)[None], L, 1, 0.0)
    return Kr[0] + 1j * Ki[0]


def s4d_kernel(a, B, C, dt, L):
    """S4D (diagonal, ZOH) kernel K[k] = 2 Re sum_n C_n Bbar_n Abar_n^k, k < L,
    by iterating the diagonal state v <- Abar v (the "S4" wiki page, section
    "S4D": the recurrence becomes elementwise). a, B, C: [H, Nh]; dt: [H]."""
    a = np.asarray(a, np.complex128); C = np.asarray(C, np.complex128)
    H, Nh = a.shape
    Ab = np.empty_like(a); Bb = np.empty_like(a)
    for h in range(H):
        Ab[h], Bb[h] = zoh_diag(a[h], B[h], float(dt[h]))
    v = Bb.copy()
    K = np.empty((H, L))
    for k in range(L):
        K[:, k] = 2.0 * np.real(np.sum(C * v, axis=1))
        v = Ab * v
    return K


# --------------------------------------------------------------- two views --
def causal_conv(u, K, D):
    """y[b,h,t] = sum_{s<=t} K[h,s] u[b,h,t-s] + D[h] u[b,h,t] (direct O(L^2);
    "The S4 kernel, from scratch", §1 and §5). u: [Bt,H,L] -> y [Bt,H,L]."""
    u = np.asarray(u, np.float64)
    Bt, H, L = u.shape
    row_h = np.tile(np.arange(H), Bt)
    y = _cloops.causal_conv(u.reshape(Bt * H, L), K, D, row_h)
    return y.reshape(Bt, H, L)


def causal_conv_adjoint(dy, K, D):
    """The adjoint of causal_conv in u, i.e. the gradient of
    <causal_conv(u, K, D), dy> with respect to u (the backward pass of §5's
    fft_conv): du[b,h,s] = sum_{t>=s} K[h,t-s] dy[b,h,t] + D[h] dy[b,h,s].
    Written as the causal sum of the time-reversed dy, reversed back."""
    dy = np.asarray(dy, np.float64)
    return np.ascontiguousarray(causal_conv(np.ascontiguousarray(dy[..., ::-1]), K, D)[..., ::-1])


def causal_conv_kernel_grad(u, dy):
    """The gradient of <causal_conv(u, K, D), dy> with respect to K and D:
    dK[h,k] = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k],  dD[h] = sum_b sum_t dy u."""
    u = np.asarray(u, np.float64)
    dy = np.asarray(dy, np.float64)
    Bt, H, L = u.shape
    dK = np.zeros((H, L))
    for b in range(Bt):
        for h in range(H):
            for k in range(L):
                dK[h, k] += np.dot(dy[b, h, k:], u[b, h, :L - k])
    dD = np.einsum("bht,bht->h", dy, u)
    return dK, dD


def causal_conv_rows_at(u_rows, row_h, K, D, ts):
    """The direct sum for selected rows (u_rows [R, L], channel row_h[r]) at
    selected output times ts only."""
    return _cloops.causal_conv_at(u_rows, K, D, row_h, ts)


def recurrence_dense(Ab, Bb, C, D, u_rows, row_h, x0=None):
    """x_t = Abar x_{t-1} + Bbar u_t, y_t = Re(C x_t) + D u_t, x_{-1} = x0 (0)
    ("The S4 kernel, from scratch", §5 recurrent view; §1 output map).
    Ab [H,N,N], Bb, C [H,N]; u_rows [R,T] -> (y [R,T], final state)."""
    return _cloops.recurrence_dense(Ab, Bb, C, D, row_h, u_rows, x0)


def recurrence_diag(Ab, Bb, C, D, u_rows, row_h, x0=None):
    """Diagonal recurrence over the stored half of a conjugate-closed system:
    x_t = Abar x_{t-1} + Bbar u_t, y_t = 2 Re(C x_t) + D u_t."""
    return _cloops.recurrence_diag(Ab, Bb, C, D, row_h, u_rows, x0)
