"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test names what fixes the value: numbers printed on the pages, a closed
form, an invariant, a library routine, or brute force.
"""
import math
import os

import numpy as np
import pytest
from numpy.polynomial import legendre as npleg

import s4inputs
from oracle import hippo, ssm, workloads
from conftest import read_golden


# ----------------------------------------------------------- discretisation --
def test_zoh_worked_example_printed_values(golden_dir):
    """Glossary page "Structured state-space sequence model and S4", section
    "Follow one input through memory": a=-1, dt=1, B=C=1 (values printed to
    10 decimals). The conjugate-closed S4D kernel doubles a stored mode, so a
    real scalar mode is represented with C = 1/2."""
    g = read_golden(os.path.join(golden_dir, "zoh_scalar_worked_example.txt"))
    Ab, Bb = ssm.zoh_diag(np.array([-1.0 + 0j]), np.array([1.0 + 0j]), 1.0)
    assert abs(Ab[0] - g["Abar"]) < 1e-10 and abs(Ab[0].imag) == 0
    assert abs(Bb[0] - g["Bbar"]) < 1e-10
    K = ssm.s4d_kernel(np.array([[-1.0 + 0j]]), np.array([[1.0 + 0j]]), np.array([[0.5 + 0j]]),
                       np.array([1.0]), 2)
    assert abs(K[0, 0] - g["k0"]) < 1e-10 and abs(K[0, 1] - g["k1"]) < 1e-10
    u = np.array([[[1.0, 0.0]]])
    y = ssm.causal_conv(u, K, np.array([0.0]))
    assert abs(y[0, 0, 0] - g["y1"]) < 1e-10 and abs(y[0, 0, 1] - g["y2"]) < 1e-10
    yr, _ = ssm.recurrence_diag(Ab[None], Bb[None], np.array([[0.5 + 0j]]), np.array([0.0]),
                                u[0], np.array([0]))
    assert abs(yr[0, 0] - g["y1"]) < 1e-10 and abs(yr[0, 1] - g["y2"]) < 1e-10


def test_zoh_taylor_branch_matches_expm1():
    """The series branch (|dt a| < 1e-4) against numpy's expm1 (library)."""
    for a in (1e-7 + 2e-7j, -3e-6 + 0j, 2e-5 - 1e-5j, 0.0 + 0j):
        Ab, Bb = ssm.zoh_diag(np.array([a]), np.array([1.0 + 0j]), 0.5)
        x = 0.5 * a
        ref = 0.5 if a == 0 else np.expm1(x) / a
        assert abs(Bb[0] - ref) <= 1e-15 * abs(ref)
    # just above the threshold the direct form (exp(x) - 1)/a loses about
    # eps/|x| = 1e-12 relative to cancellation; that bound is what is checked
    for x in (1.0001e-4, 3e-4, 0.1):
        a = x / 0.5
        _, b1 = ssm.zoh_diag(np.array([a + 0j]), np.array([1 + 0j]), 0.5)
        ref = np.expm1(x) / a
        assert abs(b1[0] - ref) < 4e-16 / x * abs(ref)


def test_bilinear_scalar_closed_form():
    """a=-1, dt=1: Abar=(1-1/2)/(1+1/2)=1/3, Bbar=dt/(1+1/2)=2/3 by hand, so
    the kernel is (2/3)(1/3)^k ("The S4 kernel, from scratch", §3)."""
    Ab, Bb = ssm.bilinear(np.array([[-1.0]]), np.array([1.0]), 1.0)
    assert abs(Ab[0, 0] - 1 / 3) < 1e-15 and abs(Bb[0] - 2 / 3) < 1e-15
    K = ssm.truncated_kernel(Ab, Bb, np.array([1.0 + 0j]), 4)
    assert np.allclose(K.real, [2 / 3, 2 / 9, 2 / 27, 2 / 81], atol=1e-15, rtol=0)


# ------------------------------------------------------------------- HiPPO --
def _legs_coeffs(d, N):
    """kappa_n = int_0^1 s^d sqrt(2n+1) P_n(2s-1) ds (Gauss-Legendre, exact)."""
    x, w = npleg.leggauss(16)
    s = (x + 1) / 2
    out = np.zeros(N)
    for n in range(N):
        c = np.zeros(n + 1); c[n] = 1
        out[n] = 0.5 * np.sum(w * s ** d * math.sqrt(2 * n + 1) * npleg.legval(2 * s - 1, c))
    return out


@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_hippo_legs_memorizes_polynomials(d):
    """HiPPO-LegS keeps the exact Legendre coefficients of the history
    ("The S4 kernel, from scratch", §2: memorizes history through orthogonal
    polynomial projections). For u(s) = s^d on [0, t] the coefficients are
    c(t) = t^d kappa, and the LegS ODE c' = (A c + B u)/t at t = 1 must give
    d kappa = A kappa + B. Coefficients from numpy's Legendre routines."""
    N = 10
    A, B = hippo.make_hippo(N)
    kappa = _legs_coeffs(d, N)
    assert np.allclose(A @ kappa + B, d * kappa, atol=1e-12)


def test_nplr_symmetric_part():
    """§2: A = A_normal - P P^T with A_normal normal; here sym(A + P P^T) = -I/2."""
    A, P, _ = hippo.make_nplr_hippo(64)
    An = A + np.outer(P, P)
    assert np.abs((An + An.T) / 2 + 0.5 * np.eye(64)).max() < 1e-12
    assert np.abs(An @ An.T - An.T @ An).max() < 1e-9   # normal


@pytest.mark.parametrize("N", [4, 8, 64])
def test_dplr_reconstructs_hippo(N):
    """§2: in the eigenbasis V, A = V (Lambda - P Q^*) V^* with Q = P; the
    conjugate half is implicit, so V_f = [V, conj V] must be unitary."""
    A, P, B = hippo.make_nplr_hippo(N)
    lam, pt, bt, V = hippo.make_dplr_hippo(N)
    assert np.all(np.abs(lam.real + 0.5) < 1e-12) and np.all(lam.imag > 0)
    Vf = np.concatenate([V, V.conj()], 1)
    assert np.abs(Vf.conj().T @ Vf - np.eye(N)).max() < 1e-12
    Af, Bf, _ = ssm.full_system(lam, pt, pt, bt, np.zeros_like(bt))
    assert np.abs(Vf @ Af @ Vf.conj().T - A).max() < 1e-11 * N
    assert np.abs(Vf @ Bf - B).max() < 1e-12 * N


@pytest.mark.parametrize("N", [4, 6, 8])
def test_dplr_spectrum_is_hippo_spectrum(N):
    """A is lower triangular with diagonal -(n+1), so its eigenvalues are
    -1..-N; the DPLR matrix must have the same spectrum (small N, where the
    non-normal eigenproblem is still well conditioned)."""
    lam, pt, _, _ = hippo.make_dplr_hippo(N)
    Af, _, _ = ssm.full_system(lam, pt, pt, pt, pt)
    ev = np.sort(np.linalg.eigvals(Af).real)
    assert np.allclose(ev, -np.arange(N, 0, -1), atol=1e-6)


def test_stored_fixture_matches_oracle():
    """The stored N=64 modes equal the oracle's (phase-invariant quantities)."""
    lam, p, b = s4inputs.load_hippo_dplr(64)
    lam2, p2, b2, _ = hippo.make_dplr_hippo(64)
    assert np.abs(lam - lam2).max() < 1e-12
    assert np.abs(np.abs(p) - np.abs(p2)).max() < 1e-12
    assert np.abs(p * b.conj() - p2 * b2.conj()).max() < 1e-12


# ------------------------------------------------------------------ kernel --
@pytest.fixture(scope="module")
def cfg1():
    return s4inputs.make_inputs(1)


def test_aliased_kernel_bruteforce_equals_closed_form(cfg1):
    """§4 "Aliasing": the period sum by brute force equals the closed form
    Cbar Abar^k (I - Abar^L)^-1 Bbar."""
    Kc = workloads.dplr_kernel(cfg1, method="closed")
    Kb = workloads.dplr_kernel(cfg1, method="brute")
    for h in range(cfg1["H"]):
        assert np.abs(Kc[h] - Kb[h]).max() <= 1e-12 * np.abs(Kb[h]).max()


def test_kernel_dft_equals_generating_function(cfg1):
    """§4: the DFT of the aliased K at the L-th roots of unity equals the
    generating function (2/(1+z)) C (g I - A)^-1 B, by dense solves (numpy FFT
    and LAPACK; no Cauchy, no Woodbury)."""
    K = workloads.dplr_kernel(cfg1, channels=[0, 3])
    L = cfg1["L"]
    z = ssm.roots_of_unity(L)
    j = np.r_[0:40, L // 2 - 7:L // 2, L // 2 + 1:L // 2 + 9, L - 30:L]
    for i, h in enumerate([0, 3]):
        A, Bf, Cf, dt = workloads.dplr_channel_system(cfg1, h)
        ref = ssm.generating_function_continuous(A, Bf, Cf, dt, z[j])
        got = np.fft.fft(K[i])[j]
        assert np.abs(got - ref).max() <= 1e-11 * np.abs(ref).max()


def test_pages_cauchy_woodbury_equals_resolvent(cfg1):
    """§4: the four Cauchy sums with the rank-1 Woodbury correction equal the
    dense resolvent form (pins the reading conj(Q) in k10, k11)."""
    L = cfg1["L"]
    z = ssm.roots_of_unity(L)[1:L // 2]
    for h in range(cfg1["H"]):
        A, Bf, Cf, dt = workloads.dplr_channel_system(cfg1, h)
        cat = lambda x: np.concatenate([x, x.conj()]).astype(np.complex128)
        cw = ssm.cauchy_woodbury(cat(cfg1["Lambda"][h]), cat(cfg1["P"][h]), cat(cfg1["Q"][h]),
                                 Bf, Cf, dt, z)
        ref = ssm.generating_function_continuous(A, Bf, Cf, dt, z)
        assert np.abs(cw - ref).max() <= 1e-11 * np.abs(ref).max()


def test_discrete_generating_function_equals_continuous_form(cfg1):
    """Pins Bbar = (I - dt/2 A)^-1 dt B and Cbar = C: the discrete generating
    function Cbar (I - z Abar)^-1 Bbar equals §4's continuous-form expression."""
    A, Bf, Cf, dt = workloads.dplr_channel_system(cfg1, 1)
    Ab, Bb = ssm.bilinear(A, Bf, dt)
    z = np.exp(-2j * np.pi * np.array([0.01, 0.1, 0.3, 0.49]))
    a = ssm.generating_function_discrete(Ab, Bb, Cf, z)
    b = ssm.generating_function_continuous(A, Bf, Cf, dt, z)
    assert np.abs(a - b).max() < 1e-12 * np.abs(b).max()


def test_dc_gain_and_nyquist_closed_forms(cfg1):
    """sum_k K[k] = -C A^-1 B (bilinear keeps the DC gain, z = 1) and
    sum_k (-1)^k K[k] = dt Re sum_n C_n B_n (limit of §4's formula at z = -1,
    where the Woodbury term vanishes)."""
    K = workloads.dplr_kernel(cfg1)
    L = cfg1["L"]
    for h in range(cfg1["H"]):
        A, Bf, Cf, dt = workloads.dplr_channel_system(cfg1, h)
        dc = -(Cf @ np.linalg.solve(A, Bf))
        assert abs(K[h].sum() - dc.real) < 1e-12 * np.abs(K[h]).sum()
        nyq = dt * np.real(np.sum(cfg1["C"][h].astype(np.complex128) * cfg1["B"][h].astype(np.complex128)))
        alt = np.sum(K[h] * (-1.0) ** np.arange(L))
        assert abs(alt - nyq) < 1e-12 * np.abs(K[h]).sum()


def test_diagonal_case_closed_form():
    """P = Q = 0: each mode is a scalar bilinear system, so
    K[k] = 2 Re sum_n C_n Bbar_n Abar_n^k / (1 - Abar_n^L) (geometric series)."""
    inp = s4inputs.random_dplr(3, H=2, Nh=5, L=64, Bt=1, lowrank=0.0)
    K = workloads.dplr_kernel(inp)
    k = np.arange(64)
    for h in range(2):
        dt = math.exp(float(inp["log_dt"][h]))
        lam = inp["Lambda"][h].astype(np.complex128)
        ab = (1 + dt * lam / 2) / (1 - dt * lam / 2)
        bb = dt / (1 - dt * lam / 2) * inp["B"][h].astype(np.complex128)
        c = inp["C"][h].astype(np.complex128)
        ref = 2 * np.real(np.sum((c * bb / (1 - ab ** 64))[:, None] * ab[:, None] ** k[None], 0))
        assert np.abs(K[h] - ref).max() < 1e-12 * np.abs(ref).max()


def test_bilinear_stability(cfg1):
    """Re(Lambda) < 0 with Q = P keeps the spectral radius of Abar below 1
    (eigenvalues inside the unit circle, the "S4" page on infraphysics)."""
    for h in range(cfg1["H"]):
        Ab, _, _ = workloads.dplr_discretized(cfg1, h)
        assert np.max(np.abs(np.linalg.eigvals(Ab))) < 1.0


# --------------------------------------------------------------- two views --
def test_direct_conv_matches_numpy_convolve():
    rng = np.random.default_rng(5)
    u = rng.standard_normal((2, 3, 50)); K = rng.standard_normal((3, 50)); D = rng.standard_normal(3)
    y = ssm.causal_conv(u, K, D)
    for b in range(2):
        for h in range(3):
            ref = np.convolve(K[h], u[b, h])[:50] + D[h] * u[b, h]
            assert np.abs(y[b, h] - ref).max() < 1e-12
    ts = np.array([0, 7, 49])
    ya = ssm.causal_conv_rows_at(u[1], np.arange(3), K, D, ts)
    assert np.abs(ya - y[1][:, ts]).max() < 1e-13


def test_impulse_response_is_kernel_plus_feedthrough():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((2, 32)); D = np.array([0.7, -1.3])
    u = np.zeros((1, 2, 32)); u[:, :, 0] = 1
    y = ssm.causal_conv(u, K, D)
    assert np.abs(y[0] - (K + D[:, None] * (np.arange(32) == 0))).max() < 1e-15


def test_recurrence_equals_convolution_truncated(cfg1):
    """§5 / glossary "One linear layer, two computational views": the
    recurrence and the convolution with the truncated kernel agree."""
    h = 2
    Ab, Bb, Cf = workloads.dplr_discretized(cfg1, h)
    L = 256
    Kt = ssm.truncated_kernel(Ab, Bb, Cf, L).real
    u = cfg1["u"][:, h, :L].astype(np.float64)
    yr, _ = ssm.recurrence_dense(Ab[None], Bb[None], Cf[None], np.array([float(cfg1["D"][h])]),
                                 u, np.zeros(u.shape[0], np.int64))
    yc = ssm.causal_conv(u[:, None, :], Kt[None], np.array([float(cfg1["D"][h])]))[:, 0]
    assert np.abs(yr - yc).max() < 1e-12 * np.abs(yc).max()


def test_recurrence_matches_aliased_conv_once_decayed():
    """§4 "Aliasing": once the kernel has decayed within L, the aliased
    kernel's convolution matches the exact recurrence (~1e-7 on the page)."""
    inp = s4inputs.make_inputs(1, H=2, L=1024)
    inp["log_dt"][:] = np.float32(math.log(0.06))  # dt L / 2 > 30: decayed
    K = workloads.dplr_kernel(inp)
    y = ssm.causal_conv(inp["u"], K, inp["D"].astype(np.float64))
    for h in range(2):
        Ab, Bb, Cf = workloads.dplr_discretized(inp, h)
        yr, _ = ssm.recurrence_dense(Ab[None], Bb[None], Cf[None], np.array([float(inp["D"][h])]),
                                     inp["u"][:, h].astype(np.float64), np.zeros(inp["Bt"], np.int64))
        assert np.abs(yr - y[:, h]).max() < 1e-7 * np.abs(y[:, h]).max()


def test_s4d_kernel_closed_form_and_recurrence():
    """S4D ("S4" wiki, section "S4D"): iterated kernel equals the closed form
    2 Re sum_n C Bbar exp(k dt a_n) (numpy exp), and the elementwise
    recurrence equals the convolution with it."""
    inp = s4inputs.make_inputs(5, H=3, L=512, Bt=2)
    K = workloads.s4d_kernel(inp)
    Ab, Bb = workloads.s4d_params(inp)
    k = np.arange(512)
    for h in range(3):
        dt = math.exp(float(inp["log_dt"][h]))
        a = inp["A"][h].astype(np.complex128)
        ref = 2 * np.real(np.sum((inp["C"][h].astype(np.complex128) * Bb[h])[:, None]
                                 * np.exp(dt * np.outer(a, k)), 0))
        assert np.abs(K[h] - ref).max() < 1e-12 * np.abs(ref).max()
    y = ssm.causal_conv(inp["u"], K, inp["D"].astype(np.float64))
    rows = [(b, h) for b in range(2) for h in range(3)]
    u = np.stack([inp["u"][b, h] for b, h in rows]).astype(np.float64)
    hh = np.array([h for _, h in rows])
    yr, _ = ssm.recurrence_diag(Ab, Bb, inp["C"].astype(np.complex128), inp["D"].astype(np.float64), u, hh)
    for i, (b, h) in enumerate(rows):
        assert np.abs(yr[i] - y[b, h]).max() < 1e-11 * np.abs(y[b, h]).max()


def test_conv_adjoint_identity_and_kernel_grad_by_basis():
    """<conv(u), dy> = <u, adjoint(dy)>, and since the convolution is linear
    in K and D, its derivative along a basis kernel e_{h,k} (or D = e_h) is
    exactly the inner product with that basis output."""
    rng = np.random.default_rng(5)
    Bt, H, L = 3, 2, 40
    u = rng.standard_normal((Bt, H, L))
    dy = rng.standard_normal((Bt, H, L))
    K = rng.standard_normal((H, L))
    D = rng.standard_normal(H)
    y = ssm.causal_conv(u, K, D)
    du = ssm.causal_conv_adjoint(dy, K, D)
    assert abs(np.sum(y * dy) - np.sum(u * du)) <= 1e-12 * np.sum(np.abs(y * dy))
    dK, dD = ssm.causal_conv_kernel_grad(u, dy)
    zero = np.zeros(H)
    for h, k in [(0, 0), (1, 7), (0, L - 1), (1, 23)]:
        E = np.zeros((H, L))
        E[h, k] = 1.0
        assert abs(np.sum(ssm.causal_conv(u, E, zero) * dy) - dK[h, k]) <= 1e-12 * (1 + abs(dK[h, k]))
    for h in range(H):
        e = np.zeros(H)
        e[h] = 1.0
        assert abs(np.sum(ssm.causal_conv(u, np.zeros((H, L)), e) * dy) - dD[h]) <= 1e-12 * (1 + abs(dD[h]))
    # the adjoint is the transpose: du of a unit impulse dy picks one kernel row
    d1 = np.zeros((1, 1, L))
    d1[0, 0, 30] = 1.0
    du1 = ssm.causal_conv_adjoint(d1, K[:1], D[:1])[0, 0]
    assert np.allclose(du1[:31], K[0, 30::-1] + np.where(np.arange(31) == 30, D[0], 0.0), rtol=0, atol=1e-14)
    assert np.all(du1[31:] == 0.0)


def test_fd_gradient_matches_s4d_closed_form_derivative():
    """The finite-difference helper behind the kernel-parameter gradients,
    on the S4D kernel K[k] = 2 Re sum_n C_n Bbar_n Abar_n^k, whose derivative
    in C is closed form: d<K, G>/dRe C_n + i d<K, G>/dIm C_n
    = 2 sum_k G[k] conj(Bbar_n Abar_n^k)."""
    rng = np.random.default_rng(8)
    Nh, L = 3, 24
    a = -0.3 - rng.uniform(0, 0.5, Nh) + 1j * np.pi * np.arange(Nh)
    B = np.ones(Nh, complex)
    C = rng.standard_normal(Nh) + 1j * rng.standard_normal(Nh)
    dt = 0.07
    G = rng.standard_normal(L)

    def fun(p):
        return float(np.dot(ssm.s4d_kernel(a[None], B[None], p["C"][None], np.array([dt]), L)[0], G))

    g = workloads.fd_gradient(fun, {"C": C}, ["C"])["C"]
    Ab, Bb = ssm.zoh_diag(a, B, dt)
    ref = 2.0 * np.array([np.sum(G * np.conj(Bb[n] * Ab[n] ** np.arange(L))) for n in range(Nh)])
    assert np.abs(g - ref).max() <= 1e-7 * np.abs(ref).max()
    # a real parameter, log(dt): with Bbar Abar^k = (e^{dt a} - 1)/a B e^{k dt a},
    # d/d log(dt) = dt B (e^{(k+1) dt a} + k (e^{dt a} - 1) e^{k dt a})
    def fun_dt(p):
        return float(np.dot(ssm.s4d_kernel(a[None], B[None], C[None], np.exp(p["ld"]), L)[0], G))
    g1 = workloads.fd_gradient(fun_dt, {"ld": np.array([np.log(dt)])}, ["ld"])["ld"][0]
    k = np.arange(L)
    dK = sum(2.0 * np.real(C[n] * dt * B[n] * (np.exp((k + 1) * dt * a[n])
                                              + k * (np.exp(dt * a[n]) - 1.0) * np.exp(k * dt * a[n])))
             for n in range(Nh))
    ref_dt = float(np.dot(dK, G))
    assert abs(g1 - ref_dt) <= 1e-7 * abs(ref_dt)


def test_s4d_gradient_closed_forms_match_finite_differences():
    """The closed forms of the S4D kernel's gradient (with V_n = sum_k G[k]
    Abar_n^k, W_n = sum_k k G[k] Abar_n^k, r_n = (e^{dt a_n} - 1)/a_n:
    dC = 2 conj(Bbar V), dB = 2 conj(C r V), dA = 2 conj(C B dt^2 phi1'(dt a) V
    + C Bbar dt W), dlog_dt = 2 dt Re sum (C B Abar V + C Bbar a W)) against
    central differences of the oracle's Vandermonde sum; one mode sits in the
    small-|dt a| range where phi1' is taken from its series."""
    rng = np.random.default_rng(12)
    Nh, L, dt = 4, 40, 0.05
    a = -rng.uniform(0.05, 1.0, Nh) + 1j * rng.uniform(-20, 20, Nh)
    a[1] = -2e-3 + 1e-3j          # |dt a| = 1.1e-4: the series branch of phi1'
    B = rng.standard_normal(Nh) + 1j * rng.standard_normal(Nh)
    C = rng.standard_normal(Nh) + 1j * rng.standard_normal(Nh)
    G = rng.standard_normal(L)
    inp = dict(H=1, L=L, A=a[None].astype(np.complex64), B=B[None].astype(np.complex64),
               C=C[None].astype(np.complex64), log_dt=np.array([np.log(dt)], np.float32))
    ref = workloads.s4d_kernel_param_grad(inp, G[None])
    a, B, C = (inp[k][0].astype(np.complex128) for k in ("A", "B", "C"))
    dt = float(np.exp(np.float64(inp["log_dt"][0])))
    Ab, Bb = ssm.zoh_diag(a, B, dt)
    k = np.arange(L)
    V = np.array([np.sum(G * Ab[n] ** k) for n in range(Nh)])
    W = np.array([np.sum(k * G * Ab[n] ** k) for n in range(Nh)])
    r = Bb / B
    x = dt * a
    phi1p = np.where(np.abs(x) < 1e-3, 0.5 + x / 3 + x ** 2 / 8 + x ** 3 / 30 + x ** 4 / 144,
                     (x * np.exp(x) - (np.exp(x) - 1)) / np.where(x == 0, 1, x) ** 2)
    dC = 2 * np.conj(Bb * V)
    dB = 2 * np.conj(C * r * V)
    dA = 2 * np.conj(C * B * dt ** 2 * phi1p * V + C * Bb * dt * W)
    dld = 2 * dt * np.real(np.sum(C * B * Ab * V + C * Bb * a * W))
    for name, mine in (("C", dC), ("B", dB), ("A", dA)):
        assert np.abs(mine - ref[name][0]).max() <= 1e-6 * np.abs(ref[name][0]).max(), name
    assert abs(dld - ref["log_dt"][0]) <= 1e-6 * abs(ref["log_dt"][0])


def test_dplr_gradient_closed_forms_match_finite_differences():
    """The closed forms of the gradient through the DPLR kernel (the
    generating function of "The S4 kernel, from scratch" §4 differentiated:
    g_j = (2/L) DFT(dK)_j, the Woodbury partials e_v, a_v = conj(g_j) e_v,
    per stored mode S_v = sum_j a_v r' + conj(a_v r), S2_v likewise with the
    squares, the Nyquist closed form) against central differences of the
    oracle's dense aliased kernel."""
    inp = s4inputs.random_dplr(31, H=1, Nh=3, L=32, Bt=1)
    L = inp["L"]
    dK = np.random.default_rng(2).standard_normal(L)
    ref = workloads.dplr_kernel_param_grad(inp, dK[None])
    lam, P, Q, B, C = (inp[k][0].astype(np.complex128) for k in ("Lambda", "P", "Q", "B", "C"))
    dt = float(np.exp(np.float64(inp["log_dt"][0])))
    full = lambda x: np.concatenate([x, np.conj(x)])
    lf = full(lam)
    vs = [C * B, C * P, np.conj(Q) * B, np.conj(Q) * P]    # v00, v01, v10, v11 of the stored modes
    vf = [full(v) for v in vs]
    G = np.fft.fft(dK)
    S = [np.zeros(3, complex) for _ in range(4)]
    S2 = [np.zeros(3, complex) for _ in range(4)]
    dld = 0.0
    for j in range(L // 2):
        g = (1.0 if j == 0 else 2.0) / L * G[j]
        t = np.tan(np.pi * j / L)
        s = 1j * 2.0 * t / dt
        c = 1.0 + 1j * t
        ri = 1.0 / (s - lf)
        k = [np.sum(v * ri) for v in vf]
        den = 1.0 + k[3]
        e = [c, -c * k[2] / den, -c * k[1] / den, c * k[1] * k[2] / den ** 2]
        rn, rc = 1.0 / (s - lam), 1.0 / (s - np.conj(lam))
        for v in range(4):
            a = np.conj(g) * e[v]
            S[v] += a * rc + np.conj(a * rn)
            S2[v] += a * rc ** 2 + np.conj(a * rn ** 2)
        dld += np.real(np.conj(g) * s * sum(e[v] * np.sum(vf[v] * ri ** 2) for v in range(4)))
    gN = np.real(G[L // 2]) / L
    dC = np.conj(B) * S[0] + np.conj(P) * S[1] + gN * dt * np.conj(B)
    dB = np.conj(C) * S[0] + Q * S[2] + gN * dt * np.conj(C)
    dP = np.conj(C) * S[1] + Q * S[3]
    dQ = B * np.conj(S[2]) + P * np.conj(S[3])
    dL = sum(np.conj(vs[v]) * S2[v] for v in range(4))
    dld += gN * dt * np.real(np.sum(C * B))
    for name, mine in (("C", dC), ("B", dB), ("P", dP), ("Q", dQ), ("Lambda", dL)):
        assert np.abs(mine - ref[name][0]).max() <= 1e-6 * np.abs(ref[name][0]).max(), name
    assert abs(dld - ref["log_dt"][0]) <= 1e-6 * abs(ref["log_dt"][0])
