"""Pins of the dense zero-order hold (ZOH on the full DPLR matrix, "The S4
kernel, from scratch", §3) used for the ZOH DPLR variant."""
import numpy as np
import scipy.linalg

import s4inputs
from conftest import read_golden
from oracle import ssm, workloads


def test_scalar_is_the_printed_worked_example(golden_dir):
    """1x1: a = -1, dt = 1 gives the glossary page's Abar, k0 = Bbar and k1."""
    g = read_golden(f"{golden_dir}/zoh_scalar_worked_example.txt")
    Ab, Bb = ssm.zoh_dense(np.array([[-1.0]]), np.array([1.0]), 1.0)
    assert abs(Ab[0, 0] - g["Abar"]) < 1e-10
    assert abs(Bb[0] - g["k0"]) < 1e-10
    assert abs((Ab @ Bb)[0] - g["k1"]) < 1e-10


def test_diagonal_system_reduces_to_the_diagonal_rule():
    rng = np.random.default_rng(3)
    a = -rng.uniform(0.01, 3.0, 6) + 1j * rng.uniform(-40, 40, 6)
    a[0] = -1e-7 + 0j          # the Taylor branch of the diagonal rule
    B = rng.standard_normal(6) + 1j * rng.standard_normal(6)
    Ab, Bb = ssm.zoh_dense(np.diag(a), B, 0.05)
    Ad, Bd = ssm.zoh_diag(a, B, 0.05)
    assert np.abs(Ab - np.diag(Ad)).max() < 1e-14
    assert np.abs(Bb - Bd).max() < 1e-13


def test_step_response_identity_on_the_dplr_system():
    """A held unit input gives the continuous step response at the samples:
    sum_{j<=k} C Abar^j Bbar = C A^-1 (exp(A (k+1) dt) - I) B (solve, and expm
    at other times; a dropped dt or a wrong integral fails)."""
    inp = s4inputs.make_inputs(1, H=2, Bt=1, L=64)
    A, Bf, Cf, dt = workloads.dplr_channel_system(inp, 1)
    Ab, Bb = ssm.zoh_dense(A, Bf, dt)
    K = ssm.truncated_kernel(Ab, Bb, Cf, 64)
    S = np.cumsum(K)
    N = A.shape[0]
    for k in (0, 1, 7, 63):
        E = scipy.linalg.expm(A * (k + 1) * dt)
        ref = Cf @ np.linalg.solve(A, (E - np.eye(N)) @ Bf)
        assert abs(S[k] - ref) < 1e-9 * max(1.0, abs(ref)), k
    assert np.abs(K.imag).max() < 1e-10 * np.abs(K.real).max()


def test_two_holds_compose():
    """Holding over 2 dt = two holds over dt: Abar(2dt) = Abar(dt)^2 and
    Bbar(2dt) = Abar(dt) Bbar(dt) + Bbar(dt)."""
    inp = s4inputs.random_dplr(4, 1, 5, 64, 1)
    A, Bf, _, _ = workloads.dplr_channel_system(inp, 0)
    A1, B1 = ssm.zoh_dense(A, Bf, 0.03)
    A2, B2 = ssm.zoh_dense(A, Bf, 0.06)
    assert np.abs(A2 - A1 @ A1).max() < 1e-12 * np.abs(A2).max()
    assert np.abs(B2 - (A1 @ B1 + B1)).max() < 1e-12 * np.abs(B2).max()
