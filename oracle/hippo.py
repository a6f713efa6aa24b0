"""HiPPO-LegS -> NPLR -> DPLR in fp64 (oracle; test infrastructure only).

Follows "The S4 kernel, from scratch", §2 "HiPPO initialization -> DPLR form":
A is HiPPO-LegS; it is normal plus low rank, A = A_normal - P P^T; the normal
part is diagonalised with a Hermitian eigendecomposition and everything is
rotated into that eigenbasis, giving A = Lambda - P Q^* with Q = P.

The pages name HiPPO-LegS but do not print it. The published HiPPO-LegS
definition is used (one reading, listed in the design notes):
  A[n, k] = -sqrt((2n+1)(2k+1))  for n > k,   -(n+1) for n = k,   0 for n < k,
  B[n]    =  sqrt(2n+1),
and the low-rank factor P[n] = sqrt(n + 1/2), the only rank-1 choice for which
A + P P^T has symmetric part -I/2 (hence is normal), as §2 requires.
"""
from __future__ import annotations

import numpy as np


def make_hippo(N: int):
    """HiPPO-LegS state matrix A [N, N] and input vector B [N] (real, fp64)."""
    n = np.arange(N, dtype=np.float64)
    r = np.sqrt(2.0 * n + 1.0)
    A = -np.tril(np.outer(r, r), -1) - np.diag(n + 1.0)
    B = r.copy()
    return A, B


def make_nplr_hippo(N: int):
    """A, rank-1 P and B with A = A_normal - P P^T, A_normal normal (§2)."""
    A, B = make_hippo(N)
    P = np.sqrt(np.arange(N, dtype=np.float64) + 0.5)
    return A, P, B


def make_dplr_hippo(N: int):
    """DPLR modes of HiPPO-LegS (§2): returns (Lambda, Pt, Bt, V).

    A_normal = A + P P^T = -I/2 + S with S real skew-symmetric. The Hermitian
    matrix -i S has real eigenvalues mu and eigenvectors V; A_normal V =
    V diag(-1/2 + i mu). The eigenvalues come in +-mu pairs whose eigenvectors
    are complex conjugates, so only the Nh = N/2 modes with mu > 0 are kept
    (ascending mu); their conjugates are implicit. Pt = V^* P, Bt = V^* B and
    Q = P (so Qt = Pt). V is [N, Nh].
    """
    if N % 2:
        raise ValueError("N must be even (conjugate pairs)")
    A, P, B = make_nplr_hippo(N)
    S = A + np.outer(P, P) + 0.5 * np.eye(N)
    mu, V = np.linalg.eigh(-1j * S)
    order = np.argsort(mu)
    mu, V = mu[order], V[:, order]
    keep = mu > 0
    if keep.sum() != N // 2:
        raise RuntimeError("eigenvalues of the skew part are not in +-pairs")
    mu, V = mu[keep], V[:, keep]
    Lambda = -0.5 + 1j * mu
    Pt = V.conj().T @ P
    Bt = V.conj().T @ B
    return Lambda, Pt, Bt, V
