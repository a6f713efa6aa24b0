"""Write the stored data files that come from the oracle.

Calls only ``oracle/``. Run from the repository root:

    python -m oracle.write_fixtures

Writes ``s4inputs/hippo_legs_dplr_n64.txt``: the N=64 HiPPO-LegS DPLR modes
(Lambda, P, B for the 32 stored modes, fp64, from ``oracle.hippo``). The file
is stored because the eigenvector phases returned by LAPACK are a convention
of the library build; storing them makes the seeded inputs identical on every
machine.
"""
from __future__ import annotations

import os

from oracle import hippo

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def write_hippo_fixture(N: int = 64) -> str:
    lam, p, b, _ = hippo.make_dplr_hippo(N)
    path = os.path.join(_ROOT, "s4inputs", f"hippo_legs_dplr_n{N}.txt")
    with open(path, "w") as f:
        f.write(f"# HiPPO-LegS DPLR modes, N={N} (stored half, Im(Lambda) > 0, ascending),\n")
        f.write("# written by oracle/write_fixtures.py from oracle.hippo.make_dplr_hippo.\n")
        f.write("# columns: Re Lambda, Im Lambda, Re P, Im P, Re B, Im B   (Q = P)\n")
        for i in range(len(lam)):
            f.write(" ".join(repr(float(v)) for v in
                             (lam[i].real, lam[i].imag, p[i].real, p[i].imag, b[i].real, b[i].imag)))
            f.write("\n")
    return path


if __name__ == "__main__":
    print(write_hippo_fixture())
