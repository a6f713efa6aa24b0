"""fp64 CPU oracle for the S4 DPLR / S4D hot path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import, call, link or run
anything in this package. The product library never does, and the two share
no code: the only module both sides read is ``s4inputs`` (seeded random draws
and stored parameter data, no arithmetic of the method).

Contents:
  hippo      HiPPO-LegS -> NPLR -> DPLR ("The S4 kernel, from scratch", §2)
  ssm        discretisation (bilinear; ZOH diagonal and dense), generating
             function, the pages' Cauchy/Woodbury
             formula, aliased kernel by dense powers, direct causal
             convolution, recurrence, S4D kernel (§1, §3-§5; "S4" wiki, S4D)
  block      the S4Block around the layer: channel layer norm, GLU-gated
             projection, residual (§6 "Trainable layer")
  workloads  drivers over the seeded workloads in ``s4inputs``
  loops.c    the O(L N^2) / O(L^2) fp64 loops, compiled with gcc

Every function is pinned by a CPU test against something other than itself
(values printed on the pages, closed forms, invariants, library routines,
brute force); see tests/test_oracle_*.py. Parity unpinned: none.
"""
from . import block, hippo, ssm, workloads  # noqa: F401
from ._cloops import build as build_loops  # noqa: F401
