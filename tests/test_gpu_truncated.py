"""GPU parity of the truncated-kernel reparameterisation Ctilde = C (I - Abar^L)
("The S4 kernel, from scratch", §4, "Aliasing"): with Ctilde in place of C the
generating-function kernel is the truncated kernel Cbar Abar^k Bbar (k < L),
and its convolution equals the recurrence from a zero state with no decay
assumption."""
import numpy as np
import pytest

import s4inputs
from oracle import ssm, workloads
from gpu_helpers import K_TOL, Y_TOL, kernel_err, rel_l2, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _inputs(kind, L):
    if kind == "hippo":   # HiPPO-LegS, H = 4, Nh = 32, dt up to 0.1
        return s4inputs.make_inputs(1, L=L)
    # random DPLR, slowly decaying modes (Re Lambda down to -0.02) so the
    # aliased and truncated kernels differ
    return s4inputs.random_dplr(11, H=3, Nh=24, L=L, Bt=2, re_min=-0.5, re_max=-0.02)


@pytest.mark.parametrize("kind,L", [("hippo", 1024), ("random", 256), ("random", 4096)])
def test_ctilde_matches_oracle_and_gives_truncated_kernel(kind, L):
    import structured_state_space_dplr_b200 as s4
    inp = _inputs(kind, L)
    t = to_dev(inp, ["Lambda", "P", "Q", "B", "C", "log_dt"])
    Ct = s4.dplr_ctilde(t["Lambda"], t["P"], t["Q"], t["C"], t["log_dt"], L)
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], Ct, t["log_dt"], L)
    torch_cuda().cuda.synchronize()
    Ctg, Kg = Ct.cpu().numpy().astype(np.complex128), K.cpu().numpy()
    Nh = Ctg.shape[1]
    Kref, alias_gap = [], []
    for h in range(inp["H"]):
        Ab, Bb, Cf = workloads.dplr_discretized(inp, h)
        Ctr = Cf @ (np.eye(Ab.shape[0]) - np.linalg.matrix_power(Ab, L))
        assert np.abs(Ctg[h] - Ctr[:Nh]).max() <= 1e-4 * np.abs(Ctr).max()
        Kt = ssm.truncated_kernel(Ab, Bb, Cf, L).real
        Ka = ssm.aliased_kernel_closed(Ab, Bb, Cf, L).real
        Kref.append(Kt)
        alias_gap.append(np.abs(Ka - Kt).max() / np.abs(Kt).max())
    Kref = np.stack(Kref)
    assert kernel_err(Kg, Kref) <= K_TOL
    if kind == "random":   # the case is one where truncation matters
        assert max(alias_gap) > 100 * K_TOL


def test_truncated_conv_equals_recurrence_without_decay():
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    L = 512
    inp = _inputs("random", L)
    t = to_dev(inp)
    Ct = s4.dplr_ctilde(t["Lambda"], t["P"], t["Q"], t["C"], t["log_dt"], L)
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], Ct, t["log_dt"], L)
    y = s4.fft_conv(t["u"], K, t["D"])
    Astr, Bb = s4.dplr_discretize_structured(t["Lambda"], t["P"], t["Q"], t["B"], t["log_dt"])
    x = torch.zeros(inp["Bt"], inp["H"], Astr.shape[1], dtype=torch.complex64, device="cuda")
    yr = s4.recurrent_scan(Astr, Bb, t["C"], t["D"], x, t["u"].contiguous())
    torch.cuda.synchronize()
    assert rel_l2(y.cpu().numpy(), yr.cpu().numpy()) <= Y_TOL
