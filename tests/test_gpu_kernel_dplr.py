"""GPU parity of s4_kernel_dplr (Cauchy/Woodbury + inverse FFT) against the
oracle's dense-power aliased kernel ("The S4 kernel, from scratch", §4)."""
import math

import numpy as np
import pytest

import s4inputs
from oracle import workloads
from gpu_helpers import K_TOL, kernel_err, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _gpu_kernel(inp, L=None, flags=None):
    import structured_state_space_dplr_b200 as s4
    t = to_dev(inp, ["Lambda", "P", "Q", "B", "C", "log_dt"])
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], L or inp["L"], flags=flags)
    torch_cuda().cuda.synchronize()
    return K.cpu().numpy()


def test_cfg1_all_channels():
    inp = s4inputs.make_inputs(1)
    torch = torch_cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    Kg = _gpu_kernel(inp, flags=flags)
    Kr = workloads.dplr_kernel(inp)
    assert int(flags.item()) == 0
    assert kernel_err(Kg, Kr) <= K_TOL


@pytest.mark.parametrize("cfg,channels", [(2, [0, 1, 97, 255]), (3, [0, 128, 255]), (4, [0, 31, 63])])
def test_full_size_sampled_channels(cfg, channels):
    """Full workload sizes (the launch the benchmark times), sampled channels."""
    inp = s4inputs.make_inputs(cfg, with_u=False)
    Kg = _gpu_kernel(inp)
    Kr = workloads.dplr_kernel(inp, channels=channels)
    assert kernel_err(Kg[channels], Kr) <= K_TOL


@pytest.mark.parametrize("L", [16, 32, 64, 128, 256, 512, 2048, 8192, 16384, 32768])
def test_random_dplr_lengths(L):
    """Random DPLR (P != Q, spread Re(Lambda)), odd H, every transform plan."""
    inp = s4inputs.random_dplr(L, H=3, Nh=8, L=L, Bt=1)
    Kg = _gpu_kernel(inp)
    Kr = workloads.dplr_kernel(inp)
    assert kernel_err(Kg, Kr) <= K_TOL


@pytest.mark.parametrize("Nh", [1, 5, 32, 64, 256])
def test_mode_counts(Nh):
    inp = s4inputs.random_dplr(100 + Nh, H=2, Nh=Nh, L=512, Bt=1, im_max=200.0)
    Kg = _gpu_kernel(inp)
    Kr = workloads.dplr_kernel(inp)
    assert kernel_err(Kg, Kr) <= K_TOL


def test_diagonal_case_no_lowrank():
    inp = s4inputs.random_dplr(7, H=4, Nh=16, L=1024, Bt=1, lowrank=0.0)
    assert kernel_err(_gpu_kernel(inp), workloads.dplr_kernel(inp)) <= K_TOL


@pytest.mark.parametrize("dt", [1e-4, 1e-3, 0.1, 1.0])
def test_step_size_extremes(dt):
    inp = s4inputs.make_inputs(1, H=2, L=4096, with_u=False)
    inp["log_dt"][:] = np.float32(math.log(dt))
    assert kernel_err(_gpu_kernel(inp), workloads.dplr_kernel(inp)) <= K_TOL


def test_unstable_mode_is_flagged_not_fatal():
    torch = torch_cuda()
    inp = s4inputs.random_dplr(11, H=2, Nh=4, L=64, Bt=1)
    inp["Lambda"][1, 2] = np.complex64(0.3 + 2.0j)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    Kg = _gpu_kernel(inp, flags=flags)
    assert int(flags.item()) & 1
    assert np.all(np.isfinite(Kg[0]))
