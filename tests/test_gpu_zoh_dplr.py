"""GPU parity of the zero-order-hold DPLR variant ("The S4 kernel, from
scratch", §3, the ZOH rule on the full DPLR matrix): Abar = exp(dt A), Bbar,
and the truncated kernel Re(C_f Abar^k Bbar), against the fp64 oracle
(scipy's expm of the augmented matrix, dense powers)."""
import numpy as np
import pytest

import s4inputs
from oracle import ssm, workloads
from gpu_helpers import K_TOL, Y_TOL, kernel_err, rel_l2, to_dev, torch_cuda

pytestmark = pytest.mark.gpu

KEYS = ["Lambda", "P", "Q", "B", "C", "log_dt"]


def _inputs(kind, L):
    if kind == "hippo":          # HiPPO-LegS, H = 4, Nh = 32 (the full 64-state system)
        return s4inputs.make_inputs(1, L=L)
    if kind == "one":            # a single stored mode (N = 2)
        return s4inputs.random_dplr(23, H=2, Nh=1, L=L, Bt=1)
    if kind == "small":          # Nh = 5: the state is padded inside the kernel
        return s4inputs.random_dplr(21, H=3, Nh=5, L=L, Bt=2)
    return s4inputs.random_dplr(22, H=3, Nh=32, L=L, Bt=2, re_min=-0.5, re_max=-0.02)


@pytest.mark.parametrize("kind", ["hippo", "small", "random", "one"])
def test_discretize_zoh_matches_oracle(kind):
    import structured_state_space_dplr_b200 as s4
    inp = _inputs(kind, 64)
    t = to_dev(inp, KEYS)
    Ab, Bb, Cf = s4.dplr_discretize_zoh(*(t[k] for k in KEYS))
    torch_cuda().cuda.synchronize()
    Ab, Bb, Cf = (v.cpu().numpy().astype(np.complex128) for v in (Ab, Bb, Cf))
    for h in range(inp["H"]):
        Ar, Br, Cr = workloads.dplr_zoh_discretized(inp, h)
        assert np.abs(Ab[h] - Ar).max() <= 2e-6 * np.abs(Ar).max(), h
        assert np.abs(Bb[h] - Br).max() <= 2e-6 * np.abs(Br).max(), h
        assert np.abs(Cf[h] - Cr).max() <= 1e-7 * np.abs(Cr).max(), h


@pytest.mark.parametrize("kind,L", [("hippo", 1024), ("small", 16), ("small", 64), ("random", 256),
                                    ("random", 4096), ("one", 128)])
def test_kernel_zoh_matches_oracle(kind, L):
    """L = 16 (shorter than one 64-step block), whole blocks, long L with
    slowly decaying modes (many r <- r Abar^64 steps)."""
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    inp = _inputs(kind, L)
    t = to_dev(inp, KEYS)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    K = s4.kernel_dplr_zoh(*(t[k] for k in KEYS), L, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    Kref = workloads.dplr_zoh_kernel(inp)
    assert kernel_err(K.cpu().numpy(), Kref) <= K_TOL


def test_kernel_zoh_full_size_sampled_channels():
    """H = 256, L = 4096 (the long-sequence workload's shape), sampled channels."""
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    inp = s4inputs.make_inputs(2, with_u=False)
    t = to_dev(inp, KEYS)
    K = s4.kernel_dplr_zoh(*(t[k] for k in KEYS), inp["L"])
    torch.cuda.synchronize()
    ch = [0, 77, 255]
    Kref = workloads.dplr_zoh_kernel(inp, channels=ch)
    assert kernel_err(K.cpu().numpy()[ch], Kref) <= K_TOL


def test_zoh_convolution_equals_zoh_recurrence():
    """The ZOH kernel's convolution (s4_fft_conv) and the dense recurrence
    with the ZOH Abar (s4_recurrent_scan) agree, and both match the oracle's
    recurrence of its own ZOH system."""
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    L = 512
    inp = _inputs("random", L)
    t = to_dev(inp)
    K = s4.kernel_dplr_zoh(*(t[k] for k in KEYS), L)
    y = s4.fft_conv(t["u"], K, t["D"])
    Ab, Bb, Cf = s4.dplr_discretize_zoh(*(t[k] for k in KEYS))
    x = torch.zeros(inp["Bt"], inp["H"], Ab.shape[1], dtype=torch.complex64, device="cuda")
    yr = s4.recurrent_scan(Ab, Bb, Cf, t["D"], x, t["u"].contiguous())
    torch.cuda.synchronize()
    ys = []
    for h in range(inp["H"]):
        Ar, Br, Cr = workloads.dplr_zoh_discretized(inp, h)
        yh, _ = ssm.recurrence_dense(Ar[None], Br[None], Cr[None], np.array([float(inp["D"][h])]),
                                     inp["u"][:, h, :].astype(np.float64), np.zeros(inp["Bt"], np.int64))
        ys.append(yh)
    yref = np.stack(ys, axis=1)
    assert rel_l2(y.cpu().numpy(), yref) < Y_TOL
    assert rel_l2(yr.cpu().numpy(), yref) < Y_TOL


def test_kernel_zoh_flags_unstable_mode():
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    inp = _inputs("small", 64)
    inp["Lambda"] = inp["Lambda"].copy()
    inp["Lambda"][1, 2] = np.complex64(0.05 + 3j)     # Re(Lambda) > 0 in channel 1
    t = to_dev(inp, KEYS)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    s4.kernel_dplr_zoh(*(t[k] for k in KEYS), 64, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & 1
