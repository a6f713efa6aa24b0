"""GPU parity of the fused entry points: s4_kernel_dplr_prepare (K and the
convolution spectrum of K + D delta_0 in one launch for L <= 8192, two for
L = 16384) and
s4_forward_dplr (the whole convolution-view forward), against the fp64 oracle
and against the modular calls."""
import numpy as np
import pytest

import s4inputs
from oracle import workloads
from gpu_helpers import K_TOL, Y_TOL, kernel_err, rel_l2, sample_times, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _fused(inp):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    t = to_dev(inp)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = s4.forward_dplr(t["u"], t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"], flags=flags)
    K, ws = s4.kernel_dplr_prepare(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"], inp["L"])
    y2 = s4.fft_conv_apply(t["u"], ws)
    K3 = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], inp["L"])
    y3 = s4.fft_conv(t["u"], K3, t["D"])
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    assert torch.equal(y, y2)
    return K.cpu().numpy(), y.cpu().numpy(), K3.cpu().numpy(), y3.cpu().numpy()


@pytest.mark.parametrize("L", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768, 65536])
def test_random_dplr_all_outputs(L):
    """Every output, odd H and batch; L = 16384 takes the inverse transform
    fused into the spectrum kernel (one cluster per channel pair, K stored in
    place of the half spectra; with H = 3 the last cluster has one channel),
    longer L the separate inverse transform."""
    inp = s4inputs.random_dplr(500 + L, H=3, Nh=6, L=L, Bt=3)
    K, y, K3, y3 = _fused(inp)
    Kr = workloads.dplr_kernel(inp)
    yr = workloads.conv_full(inp, Kr)
    assert kernel_err(K, Kr) <= K_TOL
    assert rel_l2(y, yr) <= Y_TOL
    assert kernel_err(K, K3) <= K_TOL
    assert rel_l2(y, y3) <= Y_TOL


@pytest.mark.parametrize("L,H", [(16384, 1), (16384, 2), (16384, 5), (32768, 1), (32768, 4), (65536, 2)])
def test_channel_pairs_all_outputs(L, H):
    """Channel counts around the pairing of the generation kernels: at
    L = 16384 two channels are inverted and transformed at once and their
    spectra come apart by conjugate symmetry; at L >= 32768 the inverse
    transform packs channel pairs and the spectrum takes one channel per
    cluster. One channel alone, full pairs, and pairs plus a lone channel,
    each channel with its own D; every output of K and y against the
    oracle."""
    inp = s4inputs.random_dplr(900 + H + L, H=H, Nh=8, L=L, Bt=2)
    K, y, K3, y3 = _fused(inp)
    Kr = workloads.dplr_kernel(inp)
    yr = workloads.conv_full(inp, Kr)
    assert kernel_err(K, Kr) <= K_TOL
    assert rel_l2(y, yr) <= Y_TOL
    for h in range(H):
        assert rel_l2(y[:, h], yr[:, h]) <= 4 * Y_TOL
    assert kernel_err(K, K3) <= K_TOL
    assert rel_l2(y, y3) <= Y_TOL


def test_cfg1_all_outputs():
    inp = s4inputs.make_inputs(1)
    K, y, _, _ = _fused(inp)
    Kr = workloads.dplr_kernel(inp)
    assert kernel_err(K, Kr) <= K_TOL
    assert rel_l2(y, workloads.conv_full(inp, Kr)) <= Y_TOL


def test_cfg2_full_size_sampled():
    """The benchmark's workload and launch (H=256, L=4096, batch 16)."""
    inp = s4inputs.make_inputs(2)
    K, y, K3, y3 = _fused(inp)
    ch = [0, 128, 255]
    Kr = workloads.dplr_kernel(inp, channels=ch)
    assert kernel_err(K[ch], Kr) <= K_TOL
    assert kernel_err(K, K3) <= K_TOL
    ts = sample_times(inp["L"], 48, seed=22)
    rows = [(b, h) for h in ch for b in (0, 7, 15)]
    yr = workloads.conv_rows_at(inp, [Kr[ch.index(h)] for _, h in rows], rows, ts)
    ys = np.stack([y[b, h][ts] for b, h in rows])
    assert rel_l2(ys, yr) <= Y_TOL
    assert rel_l2(y, y3) <= Y_TOL
