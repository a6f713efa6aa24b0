"""GPU parity of the S4D Vandermonde kernel, the discretisations and the
recurrent step ("S4" wiki page, section "S4D"; "The S4 kernel, from
scratch", §3 and §5)."""
import math

import numpy as np
import pytest

import s4inputs
from oracle import ssm, workloads
from gpu_helpers import K_TOL, Y_TOL, kernel_err, rel_l2, sample_times, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _vdm(inp, flags=None):
    import structured_state_space_dplr_b200 as s4
    t = to_dev(inp, ["A", "B", "C", "log_dt"])
    K = s4.s4d_kernel_vandermonde(t["A"], t["B"], t["C"], t["log_dt"], inp["L"], flags=flags)
    torch_cuda().cuda.synchronize()
    return K.cpu().numpy()


@pytest.mark.parametrize("L", [16, 64, 1024, 8192])
def test_vandermonde_small(L):
    inp = s4inputs.make_inputs(5, H=6, L=L, with_u=False)
    assert kernel_err(_vdm(inp), workloads.s4d_kernel(inp)) <= K_TOL


def test_vandermonde_long_and_many_modes():
    inp = s4inputs.make_inputs(5, H=2, L=65536, with_u=False)
    assert kernel_err(_vdm(inp), workloads.s4d_kernel(inp)) <= K_TOL
    rng = np.random.default_rng(4)
    inp = s4inputs.make_inputs(5, H=2, L=256, with_u=False)
    Nh = 100
    inp["A"] = (-rng.uniform(0.01, 1, (2, Nh)) + 1j * rng.uniform(0, 300, (2, Nh))).astype(np.complex64)
    inp["B"] = np.ones((2, Nh), np.complex64)
    inp["C"] = (rng.standard_normal((2, Nh)) + 1j * rng.standard_normal((2, Nh))).astype(np.complex64)
    assert kernel_err(_vdm(inp), workloads.s4d_kernel(inp)) <= K_TOL


@pytest.mark.parametrize("Nh", [4, 33, 100])
def test_vandermonde_tensor_core_mode_chunks(Nh):
    """L = 8192 takes the tensor-core product, 32 modes per chunk: partial and
    several chunks accumulate in tensor memory; no wait runs out."""
    torch = torch_cuda()
    rng = np.random.default_rng(Nh)
    inp = s4inputs.make_inputs(5, H=3, L=8192, with_u=False)
    inp["A"] = (-rng.uniform(0.01, 1, (3, Nh)) + 1j * rng.uniform(0, 300, (3, Nh))).astype(np.complex64)
    inp["B"] = np.ones((3, Nh), np.complex64)
    inp["C"] = (rng.standard_normal((3, Nh)) + 1j * rng.standard_normal((3, Nh))).astype(np.complex64)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    Kg = _vdm(inp, flags=flags)
    assert int(flags.item()) == 0
    assert kernel_err(Kg, workloads.s4d_kernel(inp)) <= K_TOL


def test_vandermonde_cfg5_full_size_sampled():
    inp = s4inputs.make_inputs(5, with_u=False)
    Kg = _vdm(inp)
    ch = [0, 511, 1023]
    assert kernel_err(Kg[ch], workloads.s4d_kernel(inp, channels=ch)) <= K_TOL


def test_s4d_zoh_discretize():
    import structured_state_space_dplr_b200 as s4
    inp = s4inputs.make_inputs(5, H=8, L=16, with_u=False)
    inp["A"][0, 0] = np.complex64(1e-7 + 0j)      # series branch
    t = to_dev(inp, ["A", "B", "log_dt"])
    Ab, Bb = s4.s4d_discretize_zoh(t["A"], t["B"], t["log_dt"])
    Abr, Bbr = workloads.s4d_params(inp)
    assert np.abs(Ab.cpu().numpy() - Abr).max() <= 1e-6
    assert np.abs(Bb.cpu().numpy() - Bbr).max() <= 1e-6 * np.abs(Bbr).max()


def test_s4d_decode_1024_steps_matches_convolution():
    """cfg 5: 1024 single-token steps from a zero state reproduce the first
    1024 outputs of the Vandermonde kernel + FFT convolution (the truncated
    kernel makes the two views agree exactly)."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(5)
    t = to_dev(inp)
    K = s4.s4d_kernel_vandermonde(t["A"], t["B"], t["C"], t["log_dt"], inp["L"])
    y = s4.fft_conv(t["u"], K, t["D"])
    Ab, Bb = s4.s4d_discretize_zoh(t["A"], t["B"], t["log_dt"])
    Bt, H = inp["Bt"], inp["H"]
    x = torch.zeros(Bt, H, inp["Nh"], dtype=torch.complex64, device="cuda")
    T = 1024
    ys = torch.empty(Bt, H, T, device="cuda")
    for k in range(T):
        ys[:, :, k] = s4.recurrent_step(Ab, Bb, t["C"], t["D"], x, t["u"][:, :, k].contiguous())
    torch.cuda.synchronize()
    assert rel_l2(ys.cpu().numpy(), y[:, :, :T].cpu().numpy()) <= Y_TOL
    # the one-launch scan gives the same numbers as the single steps
    x2 = torch.zeros_like(x)
    ys2 = s4.recurrent_scan(Ab, Bb, t["C"], t["D"], x2, t["u"][:, :, :T].contiguous())
    torch.cuda.synchronize()
    assert torch.allclose(ys2, ys, rtol=1e-5, atol=1e-5)
    assert torch.allclose(x2, x, rtol=1e-5, atol=1e-5)
    # and the sampled rows against the oracle recurrence
    rows = [(0, 0), (7, 300), (31, 1023)]
    Abr, Bbr = workloads.s4d_params(inp, channels=[h for _, h in rows])
    u_rows = np.stack([inp["u"][b, h, :T] for b, h in rows]).astype(np.float64)
    yr, _ = ssm.recurrence_diag(Abr, Bbr, inp["C"][[h for _, h in rows]].astype(np.complex128),
                                inp["D"][[h for _, h in rows]].astype(np.float64), u_rows,
                                np.arange(len(rows)))
    yg = np.stack([ys[b, h].cpu().numpy() for b, h in rows])
    assert rel_l2(yg, yr) <= Y_TOL


def test_dplr_discretize_matches_oracle():
    import structured_state_space_dplr_b200 as s4
    inp = s4inputs.make_inputs(1, with_u=False)
    t = to_dev(inp, ["Lambda", "P", "Q", "B", "C", "log_dt"])
    Ab, Bb, Cf = s4.dplr_discretize(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"])
    for h in range(inp["H"]):
        Abr, Bbr, Cfr = workloads.dplr_discretized(inp, h)
        assert np.abs(Ab[h].cpu().numpy() - Abr).max() <= 2e-5 * np.abs(Abr).max()
        assert np.abs(Bb[h].cpu().numpy() - Bbr).max() <= 2e-5 * np.abs(Bbr).max()
        assert np.abs(Cf[h].cpu().numpy() - Cfr).max() <= 1e-7


def test_dplr_dense_decode_matches_convolution_once_decayed():
    """Dense O(N^2) steps vs the aliased-kernel convolution on channels whose
    kernel has decayed within L ("Aliasing" paragraph of §4)."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(1, L=1024)
    inp["log_dt"][:] = np.float32(math.log(0.06))
    t = to_dev(inp)
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], inp["L"])
    y = s4.fft_conv(t["u"], K, t["D"])
    Ab, Bb, Cf = s4.dplr_discretize(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"])
    x = torch.zeros(inp["Bt"], inp["H"], 64, dtype=torch.complex64, device="cuda")
    T = 256
    ys = torch.empty(inp["Bt"], inp["H"], T, device="cuda")
    for k in range(T):
        ys[:, :, k] = s4.recurrent_step(Ab, Bb, Cf, t["D"], x, t["u"][:, :, k].contiguous())
    x2 = torch.zeros_like(x)
    ys2 = s4.recurrent_scan(Ab, Bb, Cf, t["D"], x2, t["u"][:, :, :T].contiguous())
    torch.cuda.synchronize()
    assert rel_l2(ys.cpu().numpy(), y[:, :, :T].cpu().numpy()) <= Y_TOL
    assert torch.allclose(ys2, ys, rtol=1e-5, atol=1e-5)
    # oracle recurrence for two rows
    rows = [(0, 0), (1, 3)]
    ures = []
    for b, h in rows:
        Abr, Bbr, Cfr = workloads.dplr_discretized(inp, h)
        yr, _ = ssm.recurrence_dense(Abr[None], Bbr[None], Cfr[None], np.array([float(inp["D"][h])]),
                                     inp["u"][b, h, :T][None].astype(np.float64), np.array([0]))
        ures.append(rel_l2(ys[b, h].cpu().numpy(), yr[0]))
    assert max(ures) <= Y_TOL
