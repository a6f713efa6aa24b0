"""GPU parity of the structured (diagonal-plus-rank-1) DPLR decode step:
bilinear rule of "The S4 kernel, from scratch" §3 on the §2 DPLR system,
stepped as the §5 recurrent view in O(Nh) per token. Checked against the
oracle's dense bilinear discretisation and its dense recurrence over the full
conjugate-closed system."""
import numpy as np
import pytest

import s4inputs
from oracle import ssm, workloads
from gpu_helpers import Y_TOL, rel_l2, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _inputs(kind, L):
    if kind == "hippo":   # HiPPO-LegS modes, H = 4, Nh = 32, batch 2
        return s4inputs.make_inputs(1, L=L)
    # random DPLR system with P != Q and Nh = 40 (some lanes hold two modes)
    return s4inputs.random_dplr(7, H=6, Nh=40, L=L, Bt=3)


@pytest.mark.parametrize("kind", ["hippo", "random"])
def test_structured_transition_equals_dense_oracle(kind):
    import structured_state_space_dplr_b200 as s4
    inp = _inputs(kind, 64)
    t = to_dev(inp, ["Lambda", "P", "Q", "B", "log_dt"])
    Astr, Bb = s4.dplr_discretize_structured(t["Lambda"], t["P"], t["Q"], t["B"], t["log_dt"])
    Astr = Astr.cpu().numpy().astype(np.complex128)
    Bb = Bb.cpu().numpy().astype(np.complex128)
    Nh = Astr.shape[1]
    full = lambda v: np.concatenate([v, np.conj(v)])
    for h in range(inp["H"]):
        Abr, Bbr, _ = workloads.dplr_discretized(inp, h)
        a, g, be = (full(Astr[h, :, i]) for i in range(3))
        Ad = np.diag(a) - np.outer(g, be)       # Abar = diag(a) - g beta^T
        assert np.abs(Ad - Abr).max() <= 2e-5 * np.abs(Abr).max()
        assert np.abs(Bb[h] - Bbr[:Nh]).max() <= 2e-5 * np.abs(Bbr).max()


@pytest.mark.parametrize("kind", ["hippo", "random"])
def test_structured_decode_matches_dense_oracle_recurrence(kind):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    T = 300
    inp = _inputs(kind, T)
    t = to_dev(inp)
    Bt, H = inp["Bt"], inp["H"]
    Astr, Bb = s4.dplr_discretize_structured(t["Lambda"], t["P"], t["Q"], t["B"], t["log_dt"])
    Nh = Astr.shape[1]
    x = torch.zeros(Bt, H, Nh, dtype=torch.complex64, device="cuda")
    ys = torch.empty(Bt, H, T, device="cuda")
    for k in range(T):
        ys[:, :, k] = s4.recurrent_step(Astr, Bb, t["C"], t["D"], x, t["u"][:, :, k].contiguous())
    x2 = torch.zeros_like(x)
    ys2 = s4.recurrent_scan(Astr, Bb, t["C"], t["D"], x2, t["u"].contiguous())
    torch.cuda.synchronize()
    # one launch per token and T tokens per launch run the same arithmetic
    assert torch.equal(ys2, ys) and torch.equal(x2, x)
    yg, xg = ys.cpu().numpy(), x.cpu().numpy()
    yr_all, yg_all, xerr = [], [], []
    for b in range(Bt):
        for h in range(H):
            Abr, Bbr, Cfr = workloads.dplr_discretized(inp, h)
            yr, xr = ssm.recurrence_dense(Abr[None], Bbr[None], Cfr[None], np.array([float(inp["D"][h])]),
                                          inp["u"][b, h][None].astype(np.float64), np.array([0]))
            yr_all.append(yr[0])
            yg_all.append(yg[b, h])
            xr = np.asarray(xr).reshape(-1)
            # the stored half of the state, and its conjugate mirror in the oracle's full state
            assert np.abs(xr[Nh:] - np.conj(xr[:Nh])).max() <= 1e-9 * max(np.abs(xr).max(), 1e-30)
            xerr.append(np.linalg.norm(xg[b, h] - xr[:Nh]) / np.linalg.norm(xr[:Nh]))
    assert rel_l2(np.stack(yg_all), np.stack(yr_all)) <= Y_TOL
    assert max(xerr) <= 2e-4


def test_structured_and_dense_gpu_steps_agree_on_hippo_workload():
    """Same bilinear system, dense O(N^2) step and structured O(Nh) step."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(2, H=8, Bt=4, L=128)
    t = to_dev(inp)
    Ab, Bbd, Cf = s4.dplr_discretize(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"])
    Astr, Bbs = s4.dplr_discretize_structured(t["Lambda"], t["P"], t["Q"], t["B"], t["log_dt"])
    xd = torch.zeros(4, 8, 64, dtype=torch.complex64, device="cuda")
    xs = torch.zeros(4, 8, 32, dtype=torch.complex64, device="cuda")
    yd = s4.recurrent_scan(Ab, Bbd, Cf, t["D"], xd, t["u"].contiguous())
    ysr = s4.recurrent_scan(Astr, Bbs, t["C"], t["D"], xs, t["u"].contiguous())
    torch.cuda.synchronize()
    assert rel_l2(ysr.cpu().numpy(), yd.cpu().numpy()) <= Y_TOL
    assert rel_l2(xs.cpu().numpy(), xd[:, :, :32].cpu().numpy()) <= 2e-4
