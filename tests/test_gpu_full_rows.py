"""Full-size workloads in the benchmark's launch configuration, checked on
EVERY output of whole rows against the fp64 oracle ("The S4 kernel, from
scratch", §4 kernel and §5 fft_conv; "S4" wiki page, section "S4D").

The DPLR workloads run s4_kernel_dplr_prepare + s4_fft_conv_apply and the
S4D workload s4d_kernel_vandermonde + s4_fft_conv_prepare +
s4_fft_conv_apply, exactly as the benchmark times them; the oracle forms its
own kernel (dense powers / the truncated Vandermonde sum in fp64) and the
direct O(L^2) causal sum over the full rows."""
import numpy as np
import pytest

import s4inputs
from oracle import workloads
from gpu_helpers import K_TOL, Y_TOL, kernel_err, rel_l2, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _check_rows(inp, yg_rows, Kref, rows):
    L = inp["L"]
    hs = sorted({h for _, h in rows})
    Krows = [Kref[hs.index(h)] for _, h in rows]
    yr = workloads.conv_rows_at(inp, Krows, rows, np.arange(L))
    ys = np.stack(yg_rows)
    assert rel_l2(ys, yr) <= Y_TOL
    for i in range(len(rows)):
        assert rel_l2(ys[i], yr[i]) <= 4 * Y_TOL, rows[i]


@pytest.mark.parametrize("cfg,rows", [(2, [(0, 0), (15, 255), (8, 128)]), (3, [(0, 3), (7, 254)]),
                                      (4, [(0, 1), (3, 62)])])
def test_dplr_full_size_full_rows(cfg, rows):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(cfg)
    t = to_dev(inp)
    ws = torch.empty(s4.fft_conv_workspace_size(inp["H"], inp["L"]), dtype=torch.uint8, device="cuda")
    K = torch.empty(inp["H"], inp["L"], device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    s4.kernel_dplr_prepare(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"], inp["L"],
                           K=K, workspace=ws, flags=flags)
    y = s4.fft_conv_apply(t["u"], ws)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    hs = sorted({h for _, h in rows})
    Kref = workloads.dplr_kernel(inp, channels=hs)
    assert kernel_err(K[hs].cpu().numpy(), Kref) <= K_TOL
    _check_rows(inp, [y[b, h].cpu().numpy() for b, h in rows], Kref, rows)


def test_s4d_full_size_full_rows():
    """Workload 5 (H = 1024, L = 8192, batch 32): four whole rows spread over
    the batch and the channels."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(5)
    t = to_dev(inp)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    K = s4.s4d_kernel_vandermonde(t["A"], t["B"], t["C"], t["log_dt"], inp["L"], flags=flags)
    ws = s4.fft_conv_prepare(K, t["D"])
    y = s4.fft_conv_apply(t["u"], ws)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    rows = [(0, 0), (9, 333), (20, 700), (31, 1023)]
    hs = sorted({h for _, h in rows})
    Kref = workloads.s4d_kernel(inp, channels=hs)
    assert kernel_err(K[hs].cpu().numpy(), Kref) <= K_TOL
    _check_rows(inp, [y[b, h].cpu().numpy() for b, h in rows], Kref, rows)
