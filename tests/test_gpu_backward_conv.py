"""GPU parity of the convolution's backward pass ("The S4 kernel, from
scratch", §5 fft_conv, trained as in §6): du by the adjoint (correlation)
convolution, dK and dD by the batch correlation of dy with u, against the
oracle's direct definitions (causal_conv_adjoint, causal_conv_kernel_grad)."""
import numpy as np
import pytest

from oracle import ssm
from gpu_helpers import Y_TOL, rel_l2, torch_cuda

pytestmark = pytest.mark.gpu

G_TOL = 1e-4   # per channel: max |d dK| / max |dK_ref|


def _case(seed, Bt, H, L, decay=True):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((Bt, H, L)).astype(np.float32)
    dy = rng.standard_normal((Bt, H, L)).astype(np.float32)
    K = rng.standard_normal((H, L)).astype(np.float32)
    if decay:   # kernels shaped like S4's: largest at small lags
        K *= np.exp(-np.arange(L) / (0.1 * L)).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    return u, dy, K, D


@pytest.mark.parametrize("L,Bt,H", [(16, 3, 2), (64, 2, 3), (512, 5, 2), (4096, 3, 2), (8192, 2, 2), (16384, 2, 2)])
def test_adjoint_convolution(L, Bt, H):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    u, dy, K, D = _case(L + Bt, Bt, H, L)
    Kd, Dd, dyd = (torch.from_numpy(a).cuda() for a in (K, D, dy))
    ws = s4.fft_conv_prepare(Kd, Dd)
    du = s4.fft_conv_apply_adjoint(dyd, ws)
    torch.cuda.synchronize()
    ref = ssm.causal_conv_adjoint(dy, K.astype(np.float64), D.astype(np.float64))
    assert rel_l2(du.cpu().numpy(), ref) <= Y_TOL


@pytest.mark.parametrize("L,Bt,H", [(16, 3, 2), (128, 2, 3), (1024, 5, 2), (4096, 4, 2), (8192, 3, 1),
                                    (16384, 3, 2), (32768, 2, 1), (65536, 2, 1), (16384, 1, 3)])
def test_kernel_and_skip_gradients(L, Bt, H):
    """L <= 8192: the batch correlation kernel; longer L: per batch row, the
    adjoint convolution with u's spectrum (the cluster transforms)."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    u, dy, _, _ = _case(7 * L + Bt, Bt, H, L)
    dK, dD = s4.fft_conv_kernel_grad(torch.from_numpy(u).cuda(), torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    dKr, dDr = ssm.causal_conv_kernel_grad(u, dy)
    dKg = dK.cpu().numpy()
    err = max(np.abs(dKg[h] - dKr[h]).max() / np.abs(dKr[h]).max() for h in range(H))
    assert err <= G_TOL
    assert rel_l2(dKg, dKr) <= Y_TOL
    assert np.allclose(dD.cpu().numpy(), dDr, rtol=1e-4, atol=1e-4 * np.abs(dDr).max())


def test_backward_matches_oracle_on_full_size_channels():
    """H = 256, L = 4096, batch 16 (the forward bench's shape), sampled channels."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    Bt, H, L = 16, 256, 4096
    u, dy, K, D = _case(99, Bt, H, L)
    ud, dyd, Kd, Dd = (torch.from_numpy(a).cuda() for a in (u, dy, K, D))
    ws = s4.fft_conv_prepare(Kd, Dd)
    du = s4.fft_conv_apply_adjoint(dyd, ws)
    dK, dD = s4.fft_conv_kernel_grad(ud, dyd)
    torch.cuda.synchronize()
    ch = [0, 131, 255]
    dKr, dDr = ssm.causal_conv_kernel_grad(u[:, ch], dy[:, ch])
    dKg = dK.cpu().numpy()[ch]
    assert max(np.abs(dKg[i] - dKr[i]).max() / np.abs(dKr[i]).max() for i in range(len(ch))) <= G_TOL
    assert np.allclose(dD.cpu().numpy()[ch], dDr, rtol=1e-4, atol=1e-4 * np.abs(dDr).max())
    rows = (0, 7, 15)
    dur = ssm.causal_conv_adjoint(dy[np.ix_(rows, ch)], K[ch].astype(np.float64), D[ch].astype(np.float64))
    assert rel_l2(du.cpu().numpy()[np.ix_(rows, ch)], dur) <= Y_TOL
