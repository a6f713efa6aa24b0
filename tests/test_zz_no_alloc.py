"""s4_fft_conv_static: the FFT convolution for callers that cannot allocate
device memory (a plugin whose host application owns all GPU memory, or a
real-time path that must not call cudaMalloc). It uses the library's own
device scratch array instead of a caller workspace; its results must match
s4_fft_conv's. This file is collected last so that a stop-at-first-failure
run has already run every other test."""
import numpy as np
import pytest

from gpu_helpers import Y_TOL, rel_l2, torch_cuda

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_conv_two_calls_in_a_row():
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    rng = np.random.default_rng(2024)
    cases = [(16, 256, 4096), (3, 5, 1024)]   # second call: other sizes, odd batch
    outs = []
    for Bt, H, L in cases:
        u = torch.from_numpy(rng.standard_normal((Bt, H, L), dtype=np.float32)).cuda()
        K = torch.from_numpy((rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 4)))
                             .astype(np.float32)).cuda()
        D = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).cuda()
        y_static = s4.fft_conv_static(u, K, D)
        y_ref = s4.fft_conv(u, K, D)
        outs.append((y_static, y_ref))
    torch.cuda.synchronize()
    for y_static, y_ref in outs:
        assert rel_l2(y_static.cpu().numpy(), y_ref.cpu().numpy()) <= Y_TOL


def test_static_scratch_rejects_sizes_beyond_its_limit():
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    H, L = 1024, 4096          # needs 64 MiB of scratch, the array holds 32 MiB
    u = torch.zeros(1, H, L, device="cuda")
    K = torch.zeros(H, L, device="cuda")
    D = torch.zeros(H, device="cuda")
    with pytest.raises(s4.S4Error) as e:
        s4.fft_conv_static(u, K, D)
    assert e.value.status == 2
