"""s4_fft_conv_static: the FFT convolution for callers that cannot allocate
device memory (a plugin whose host application owns all GPU memory, or a
real-time path that must not call cudaMalloc and take its implicit device
synchronisation). It uses the library's own device scratch array instead of
a caller workspace and runs the same kernels as s4_fft_conv, so its results
must equal s4_fft_conv's bit for bit and match the fp64 oracle's direct sum.
This file is collected last so that a stop-at-first-failure run has already
run every other test."""
import numpy as np
import pytest

from oracle import ssm
from gpu_helpers import Y_TOL, rel_l2, sample_times, torch_cuda

pytestmark = pytest.mark.gpu

LIMIT = 32 << 20   # S4_STATIC_SCRATCH_BYTES


def _case(rng, Bt, H, L):
    torch = torch_cuda()
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    K = (rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 4))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    return (u, K, D), tuple(torch.from_numpy(a).cuda() for a in (u, K, D))


def _oracle_rows(u, K, D, rows, ts):
    ur = np.stack([u[b, h] for b, h in rows]).astype(np.float64)
    hh = np.array([h for _, h in rows])
    return ssm.causal_conv_rows_at(ur, hh, K.astype(np.float64), D.astype(np.float64), ts)


def test_static_scratch_matches_workspace_conv_two_calls_in_a_row():
    """Two static calls in a row, each checked bit for bit against
    s4_fft_conv and, on every output, against the oracle. The shapes cover
    the one-CTA path (L = 1024, 4096) and the cluster path whose scratch
    also holds the first-pass table and the per-cluster slots (L = 32768,
    65536)."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    rng = np.random.default_rng(2024)
    for pair in ([(16, 256, 4096), (3, 5, 1024)], [(1, 4, 65536), (2, 4, 32768)]):
        outs = []
        for Bt, H, L in pair:
            host, (u, K, D) = _case(rng, Bt, H, L)
            y_static = s4.fft_conv_static(u, K, D)
            y_ref = s4.fft_conv(u, K, D)
            outs.append((host, y_static, y_ref))
        torch.cuda.synchronize()
        for (u, K, D), y_static, y_ref in outs:
            assert torch.equal(y_static, y_ref)
            Bt, H, L = u.shape
            rows = [(b, h) for b in range(Bt) for h in range(H)][:6]
            yr = _oracle_rows(u, K, D, rows, np.arange(L))
            yg = y_static.cpu().numpy()
            ys = np.stack([yg[b, h] for b, h in rows])
            assert rel_l2(ys, yr) <= Y_TOL
            for i in range(len(rows)):
                assert rel_l2(ys[i], yr[i]) <= 4 * Y_TOL


def test_static_scratch_at_its_limit_and_just_beyond():
    """At L = 65536 (spectrum, first-pass table and cluster slots all in the
    array) the largest H whose workspace fits the 32 MiB runs and matches
    s4_fft_conv; one more channel is rejected before anything is launched."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    L = 65536
    H = 1
    while s4.fft_conv_workspace_size(H + 1, L) <= LIMIT:
        H += 1
    assert s4.fft_conv_workspace_size(H, L) <= LIMIT < s4.fft_conv_workspace_size(H + 1, L)
    rng = np.random.default_rng(7)
    (u, K, D), (ud, Kd, Dd) = _case(rng, 1, H, L)
    y_static = s4.fft_conv_static(ud, Kd, Dd)
    y_ref = s4.fft_conv(ud, Kd, Dd)
    torch.cuda.synchronize()
    assert torch.equal(y_static, y_ref)
    ts = sample_times(L, 64, seed=L)
    rows = [(0, h) for h in range(H)]
    yr = _oracle_rows(u, K, D, rows, ts)
    yg = y_static.cpu().numpy()
    assert rel_l2(np.stack([yg[b, h][ts] for b, h in rows]), yr) <= Y_TOL
    u1 = torch.zeros(1, H + 1, L, device="cuda")
    with pytest.raises(s4.S4Error) as e:
        s4.fft_conv_static(u1, torch.zeros(H + 1, L, device="cuda"), torch.zeros(H + 1, device="cuda"))
    assert e.value.status == 2


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


def test_static_call_allocates_no_device_memory():
    """After a first call with the same shapes (which looks up the scratch
    address and loads the kernels), a call with a preallocated output leaves
    the device's free memory unchanged."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    rng = np.random.default_rng(11)
    _, (u, K, D) = _case(rng, 4, 8, 8192)
    out = torch.empty_like(u)
    s4.fft_conv_static(u, K, D, out=out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    s4.fft_conv_static(u, K, D, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free1 - free0) <= (2 << 20), (free0, free1)


def test_static_call_rejects_memory_the_device_cannot_address():
    """Plain (unregistered) host memory handed to the C ABI is refused before
    any launch: the kernels on the current device could not read it."""
    import ctypes

    import structured_state_space_dplr_b200 as s4
    from structured_state_space_dplr_b200 import _lib
    torch = torch_cuda()
    Bt, H, L = 1, 2, 1024
    u_host = np.zeros((Bt, H, L), np.float32)
    K = torch.zeros(H, L, device="cuda")
    D = torch.zeros(H, device="cuda")
    y = torch.empty(Bt, H, L, device="cuda")
    p = ctypes.c_void_p
    st = _lib.lib().s4_fft_conv_static(p(u_host.ctypes.data), p(K.data_ptr()), p(D.data_ptr()), Bt, H, L,
                                       p(y.data_ptr()), p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.S4_ERR_INVALID_ARG
    # the library still works afterwards
    u = torch.ones(Bt, H, L, device="cuda")
    assert torch.equal(s4.fft_conv_static(u, K, D), s4.fft_conv(u, K, D))
