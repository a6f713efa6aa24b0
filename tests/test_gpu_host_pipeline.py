"""The host-buffer entry points (s4_forward_dplr_host, s4_fft_conv_host):
chunked uploads, convolutions and downloads give exactly the device-buffer
results, and the oracle's."""
import numpy as np
import pytest

import s4inputs
from oracle import workloads
from gpu_helpers import Y_TOL, rel_l2, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Bt,chunks,pinned", [(5, 2, True), (4, 1, False), (3, 8, True), (16, 8, True)])
def test_forward_dplr_host_equals_device_path(Bt, chunks, pinned):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(2, H=16, Bt=Bt, L=512)
    t = to_dev(inp)
    y_dev = s4.forward_dplr(t["u"], t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"])
    u_host = torch.from_numpy(inp["u"].copy())
    if pinned:
        u_host = u_host.pin_memory()
    y_host = s4.forward_dplr_host(u_host, t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"],
                                  chunks=chunks)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(y_host, y_dev.cpu())


def test_fft_conv_host_matches_device_path_and_oracle():
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(1)   # H = 4, L = 1024, batch 2
    t = to_dev(inp)
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], inp["L"])
    y_dev = s4.fft_conv(t["u"], K, t["D"])
    y_host = s4.fft_conv_host(torch.from_numpy(inp["u"].copy()).pin_memory(), K, t["D"], chunks=3)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(y_host, y_dev.cpu())
    Kr = workloads.dplr_kernel(inp)
    yr = workloads.conv_full(inp, Kr)
    assert rel_l2(y_host.numpy(), yr) <= Y_TOL


@pytest.mark.parametrize("Bt,H,L,chunks", [(3, 6, 16384, 8), (2, 5, 4096, 16), (2, 3, 32768, 4), (1, 4, 8192, 4)])
def test_channel_sliced_chunks_equal_device_path(Bt, H, L, chunks):
    """Fewer row pairs than chunks: up to L = 16384 the pipeline also cuts
    channel slices (uneven ones included); longer L keeps whole row pairs.
    Either way the result is the device path's, bit for bit."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    rng = np.random.default_rng(L + Bt)
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    K = torch.from_numpy((rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 4))).astype(np.float32)).cuda()
    D = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).cuda()
    y_dev = s4.fft_conv(torch.from_numpy(u).cuda(), K, D)
    y_host = s4.fft_conv_host(torch.from_numpy(u).pin_memory(), K, D, chunks=chunks)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(y_host, y_dev.cpu())


def test_calls_in_flight_on_separate_streams_keep_their_results():
    """Three host-buffer calls with different parameters and inputs, each on
    its own stream with its own staging buffers, workspace, K and host
    output, queued back to back so that they overlap on the shared copy
    streams; the six steps rotate through the three buffer sets (a set is
    reused once its stream has finished the previous call). Every host
    output equals its own device-path result."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    H, L, Bt = 8, 4096, 6
    cases = []
    for seed in range(3):
        inp = s4inputs.make_inputs(2, seed=seed, H=H, Bt=Bt, L=L)
        t = to_dev(inp)
        y_ref = s4.forward_dplr(t["u"], t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"]).cpu()
        cases.append({"t": t, "u_host": torch.from_numpy(inp["u"].copy()).pin_memory(), "y_ref": y_ref,
                      "y_host": torch.empty(Bt, H, L).pin_memory(), "u_dev": torch.empty(Bt, H, L, device="cuda"),
                      "y_dev": torch.empty(Bt, H, L, device="cuda"), "K": torch.empty(H, L, device="cuda"),
                      "ws": torch.empty(s4.fft_conv_workspace_size(H, L), dtype=torch.uint8, device="cuda"),
                      "stream": torch.cuda.Stream()})
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    for c in cases:
        c["stream"].wait_stream(cur)
    for step in range(6):
        c = cases[step % 3]
        t = c["t"]
        with torch.cuda.stream(c["stream"]):
            s4.forward_dplr_host(c["u_host"], t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], t["D"],
                                 y_host=c["y_host"], K=c["K"], u_dev=c["u_dev"], y_dev=c["y_dev"],
                                 workspace=c["ws"], chunks=2)
    for c in cases:
        cur.wait_stream(c["stream"])
    torch.cuda.synchronize()
    for c in cases:
        assert torch.equal(c["y_host"], c["y_ref"])
