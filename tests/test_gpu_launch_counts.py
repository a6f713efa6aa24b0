"""Launches per forward step, read from the kernel nodes of CUDA graphs that
capture the two stages exactly as the bench does (generation: the DPLR
kernel + spectrum, or the S4D Vandermonde kernel + spectrum; then the
convolution). The bench reports its `gpu_launches` from the same graph
nodes; this ties that count to the launches the library is designed to
issue at each length. Launch counts depend on L and the variant only, so
the workloads run here with a few channels and one row."""
import pytest

import bench
import s4inputs
from gpu_helpers import to_dev, torch_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_forward_launches_match_the_captured_graph(cfg):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    c = s4inputs.CONFIGS[cfg]
    H, L = 4, c["L"]
    inp = s4inputs.make_inputs(cfg, seed=1, H=H, Bt=1)
    d = to_dev(inp)
    K = torch.empty(H, L, device="cuda")
    y = torch.empty(1, H, L, device="cuda")
    ws = torch.empty(s4.fft_conv_workspace_size(H, L), dtype=torch.uint8, device="cuda")
    s4d = c["kind"] == "s4d"

    def gen():
        if s4d:
            s4.s4d_kernel_vandermonde(d["A"], d["B"], d["C"], d["log_dt"], L, out=K)
            s4.fft_conv_prepare(K, d["D"], workspace=ws)
        else:
            s4.kernel_dplr_prepare(d["Lambda"], d["P"], d["Q"], d["B"], d["C"], d["log_dt"], d["D"], L,
                                   K=K, workspace=ws)

    def conv():
        s4.fft_conv_apply(d["u"], ws, out=y)

    gen()
    conv()
    torch.cuda.synchronize()
    y_eager = y.clone()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g1, g2 = torch.cuda.CUDAGraph(keep_graph=True), torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g1, stream=cap):
            gen()
        with torch.cuda.graph(g2, stream=cap):
            conv()
    torch.cuda.current_stream().wait_stream(cap)
    n = bench.graph_kernel_nodes(g1) + bench.graph_kernel_nodes(g2)
    assert n == bench.launches_per_step(c), (cfg, n)
    y.zero_()
    g1.replay()
    g2.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)
