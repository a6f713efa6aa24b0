"""S4Block on the GPU (channel layer norm, tensor-core GLU projection with
residual, the composed block) against the fp64 oracle ("The S4 kernel, from
scratch", §6 "Trainable layer")."""
import numpy as np
import pytest

import s4inputs
from gpu_helpers import Y_TOL, rel_l2, to_dev, torch_cuda
from oracle import block, workloads

pytestmark = pytest.mark.gpu

# The projection's operands are split into bf16 high and low parts and three
# products are kept (A_hi B_hi + A_hi B_lo + A_lo B_hi): each term
# w * y is off by at most ~3 * 2^-17 |w y| (two split residues of 2^-18 and
# the dropped lo * lo term), plus fp32 accumulation. Bound per output on the
# sum of |terms|, with a factor 2 of margin:
TERM_TOL = 5e-5


def _rng_block(seed, Bt, H, L):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bt, H, L)).astype(np.float32)
    y = rng.standard_normal((Bt, H, L)).astype(np.float32)
    p = s4inputs.block_params(seed, H)
    return x, y, p


def _glu_bound(y, W, bias):
    """Elementwise error bound of out = x + v * sigmoid(g) for the split
    products: dv + 0.25 |v| dg, dv and dg = TERM_TOL x the sums of |terms|."""
    y = np.asarray(y, np.float64)
    W = np.asarray(W, np.float64)
    H = y.shape[1]
    S = np.einsum("oh,bht->bot", np.abs(W), np.abs(y)) + np.abs(np.asarray(bias, np.float64))[None, :, None]
    p = np.einsum("oh,bht->bot", W, y) + np.asarray(bias, np.float64)[None, :, None]
    return TERM_TOL * (S[:, :H] + 0.25 * np.abs(p[:, :H]) * S[:, H:]) + 1e-6


@pytest.mark.parametrize("Bt,H,L", [(2, 4, 16), (3, 100, 64), (2, 256, 1024), (1, 1024, 256)])
def test_layernorm_channels(Bt, H, L):
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    x, _, p = _rng_block(1, Bt, H, L)
    x = x * 3.0 + 7.0          # a large common offset: the shifted sums must not cancel
    d = to_dev({"x": x, "gamma": p["gamma"], "beta": p["beta"]})
    z = s4.layernorm_channels(d["x"], d["gamma"], d["beta"], p["eps"])
    torch.cuda.synchronize()
    ref = block.layer_norm_channels(x, p["gamma"], p["beta"], p["eps"])
    err = np.abs(z.cpu().numpy() - ref).max()
    assert err < 2e-5 * np.abs(ref).max(), err
    # in place gives the same values
    s4.layernorm_channels(d["x"], d["gamma"], d["beta"], p["eps"], out=d["x"])
    torch.cuda.synchronize()
    assert torch.equal(d["x"], z)


@pytest.mark.parametrize("Bt,H,L", [(2, 64, 128), (3, 100, 16), (2, 1, 64), (2, 256, 512), (1, 130, 32),
                                    (1, 1024, 256)])
def test_glu_projection_residual(Bt, H, L):
    """Whole tiles, ragged channel counts (partial row blocks and channel
    chunks), the smallest L (MMA N = 16), one channel, H = 1024 (32 chunks)."""
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    x, y, p = _rng_block(2, Bt, H, L)
    d = to_dev({"x": x, "y": y, "W": p["W"], "bias": p["bias"]})
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = s4.glu_projection_prepare(d["W"])
    out = s4.glu_projection_residual(d["y"], d["x"], d["bias"], ws, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    ref = x.astype(np.float64) + block.glu_projection(y, p["W"], p["bias"])
    err = np.abs(out.cpu().numpy() - ref)
    bound = _glu_bound(y, p["W"], p["bias"])
    assert (err <= bound).all(), (err.max(), np.unravel_index(np.argmax(err - bound), err.shape))
    assert rel_l2(out.cpu().numpy() - x, ref - x) < Y_TOL
    # out may be x (in place)
    s4.glu_projection_residual(d["y"], d["x"], d["bias"], ws, out=d["x"], flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(d["x"], out)


def test_glu_projection_full_size_sampled():
    """H = 256, L = 4096, batch 16 (the long-sequence workload's shape): all
    outputs at sampled (b, t) columns against the oracle."""
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    Bt, H, L = 16, 256, 4096
    x, y, p = _rng_block(3, Bt, H, L)
    d = to_dev({"x": x, "y": y, "W": p["W"], "bias": p["bias"]})
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = s4.glu_projection_prepare(d["W"])
    out = s4.glu_projection_residual(d["y"], d["x"], d["bias"], ws, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    o = out.cpu().numpy()
    rng = np.random.default_rng(4)
    ts = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 4095], rng.integers(0, L, 20)]))
    for b in (0, 7, 15):
        ys, xs = y[b:b + 1][:, :, ts], x[b:b + 1][:, :, ts]
        ref = xs.astype(np.float64) + block.glu_projection(ys, p["W"], p["bias"])
        assert (np.abs(o[b:b + 1][:, :, ts] - ref) <= _glu_bound(ys, p["W"], p["bias"])).all()


@pytest.mark.parametrize("H,L,Bt", [(4, 1024, 2), (64, 256, 3), (100, 16, 1)])
def test_block_forward_dplr(H, L, Bt):
    """The composed block with the DPLR layer: norm -> convolution with the
    aliased kernel (and D) -> projection, GLU, residual."""
    torch = torch_cuda()
    import structured_state_space_dplr_b200 as s4
    inp = s4inputs.make_inputs(1, H=H, Bt=Bt, L=L)
    p = s4inputs.block_params(5, H)
    x = inp["u"]
    d = to_dev(inp)
    d.update(to_dev({"gamma": p["gamma"], "beta": p["beta"], "W": p["W"], "bias": p["bias"]}))
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    conv_ws = torch.empty(s4.fft_conv_workspace_size(H, L), dtype=torch.uint8, device="cuda")
    s4.kernel_dplr_prepare(d["Lambda"], d["P"], d["Q"], d["B"], d["C"], d["log_dt"], d["D"], L,
                           workspace=conv_ws, flags=flags)
    glu_ws = s4.glu_projection_prepare(d["W"])
    out, z, yv = s4.block_forward(d["u"], d["gamma"], d["beta"], p["eps"], conv_ws, d["bias"], glu_ws, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    K = workloads.dplr_kernel(inp)
    ref = block.s4_block(x, p["gamma"], p["beta"], p["eps"], K, inp["D"].astype(np.float64), p["W"], p["bias"])
    assert rel_l2(out.cpu().numpy() - x, ref - x) < Y_TOL
    zref = block.layer_norm_channels(x, p["gamma"], p["beta"], p["eps"])
    assert rel_l2(z.cpu().numpy(), zref) < 1e-5
