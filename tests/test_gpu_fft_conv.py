"""GPU parity of s4_fft_conv (zero-padded causal FFT convolution + D u)
against the oracle's direct O(L^2) sum ("The S4 kernel, from scratch", §5)."""
import numpy as np
import pytest

import s4inputs
from oracle import ssm, workloads
from gpu_helpers import Y_TOL, K_TOL, kernel_err, rel_l2, sample_times, to_dev, torch_cuda

pytestmark = pytest.mark.gpu


def _conv(u, K, D):
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    y = s4.fft_conv(torch.from_numpy(u).cuda(), torch.from_numpy(K).cuda(), torch.from_numpy(D).cuda())
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("L", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096])
@pytest.mark.parametrize("Bt,H", [(1, 1), (3, 2), (4, 3)])
def test_random_kernel_full_outputs(L, Bt, H):
    """Random (non-SSM) kernels: every output, odd batch (unpaired row) and H."""
    rng = np.random.default_rng(L * 10 + Bt)
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    K = (rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 4))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    yg = _conv(u, K, D)
    yr = ssm.causal_conv(u, K.astype(np.float64), D.astype(np.float64))
    assert rel_l2(yg, yr) <= Y_TOL
    # and per row, so a single bad row cannot hide in the norm
    for b in range(Bt):
        for h in range(H):
            assert rel_l2(yg[b, h], yr[b, h]) <= 4 * Y_TOL


@pytest.mark.parametrize("Bt,H", [(1, 1), (3, 2), (6, 3)])
def test_cluster_of_two_full_outputs(Bt, H):
    """L = 16384 (the transform split four ways over a cluster of two CTAs):
    every output, unpaired rows, several channels (at most nine row pairs,
    one per cluster; the test of more row pairs than resident units below
    gives each cluster several)."""
    L = 16384
    rng = np.random.default_rng(1600 + Bt)
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    K = (rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 4))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    yg = _conv(u, K, D)
    yr = ssm.causal_conv(u, K.astype(np.float64), D.astype(np.float64))
    assert rel_l2(yg, yr) <= Y_TOL
    for b in range(Bt):
        for h in range(H):
            assert rel_l2(yg[b, h], yr[b, h]) <= 4 * Y_TOL


@pytest.mark.parametrize("L", [8192, 16384, 32768, 65536])
def test_long_lengths_full_rows(L):
    """Every output of every row (an unpaired row included) at the long
    lengths: the cluster kernels' rank ranges, the cooperative first pass
    and the first-pass table in global memory all show up in full rows."""
    rng = np.random.default_rng(L)
    Bt, H = 3, 2
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    K = (rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 3))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    yg = _conv(u, K, D)
    rows = [(b, h) for b in range(Bt) for h in range(H)]
    ur = np.stack([u[b, h] for b, h in rows]).astype(np.float64)
    hh = np.array([h for _, h in rows])
    yr = ssm.causal_conv_rows_at(ur, hh, K.astype(np.float64), D.astype(np.float64), np.arange(L))
    ys = np.stack([yg[b, h] for b, h in rows])
    assert rel_l2(ys, yr) <= Y_TOL
    for i in range(len(rows)):
        assert rel_l2(ys[i], yr[i]) <= 4 * Y_TOL


def test_impulse_gives_kernel_plus_D():
    L, H = 1024, 3
    rng = np.random.default_rng(3)
    K = rng.standard_normal((H, L)).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    u = np.zeros((2, H, L), np.float32)
    u[:, :, 0] = 1.0
    yg = _conv(u, K, D)
    ref = K.astype(np.float64).copy()
    ref[:, 0] += D
    for b in range(2):
        assert rel_l2(yg[b], ref) <= Y_TOL


def test_cfg1_end_to_end():
    """GPU kernel -> GPU conv against oracle kernel -> direct conv, every output."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(1)
    t = to_dev(inp)
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], inp["L"])
    y = s4.fft_conv(t["u"], K, t["D"])
    torch.cuda.synchronize()
    Kr = workloads.dplr_kernel(inp)
    yr = workloads.conv_full(inp, Kr)
    assert kernel_err(K.cpu().numpy(), Kr) <= K_TOL
    assert rel_l2(y.cpu().numpy(), yr) <= Y_TOL


@pytest.mark.parametrize("cfg,channels", [(2, [0, 77, 255]), (3, [0, 200]), (4, [5, 63])])
def test_full_size_sampled(cfg, channels):
    """Full workload sizes and the benchmark's launch: GPU K and GPU y, checked
    on sampled channels, rows and output times against the oracle."""
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    inp = s4inputs.make_inputs(cfg)
    t = to_dev(inp)
    K = s4.kernel_dplr(t["Lambda"], t["P"], t["Q"], t["B"], t["C"], t["log_dt"], inp["L"])
    y = s4.fft_conv(t["u"], K, t["D"])
    torch.cuda.synchronize()
    Kr = workloads.dplr_kernel(inp, channels=channels)
    Kg = K.cpu().numpy()
    assert kernel_err(Kg[channels], Kr) <= K_TOL
    L = inp["L"]
    ts = sample_times(L, 48, seed=cfg)
    rows = [(b, h) for h in channels for b in (0, inp["Bt"] - 1)]
    Krows = [Kr[channels.index(h)] for _, h in rows]
    yr = workloads.conv_rows_at(inp, Krows, rows, ts)
    yg = y.cpu().numpy()
    ys = np.stack([yg[b, h][ts] for b, h in rows])
    assert rel_l2(ys, yr) <= Y_TOL


def test_prepare_apply_matches_one_call():
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    rng = np.random.default_rng(9)
    u = torch.from_numpy(rng.standard_normal((5, 4, 2048), dtype=np.float32)).cuda()
    K = torch.from_numpy(rng.standard_normal((4, 2048)).astype(np.float32)).cuda()
    D = torch.from_numpy(rng.standard_normal(4).astype(np.float32)).cuda()
    y1 = s4.fft_conv(u, K, D)
    ws = s4.fft_conv_prepare(K, D)
    y2 = s4.fft_conv_apply(u, ws)
    y3 = s4.fft_conv_apply(u[:3].contiguous(), ws)
    ws0 = s4.fft_conv_prepare(K)          # no feed-through term
    y4 = s4.fft_conv_apply(u, ws0)
    torch.cuda.synchronize()
    assert rel_l2((y4 + D[None, :, None] * u).cpu().numpy(), y1.cpu().numpy()) <= Y_TOL
    assert torch.equal(y1, y2)
    # rows 0 and 1 form the same packed pair in both calls; row 2 is paired
    # with row 3 in one call and alone in the other, so it only rounds alike
    assert torch.equal(y1[:2], y3[:2])
    assert rel_l2(y3[2].cpu().numpy(), y1[2].cpu().numpy()) <= Y_TOL


def test_workspace_too_small_is_rejected():
    import structured_state_space_dplr_b200 as s4
    torch = torch_cuda()
    u = torch.zeros(2, 2, 256, device="cuda")
    K = torch.zeros(2, 256, device="cuda")
    D = torch.zeros(2, device="cuda")
    ws = torch.empty(s4.fft_conv_workspace_size(2, 256) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(s4.S4Error) as e:
        s4.fft_conv(u, K, D, workspace=ws)
    assert e.value.status == 3


@pytest.mark.parametrize("Bt,H,L", [(3, 100, 16384), (3, 200, 4096)])
def test_more_row_pairs_than_resident_units_with_an_unpaired_row(Bt, H, L):
    """Each persistent CTA (cluster at L = 16384) runs several row pairs, and
    with an odd batch every other pair has no second row: at L = 16384 the
    L2 prefetch of a following pair skips that row, at L = 4096 the staged
    copy zero-fills it. Every output of rows from late pairs (paired and
    unpaired) against the oracle's direct sum."""
    rng = np.random.default_rng(1700 + L)
    u = rng.standard_normal((Bt, H, L), dtype=np.float32)
    K = (rng.standard_normal((H, L)) * np.exp(-np.arange(L) / (L / 4))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    yg = _conv(u, K, D)
    rows = [(2, H - 1), (0, H - 1), (1, H - 1), (2, H // 2 + 1), (2, 3 * H // 4), (0, H // 2)]
    ur = np.stack([u[b, h] for b, h in rows]).astype(np.float64)
    yr = ssm.causal_conv_rows_at(ur, np.array([h for _, h in rows]), K.astype(np.float64), D.astype(np.float64),
                                 np.arange(L))
    for i, (b, h) in enumerate(rows):
        assert rel_l2(yg[b, h], yr[i]) <= 4 * Y_TOL, (b, h)
