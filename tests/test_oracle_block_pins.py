"""Pins of the S4Block oracle (pre-norm, GLU-gated projection, residual;
"The S4 kernel, from scratch", §6) against library routines, closed forms
and invariants."""
import math

import numpy as np
import torch
import torch.nn.functional as F

import s4inputs
from oracle import block, ssm


def _rand(seed, Bt=2, H=6, L=9):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bt, H, L)) * 1.7 + 0.4
    return rng, x


def test_sigmoid_closed_form_and_extremes():
    xs = np.array([-800.0, -30.0, -1.0, 0.0, 0.5, 30.0, 800.0])
    s = block.sigmoid(xs)
    for x, v in zip(xs[1:-1], s[1:-1]):
        assert abs(v - 1.0 / (1.0 + math.exp(-x))) < 1e-16
    assert s[0] == 0.0 and s[-1] == 1.0 and s[3] == 0.5


def test_layer_norm_matches_torch_layer_norm():
    rng, x = _rand(1)
    g = rng.standard_normal(6); b = rng.standard_normal(6)
    z = block.layer_norm_channels(x, g, b, 1e-5)
    ref = F.layer_norm(torch.from_numpy(x).transpose(1, 2), (6,), torch.from_numpy(g),
                       torch.from_numpy(b), eps=1e-5).transpose(1, 2).numpy()
    assert np.abs(z - ref).max() < 1e-13


def test_layer_norm_invariants():
    rng, x = _rand(2, H=17)
    eps = 0.3
    z = block.layer_norm_channels(x, np.ones(17), np.zeros(17), eps)
    var = x.var(axis=1)                      # biased
    assert np.abs(z.mean(axis=1)).max() < 1e-14
    assert np.abs((z ** 2).mean(axis=1) - var / (var + eps)).max() < 1e-14
    # scale and shift invariance (up to eps, which scales with the variance)
    z2 = block.layer_norm_channels(3.0 * x - 5.0, np.ones(17), np.zeros(17), 9.0 * eps)
    assert np.abs(z2 - z).max() < 1e-13
    # a channel-constant input gives beta
    c = np.broadcast_to(rng.standard_normal((2, 1, 9)), (2, 17, 9))
    beta = rng.standard_normal(17)
    zc = block.layer_norm_channels(c, rng.standard_normal(17), beta, 1e-5)
    # (x - mean) is a rounding residue, amplified by 1/sqrt(eps)
    assert np.abs(zc - beta[None, :, None]).max() < 1e-12


def test_glu_projection_matches_torch_linear_and_glu():
    rng, y = _rand(3, H=5)
    W = rng.standard_normal((10, 5)); bias = rng.standard_normal(10)
    g = block.glu_projection(y, W, bias)
    ref = F.glu(F.linear(torch.from_numpy(y).transpose(1, 2), torch.from_numpy(W), torch.from_numpy(bias)),
                dim=-1).transpose(1, 2).numpy()
    assert np.abs(g - ref).max() < 1e-14


def test_glu_value_and_gate_rows():
    """W = [I; 0], bias = [0; c]: the value rows pass y and the gate rows give
    sigmoid(c); a swap of value and gate would give c * sigmoid(y)."""
    rng, y = _rand(4, H=4)
    W = np.vstack([np.eye(4), np.zeros((4, 4))])
    c = np.array([-2.0, 0.0, 1.0, 3.0])
    g = block.glu_projection(y, W, np.concatenate([np.zeros(4), c]))
    assert np.abs(g - y * (1.0 / (1.0 + np.exp(-c)))[None, :, None]).max() < 1e-15


def test_block_reduces_to_residual_and_to_norm_path():
    rng, x = _rand(5, H=4, L=12)
    g, b = rng.standard_normal(4), rng.standard_normal(4)
    K, D = rng.standard_normal((4, 12)), rng.standard_normal(4)
    # a zero projection leaves x
    out = block.s4_block(x, g, b, 1e-5, K, D, np.zeros((8, 4)), np.zeros(8))
    assert np.abs(out - x).max() == 0.0
    # K = delta_0, D = 0: the S4 layer is the identity
    Kd = np.zeros((4, 12)); Kd[:, 0] = 1.0
    W, bias = rng.standard_normal((8, 4)), rng.standard_normal(8)
    out = block.s4_block(x, g, b, 1e-5, Kd, np.zeros(4), W, bias)
    xt = torch.from_numpy(x).transpose(1, 2)
    z = F.layer_norm(xt, (4,), torch.from_numpy(g), torch.from_numpy(b), eps=1e-5)
    ref = (xt + F.glu(F.linear(z, torch.from_numpy(W), torch.from_numpy(bias)), dim=-1)).transpose(1, 2).numpy()
    assert np.abs(out - ref).max() < 1e-13


def test_block_matches_library_composition():
    """Norm (torch), convolution (numpy.convolve per row), projection and GLU
    (torch), residual: the whole block, random parameters."""
    p = s4inputs.block_params(0, 3)
    rng = np.random.default_rng(6)
    x = rng.standard_normal((2, 3, 20))
    K, D = rng.standard_normal((3, 20)), rng.standard_normal(3)
    out = block.s4_block(x, p["gamma"], p["beta"], p["eps"], K, D, p["W"], p["bias"])
    f64 = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    z = F.layer_norm(f64(x).transpose(1, 2), (3,), f64(p["gamma"]), f64(p["beta"]),
                     eps=p["eps"]).transpose(1, 2).numpy()
    y = np.empty_like(z)
    for bb in range(2):
        for h in range(3):
            y[bb, h] = np.convolve(K[h], z[bb, h])[:20] + D[h] * z[bb, h]
    ref = x + F.glu(F.linear(f64(y).transpose(1, 2), f64(p["W"]), f64(p["bias"])), dim=-1).transpose(1, 2).numpy()
    assert np.abs(out - ref).max() < 1e-12
    assert np.abs(ssm.causal_conv(z, K, D) - y).max() < 1e-12
