"""Plain fp64 definition of the S4Block around the S4 convolution (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"The S4 kernel, from scratch", §6 "Trainable layer": the block puts a
pre-norm in front of the S4 layer and, after it, a projection gated by a GLU
and a residual connection. The page names the three parts and nothing more;
the readings taken here:

* the pre-norm is a layer norm over the H channels at each (batch, time):
  mean and biased variance over h, eps inside the square root, then a
  per-channel scale gamma[h] and shift beta[h];
* the S4 layer is the causal convolution of §5 with the kernel K and the
  feed-through D (``ssm.causal_conv``), applied to the normalised input;
* the projection is affine over channels, W [2H, H] and bias [2H], at each
  (batch, time); the GLU takes rows [0, H) as the value and rows [H, 2H) as
  the gate: value * sigmoid(gate);
* no other activation; the residual adds the block's input x.
"""
from __future__ import annotations

import numpy as np

from . import ssm


def sigmoid(x):
    """1 / (1 + exp(-x)), evaluated without overflow for either sign."""
    x = np.asarray(x, np.float64)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def layer_norm_channels(x, gamma, beta, eps):
    """z[b,h,t] = (x[b,h,t] - mean_h x[b,:,t]) / sqrt(var_h x[b,:,t] + eps)
    * gamma[h] + beta[h], with the biased variance (mean of squares about
    the mean). x: [Bt, H, L]."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    g = np.asarray(gamma, np.float64)[None, :, None]
    b = np.asarray(beta, np.float64)[None, :, None]
    return (x - mu) / np.sqrt(var + eps) * g + b


def glu_projection(y, W, bias):
    """p[b,:,t] = W y[b,:,t] + bias (W [2H, H]); returns
    p[b,:H,t] * sigmoid(p[b,H:,t]), shape [Bt, H, L]."""
    y = np.asarray(y, np.float64)
    H = y.shape[1]
    p = np.einsum("oh,bht->bot", np.asarray(W, np.float64), y) + np.asarray(bias, np.float64)[None, :, None]
    return p[:, :H] * sigmoid(p[:, H:])


def s4_block(x, gamma, beta, eps, K, D, W, bias):
    """out = x + GLU(W S4(LN(x)) + bias), S4(z) = causal_conv(z, K, D)."""
    z = layer_norm_channels(x, gamma, beta, eps)
    y = ssm.causal_conv(z, K, D)
    return np.asarray(x, np.float64) + glu_projection(y, W, bias)
