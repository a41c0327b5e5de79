"""Oracle for the causal depthwise convolution of the Multi-Head Fourier block
-- TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle``).

What it computes (Caracal: Causal Architecture via Spectral Mixing, "Key
design 1", the first step of the four-step MHF pipeline: a causal depthwise
1-D convolution with kernel size 3 that restores local patterns once the
positional encoding is gone): for channel-last [B, L, D] arrays and a K-tap
kernel per channel,

    y[b, t, d] = bias[d] + sum_{k<K} w[d][k] * x[b, t - (K - 1) + k, d],
    x[b, t, d] = 0 for t < 0                                    (causal pad)

with w in the layout of a depthwise Conv1d weight, [D, 1, K] flattened to
[D, K].  Readings where the page is silent: causal means K - 1 zeros on the
left and none on the right (the same convention as the page's causal
sequence convolution); the bias is present, as in a default Conv1d; the
output is the convolution alone (a residual connection, if any, is the
caller's); K = 3 is the page's value, other K are allowed.

Besides y it returns yabs = |bias| + sum |w| |x|, the scale of y's rounding
error.  Float64 numpy, one shifted multiply-add per tap; pins:
tests/test_oracle_dwconv_pins.py.
"""
from __future__ import annotations

import numpy as np


def causal_dwconv(x: np.ndarray, w: np.ndarray, bias: np.ndarray | None):
    """y and yabs (float64 [B, L, D]) for x [B, L, D] and w [D, K]."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    if x.ndim != 3:
        raise ValueError("x must be [B, L, D]")
    B, L, D = x.shape
    if w.ndim != 2 or w.shape[0] != D:
        raise ValueError("w must be [D, K]")
    K = w.shape[1]
    y = np.zeros((B, L, D), np.float64)
    yabs = np.zeros((B, L, D), np.float64)
    for k in range(K):
        lag = K - 1 - k                      # tap k reads x at time t - lag
        if lag >= L:
            continue
        y[:, lag:, :] += w[:, k] * x[:, : L - lag, :]
        yabs[:, lag:, :] += np.abs(w[:, k]) * np.abs(x[:, : L - lag, :])
    if bias is not None:
        bias = np.asarray(bias, np.float64).reshape(D)
        y += bias
        yabs += np.abs(bias)
    return y, yabs
