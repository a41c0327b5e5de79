"""Oracle for the gate stream of the Multi-Head Fourier block -- TEST
INFRASTRUCTURE ONLY (same rule as the package: only ``tests/``, the smoke
check and the CPU legs of the benchmark use it).

What it computes (Caracal: Causal Architecture via Spectral Mixing, "Key
design 1", the four-step MHF pipeline): the gate stream is

    x_g = Conv1d_G2( sigma( Linear_G1(x_norm) ) )

where the 1-D convolution is grouped by head (n_head groups, so channels mix
only inside a head), and the sequence convolution r_t = sum_{j<=t} v_j g_{t-j}
then takes g = x_g.  This module starts from a = Linear_G1(x_norm), the
projection's output, so for channel-last [B, L, D] arrays with C = D / H
channels per head and kernel size K:

    s[b, t, c]  = 1 / (1 + exp(-a[b, t, c]))                     (logistic)
    g[b, t, c]  = bias[c] + sum_{k<K} sum_{c' in head(c)}
                      w[c, c' - h0(c), k] * s[b, t - (K - 1) + k, c']
    s[b, t, .]  = 0 for t < 0                                      (causal pad)

with w in the layout of a grouped Conv1d weight, [D, C, K] (output channel,
input channel within the head, tap).  Readings where the page is silent:
sigma is the logistic function; the convolution is causal (K - 1 zeros on the
left, none on the right), since a centred kernel would let g_t see a_{t+1}
and the block is a next-token predictor; K is a parameter (the page gives no
kernel size for G2); the bias is present, as in a default Conv1d.

Besides g it returns the absolute chain gabs = |bias| + sum |w| s (s > 0), the
scale of g's rounding error.  ``mhf_gated_conv`` composes the gate with the
pinned causal-convolution oracle and returns r together with the error scale
den = sum_j |v_j| gabs_{t-j}.

Written in float64 numpy, one matrix product per (head, tap); pins:
tests/test_oracle_mhf_pins.py (hand-computed fixture, a pure-Python loop,
torch's grouped conv1d, closed forms, causality, head isolation, and mutants
of this source that the pins must reject).
"""
from __future__ import annotations

import numpy as np


def sigmoid(a: np.ndarray) -> np.ndarray:
    """Logistic function in float64."""
    return 1.0 / (1.0 + np.exp(-np.asarray(a, np.float64)))


def mhf_gate(a: np.ndarray, w: np.ndarray, bias: np.ndarray | None, n_head: int):
    """g and gabs (float64 [B, L, D]) for a [B, L, D], w [D, D/n_head, K]."""
    a = np.asarray(a, np.float64)
    w = np.asarray(w, np.float64)
    if a.ndim != 3:
        raise ValueError("a must be [B, L, D]")
    B, L, D = a.shape
    if n_head < 1 or D % n_head:
        raise ValueError("D must be a multiple of n_head")
    C = D // n_head
    if w.ndim != 3 or w.shape[0] != D or w.shape[1] != C:
        raise ValueError("w must be [D, D/n_head, K]")
    K = w.shape[2]
    s = sigmoid(a)
    g = np.zeros((B, L, D), np.float64)
    gabs = np.zeros((B, L, D), np.float64)
    for h in range(n_head):
        ch = slice(h * C, (h + 1) * C)
        for k in range(K):
            lag = K - 1 - k          # tap k reads s at time t - lag
            if lag >= L:
                continue
            src = s[:, : L - lag, ch]                    # times 0 .. L-1-lag
            wk = w[ch, :, k]                             # [C out, C in]
            g[:, lag:, ch] += src @ wk.T
            gabs[:, lag:, ch] += src @ np.abs(wk).T
    if bias is not None:
        bias = np.asarray(bias, np.float64).reshape(D)
        g += bias
        gabs += np.abs(bias)
    return g, gabs


def mhf_gated_conv(v: np.ndarray, a: np.ndarray, w: np.ndarray, bias: np.ndarray | None,
                   n_head: int, lib=None):
    """r = causal_conv(v, mhf_gate(a, w, bias)) and its error scale den, both
    float64 [B, L, D]; v is widened exactly."""
    from . import causal_conv

    g, gabs = mhf_gate(a, w, bias, n_head)
    v64 = np.asarray(v, np.float64)
    r, _ = causal_conv(v64, g, lib)
    den, _ = causal_conv(np.abs(v64), gabs, lib)
    return r, den
