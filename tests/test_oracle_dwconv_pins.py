"""The depthwise-convolution oracle (oracle/mhf_dwconv.py) against what the
page and the mathematics fix (CPU only); pins take the module so that they
can be run against planted mutants of its source."""
import os
import types

import numpy as np
import pytest
import torch

import oracle.mhf_dwconv as dw

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "mhf_dwconv_hand_examples.txt")


def _cases():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *rest = line.split()
        if key == "case":
            cur = {"name": rest[0], "shape": tuple(int(v) for v in rest[1:])}
            cases.append(cur)
        elif key == "bias" and rest == ["none"]:
            cur["bias"] = None
        else:
            cur[key] = np.array([float(v) for v in rest], np.float64)
    return cases


def _rand(B, L, D, K, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((B, L, D)), rng.uniform(-1, 1, (D, K)), rng.uniform(-1, 1, D)


def pin_golden(m):
    for c in _cases():
        B, L, D, K = c["shape"]
        y, yabs = m.causal_dwconv(c["x"].reshape(B, L, D), c["w"].reshape(D, K), c["bias"])
        np.testing.assert_allclose(y.ravel(), c["y"], rtol=0, atol=1e-12, err_msg=c["name"])
        assert (yabs >= np.abs(y) - 1e-12).all()


def pin_python_loops(m):
    for (B, L, D, K, seed) in [(2, 5, 3, 3, 1), (1, 2, 4, 4, 2), (1, 6, 2, 1, 3)]:
        x, w, bias = _rand(B, L, D, K, seed)
        ref = np.zeros((B, L, D))
        for b in range(B):
            for t in range(L):
                for d in range(D):
                    acc = bias[d]
                    for k in range(K):
                        tt = t - (K - 1) + k
                        if tt >= 0:
                            acc += w[d, k] * x[b, tt, d]
                    ref[b, t, d] = acc
        y, _ = m.causal_dwconv(x, w, bias)
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def pin_torch_depthwise_conv1d(m):
    """torch's depthwise conv1d (groups = D, float64, CPU) with K-1 zeros on the left."""
    for (B, L, D, K, seed) in [(2, 17, 12, 3, 4), (1, 9, 5, 1, 5), (3, 4, 8, 4, 6)]:
        x, w, bias = _rand(B, L, D, K, seed)
        xt = torch.nn.functional.pad(torch.from_numpy(x).transpose(1, 2), (K - 1, 0))
        yt = torch.nn.functional.conv1d(xt, torch.from_numpy(w).unsqueeze(1), torch.from_numpy(bias), groups=D)
        y, _ = m.causal_dwconv(x, w, bias)
        np.testing.assert_allclose(y, yt.transpose(1, 2).numpy(), rtol=0, atol=1e-12)


def pin_constant_input_closed_form(m):
    """x = 1: y[t, d] = bias[d] + sum_{k >= K-1-t} w[d, k]."""
    B, L, D, K = 1, 5, 6, 4
    _, w, bias = _rand(B, L, D, K, 7)
    y, _ = m.causal_dwconv(np.ones((B, L, D)), w, bias)
    for t in range(L):
        np.testing.assert_allclose(y[0, t], bias + w[:, max(0, K - 1 - t):].sum(axis=1), rtol=0, atol=1e-12)


def pin_causality_and_channels(m):
    B, L, D, K = 2, 12, 6, 3
    x, w, bias = _rand(B, L, D, K, 8)
    y0, _ = m.causal_dwconv(x, w, bias)
    for t0 in (0, 5, L - 2):
        x2 = x.copy()
        x2[:, t0 + 1:] = 9.0
        y1, _ = m.causal_dwconv(x2, w, bias)
        assert np.array_equal(y1[:, : t0 + 1], y0[:, : t0 + 1])
        assert not np.array_equal(y1[:, t0 + 1:], y0[:, t0 + 1:])
    x3 = x.copy()
    x3[:, :, 2] += 1.0
    y3, _ = m.causal_dwconv(x3, w, bias)
    others = [d for d in range(D) if d != 2]
    assert np.array_equal(y3[:, :, others], y0[:, :, others]) and (y3[:, :, 2] != y0[:, :, 2]).all()


def pin_error_scale(m):
    B, L, D, K = 2, 7, 5, 3
    x, w, bias = _rand(B, L, D, K, 9)
    y, yabs = m.causal_dwconv(x, w, bias)
    assert (yabs >= np.abs(y) * (1 - 1e-12)).all()
    y, yabs = m.causal_dwconv(np.abs(x), np.abs(w), np.abs(bias))
    np.testing.assert_allclose(yabs, y, rtol=1e-13, atol=0)


PINS = [pin_golden, pin_python_loops, pin_torch_depthwise_conv1d, pin_constant_input_closed_form,
        pin_causality_and_channels, pin_error_scale]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(dw)


MUTANTS = {
    "flipped_taps": ("lag = K - 1 - k", "lag = k"),
    "anticausal_shift": ("y[:, lag:, :] += w[:, k] * x[:, : L - lag, :]", "y[:, : L - lag, :] += w[:, k] * x[:, lag:, :]"),
    "dropped_bias": ("        y += bias\n", "        y += 0 * bias\n"),
    "signed_error_scale": ("np.abs(w[:, k]) * np.abs(x[:, : L - lag, :])", "w[:, k] * x[:, : L - lag, :]"),
    "dropped_last_tap": ("for k in range(K):", "for k in range(K - 1):"),
    "channel_mixup": ("y[:, lag:, :] += w[:, k] * x[:, : L - lag, :]", "y[:, lag:, :] += w[::-1, k] * x[:, : L - lag, :]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(dw.__file__).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"oracle.mhf_dwconv_mut_{name}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects mutant {name}"
