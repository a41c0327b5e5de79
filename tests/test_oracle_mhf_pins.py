"""The gate-stream oracle (oracle/mhf_gate.py) against what the page and the
mathematics fix (CPU only).  Each pin takes the oracle module as an argument
so that the same pins can be run against planted mutants of its source."""
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle
import oracle.mhf_gate as mhf

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "mhf_gate_hand_examples.txt")


def _cases():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *rest = line.split()
        if key == "case":
            cur = {"name": rest[0], "shape": tuple(int(x) for x in rest[1:])}
            cases.append(cur)
        elif key == "bias" and rest == ["none"]:
            cur["bias"] = None
        else:
            cur[key] = np.array([float(x) for x in rest], np.float64)
    return cases


def _logit(s):
    return np.log(s / (1.0 - s))


def _rand(B, L, D, H, K, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    C = D // H
    a = rng.standard_normal((B, L, D))
    w = rng.uniform(-1, 1, (D, C, K)) / math.sqrt(C * K)
    bias = rng.uniform(-1, 1, D)
    return a, w, bias


def pin_golden(m):
    for c in _cases():
        B, L, D, H, K = c["shape"]
        a = _logit(c["s"]).reshape(B, L, D)
        w = c["w"].reshape(D, D // H, K)
        g, gabs = m.mhf_gate(a, w, c["bias"], H)
        np.testing.assert_allclose(g.ravel(), c["g"], rtol=0, atol=1e-12, err_msg=c["name"])
        assert (gabs >= np.abs(g) - 1e-12).all()
        r, den = m.mhf_gated_conv(c["v"].reshape(B, L, D), a, w, c["bias"], H)
        np.testing.assert_allclose(r.ravel(), c["r"], rtol=0, atol=1e-12, err_msg=c["name"])


def pin_python_loops(m):
    """Brute force: scalar loops over (b, t, c, k, c') with math.exp."""
    for (B, L, D, H, K, seed) in [(2, 5, 6, 3, 3, 1), (1, 4, 4, 1, 2, 2), (1, 3, 8, 2, 4, 3)]:
        a, w, bias = _rand(B, L, D, H, K, seed)
        C = D // H
        ref = np.zeros((B, L, D))
        for b in range(B):
            for t in range(L):
                for c in range(D):
                    h0 = (c // C) * C
                    acc = bias[c]
                    for k in range(K):
                        tt = t - (K - 1) + k
                        if tt < 0:
                            continue
                        for ci in range(C):
                            acc += w[c, ci, k] / (1.0 + math.exp(-a[b, tt, h0 + ci]))
                    ref[b, t, c] = acc
        g, _ = m.mhf_gate(a, w, bias, H)
        np.testing.assert_allclose(g, ref, rtol=0, atol=1e-12)


def pin_torch_grouped_conv1d(m):
    """A library routine for the same definition: torch's grouped conv1d (float64,
    CPU) on sigmoid(a) with K-1 zeros on the left."""
    for (B, L, D, H, K, seed) in [(2, 17, 12, 3, 1, 4), (1, 33, 16, 2, 3, 5), (3, 9, 8, 8, 4, 6),
                                  (1, 2, 6, 1, 4, 7)]:
        a, w, bias = _rand(B, L, D, H, K, seed)
        x = torch.sigmoid(torch.from_numpy(a)).transpose(1, 2)          # [B, D, L]
        x = torch.nn.functional.pad(x, (K - 1, 0))
        y = torch.nn.functional.conv1d(x, torch.from_numpy(w), torch.from_numpy(bias), groups=H)
        g, _ = m.mhf_gate(a, w, bias, H)
        np.testing.assert_allclose(g, y.transpose(1, 2).numpy(), rtol=0, atol=1e-12)


def pin_constant_input_closed_form(m):
    """a = 0: sigmoid = 1/2, so g[t, c] = bias[c] + (1/2) sum_{k >= K-1-t} sum_c' w[c, c', k]."""
    B, L, D, H, K = 1, 6, 8, 2, 4
    _, w, bias = _rand(B, L, D, H, K, 8)
    g, _ = m.mhf_gate(np.zeros((B, L, D)), w, bias, H)
    for t in range(L):
        kmin = max(0, K - 1 - t)
        ref = bias + 0.5 * w[:, :, kmin:].sum(axis=(1, 2))
        np.testing.assert_allclose(g[0, t], ref, rtol=0, atol=1e-12)


def pin_causality(m):
    """Changing a (or v) after t0 leaves g and r up to t0 unchanged, bit for bit."""
    B, L, D, H, K = 2, 20, 8, 2, 3
    a, w, bias = _rand(B, L, D, H, K, 9)
    v = np.random.Generator(np.random.PCG64(10)).standard_normal((B, L, D))
    g0, _ = m.mhf_gate(a, w, bias, H)
    r0, _ = m.mhf_gated_conv(v, a, w, bias, H)
    for t0 in (0, 7, L - 2):
        a2, v2 = a.copy(), v.copy()
        a2[:, t0 + 1:] = 50.0
        v2[:, t0 + 1:] = -3.0
        g1, _ = m.mhf_gate(a2, w, bias, H)
        r1, _ = m.mhf_gated_conv(v2, a2, w, bias, H)
        assert np.array_equal(g1[:, : t0 + 1], g0[:, : t0 + 1])
        assert np.array_equal(r1[:, : t0 + 1], r0[:, : t0 + 1])
        assert not np.array_equal(g1[:, t0 + 1:], g0[:, t0 + 1:])


def pin_head_isolation(m):
    """Changing the inputs of head 1 changes head 1's outputs and nothing else."""
    B, L, D, H, K = 1, 7, 12, 3, 2
    a, w, bias = _rand(B, L, D, H, K, 11)
    C = D // H
    g0, _ = m.mhf_gate(a, w, bias, H)
    a2 = a.copy()
    a2[:, :, C:2 * C] += 1.0
    g1, _ = m.mhf_gate(a2, w, bias, H)
    assert np.array_equal(g1[:, :, :C], g0[:, :, :C])
    assert np.array_equal(g1[:, :, 2 * C:], g0[:, :, 2 * C:])
    assert (g1[:, :, C:2 * C] != g0[:, :, C:2 * C]).all()


def pin_error_scales(m):
    """gabs >= |g| and den >= |r| always; with w, bias, v >= 0 they are equal."""
    B, L, D, H, K = 2, 9, 8, 2, 3
    a, w, bias = _rand(B, L, D, H, K, 12)
    v = np.random.Generator(np.random.PCG64(13)).standard_normal((B, L, D))
    g, gabs = m.mhf_gate(a, w, bias, H)
    r, den = m.mhf_gated_conv(v, a, w, bias, H)
    assert (gabs >= np.abs(g) * (1 - 1e-12)).all() and (den >= np.abs(r) * (1 - 1e-12)).all()
    w, bias, v = np.abs(w), np.abs(bias), np.abs(v)
    g, gabs = m.mhf_gate(a, w, bias, H)
    r, den = m.mhf_gated_conv(v, a, w, bias, H)
    np.testing.assert_allclose(gabs, g, rtol=1e-13, atol=0)
    np.testing.assert_allclose(den, r, rtol=1e-12, atol=0)


PINS = [pin_golden, pin_python_loops, pin_torch_grouped_conv1d, pin_constant_input_closed_form,
        pin_causality, pin_head_isolation, pin_error_scales]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(mhf)


def test_rejects_bad_shapes():
    a = np.zeros((1, 4, 6))
    with pytest.raises(ValueError):
        mhf.mhf_gate(a, np.zeros((6, 3, 1)), None, 4)       # D not a multiple of H
    with pytest.raises(ValueError):
        mhf.mhf_gate(a, np.zeros((6, 2, 1)), None, 2)       # w's second dim must be D/H


# Planted mistakes: each mutant of the oracle's source must fail at least one pin.
MUTANTS = {
    "flipped_taps": ("lag = K - 1 - k", "lag = k"),
    "anticausal_pad": ("g[:, lag:, ch] += src @ wk.T", "g[:, : L - lag, ch] += s[:, lag:, ch] @ wk.T"),
    "transposed_weight": ("g[:, lag:, ch] += src @ wk.T", "g[:, lag:, ch] += src @ wk"),
    "shared_head_weights": ("wk = w[ch, :, k]", "wk = w[:C, :, k]"),
    "sigmoid_sign": ("np.exp(-np.asarray(a, np.float64))", "np.exp(np.asarray(a, np.float64))"),
    "dropped_bias": ("        g += bias\n", "        g += 0 * bias\n"),
    "signed_error_scale": ("src @ np.abs(wk).T", "src @ wk.T"),
    "dropped_last_tap": ("for k in range(K):", "for k in range(K - 1):"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(mhf.__file__).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"oracle.mhf_gate_mut_{name}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects mutant {name}"
