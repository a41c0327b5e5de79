"""Pins for the oracle: checks against things other than the oracle itself.

Each pin takes an oracle library handle (``oracle.load()`` or a mutant build)
and raises AssertionError on mismatch.  ``run_all`` returns the names of the
pins that failed, so the mutant test can require that every planted mistake is
caught by at least one pin.

Sources of truth used here (none of them is the oracle's own formula retyped):
  * hand-computed fixtures (tests/golden/conv_hand_examples.txt);
  * closed forms: delta inputs, constant inputs (arithmetic series), ramp
    inputs (sum of j(t-j) = (t^3 - t)/6), geometric kernels;
  * a library routine: numpy.convolve on single rows (fp64 and int64);
  * an independent algorithm: an fp64 real FFT of length 2L, truncated;
  * invariants: commutativity, bilinearity, shift equivariance, strict
    causality under future perturbation, den >= |r|, den == r for
    non-negative inputs, sampled == full.
"""
from __future__ import annotations

import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "conv_hand_examples.txt")


def load_golden(path: str = GOLDEN):
    cases = []
    cur = None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            if key in ("case", "bwdcase"):
                cur = {"name": rest[0], "kind": key, "shape": tuple(int(x) for x in rest[1:4])}
                cases.append(cur)
            else:
                cur[key] = np.array([float(x) for x in rest], np.float64).reshape(cur["shape"])
    return cases


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ---------------------------------------------------------------- pins ----

def pin_golden(lib):
    for c in load_golden():
        if c["kind"] == "bwdcase":
            dv, _, dg, _ = oracle.causal_conv_bwd(c["dr"], c["v"], c["g"], lib=lib)
            assert np.array_equal(dv, c["dv"]) and np.array_equal(dg, c["dg"]), (c["name"], dv.ravel(), dg.ravel())
            continue
        r, den = oracle.causal_conv(c["v"], c["g"], lib=lib)
        assert np.array_equal(r, c["r"]), (c["name"], r.ravel(), c["r"].ravel())
        assert np.array_equal(den, c["den"]), (c["name"], den.ravel(), c["den"].ravel())
        r32, den32 = oracle.causal_conv(c["v"].astype(np.float32), c["g"].astype(np.float32), lib=lib)
        assert np.array_equal(r32, c["r"]) and np.array_equal(den32, c["den"]), c["name"]
        if np.all(c["v"] == np.round(c["v"])) and np.all(c["g"] == np.round(c["g"])):
            ri = oracle.causal_conv_int(c["v"].astype(np.int32), c["g"].astype(np.int32), lib=lib)
            assert np.array_equal(ri, c["r"].astype(np.int64)), (c["name"], ri.ravel())
        B, L, D = c["shape"]
        pts = np.array([(b, t, d) for b in range(B) for t in range(L) for d in range(D)], np.int64)
        rp, dp = oracle.causal_conv_points(c["v"], c["g"], pts, lib=lib)
        assert np.array_equal(rp, c["r"].ravel()) and np.array_equal(dp, c["den"].ravel()), c["name"]


def pin_delta(lib):
    B, L, D = 2, 37, 3
    g = _rng(1).standard_normal((B, L, D))
    for s in (0, 1, 5, 36):
        v = np.zeros((B, L, D))
        v[:, s, :] = 1.0
        expect = np.zeros((B, L, D))
        expect[:, s:, :] = g[:, : L - s, :]
        r, _ = oracle.causal_conv(v, g, lib=lib)
        assert np.array_equal(r, expect), f"v=e_{s}"
        r, _ = oracle.causal_conv(g, v, lib=lib)
        assert np.array_equal(r, expect), f"g=e_{s}"
    gi = _rng(2).integers(-128, 128, (B, L, D)).astype(np.int32)
    vi = np.zeros((B, L, D), np.int32)
    vi[:, 3, :] = 1
    expect = np.zeros((B, L, D), np.int64)
    expect[:, 3:, :] = gi[:, : L - 3, :]
    assert np.array_equal(oracle.causal_conv_int(vi, gi, lib=lib), expect)


def pin_closed_forms(lib):
    B, L, D = 1, 200, 2
    t = np.arange(L, dtype=np.float64).reshape(1, L, 1)
    ones = np.ones((B, L, D))
    # constant inputs: r_t = a*c*(t+1)
    r, den = oracle.causal_conv(0.5 * ones, 3.0 * ones, lib=lib)
    assert np.array_equal(r, np.broadcast_to(1.5 * (t + 1), r.shape))
    assert np.array_equal(den, r)
    # ramp kernel: v = 1, g_k = k -> r_t = t(t+1)/2
    r, _ = oracle.causal_conv(ones, np.broadcast_to(t, ones.shape).copy(), lib=lib)
    assert np.array_equal(r, np.broadcast_to(t * (t + 1) / 2, r.shape))
    # ramp * ramp: sum_j j(t-j) = (t^3 - t)/6
    ramp = np.broadcast_to(t, ones.shape).copy()
    r, _ = oracle.causal_conv(ramp, ramp, lib=lib)
    assert np.array_equal(r, np.broadcast_to((t ** 3 - t) / 6, r.shape))
    # geometric kernel: v = 1, g_k = rho^k -> (1 - rho^(t+1)) / (1 - rho)
    rho = 0.97
    r, _ = oracle.causal_conv(ones, np.broadcast_to(rho ** t, ones.shape).copy(), lib=lib)
    expect = (1 - rho ** (t + 1)) / (1 - rho)
    assert np.allclose(r, np.broadcast_to(expect, r.shape), rtol=1e-13, atol=0)
    # alternating signs: v_j = (-1)^j, g = 1 -> r_t = 1 if t even else 0; den_t = t+1
    alt = np.broadcast_to((-1.0) ** t, ones.shape).copy()
    r, den = oracle.causal_conv(alt, ones, lib=lib)
    assert np.array_equal(r, np.broadcast_to((t % 2 == 0).astype(np.float64), r.shape))
    assert np.array_equal(den, np.broadcast_to(t + 1, den.shape))
    # integer extremes (int64-exact): all -128 -> 16384 (t+1); 127 x -128 -> -16256 (t+1)
    L = 8192
    ti = np.arange(L, dtype=np.int64).reshape(1, L, 1)
    m128 = np.full((1, L, 2), -128, np.int32)
    p127 = np.full((1, L, 2), 127, np.int32)
    assert np.array_equal(oracle.causal_conv_int(m128, m128, lib=lib)[:, :, :1], 16384 * (ti + 1))
    assert np.array_equal(oracle.causal_conv_int(p127, m128, lib=lib)[:, :, 1:], -16256 * (ti + 1))
    assert oracle.causal_conv_int(m128, m128, lib=lib)[0, -1, 0] == 2 ** 27


def pin_numpy_convolve(lib):
    B, L, D = 2, 129, 3
    rng = _rng(3)
    v = rng.standard_normal((B, L, D))
    g = rng.standard_normal((B, L, D))
    r, den = oracle.causal_conv(v, g, lib=lib)
    vi = rng.integers(-128, 128, (B, L, D)).astype(np.int32)
    gi = rng.integers(-128, 128, (B, L, D)).astype(np.int32)
    ri = oracle.causal_conv_int(vi, gi, lib=lib)
    for b in range(B):
        for d in range(D):
            ref = np.convolve(v[b, :, d], g[b, :, d])[:L]
            assert np.allclose(r[b, :, d], ref, rtol=0, atol=1e-12 * max(1.0, den[b, :, d].max()))
            refd = np.convolve(np.abs(v[b, :, d]), np.abs(g[b, :, d]))[:L]
            assert np.allclose(den[b, :, d], refd, rtol=1e-13, atol=0)
            refi = np.convolve(vi[b, :, d].astype(np.int64), gi[b, :, d].astype(np.int64))[:L]
            assert np.array_equal(ri[b, :, d], refi)


def pin_fft_independent(lib):
    """fp64 real FFT of length 2L, product, inverse, truncate: a different
    algorithm reaching the same numbers (to rounding)."""
    B, L, D = 1, 256, 8
    rng = _rng(4)
    v = rng.standard_normal((B, L, D))
    g = rng.standard_normal((B, L, D))
    r, den = oracle.causal_conv(v, g, lib=lib)
    V = np.fft.rfft(v, n=2 * L, axis=1)
    G = np.fft.rfft(g, n=2 * L, axis=1)
    ref = np.fft.irfft(V * G, n=2 * L, axis=1)[:, :L, :]
    assert np.all(np.abs(r - ref) <= 1e-12 * np.maximum(den, 1e-300) + 1e-13)


def pin_symmetries(lib):
    B, L, D = 2, 64, 4
    rng = _rng(5)
    v, g, w = (rng.standard_normal((B, L, D)) for _ in range(3))
    r_vg, den = oracle.causal_conv(v, g, lib=lib)
    r_gv, den2 = oracle.causal_conv(g, v, lib=lib)
    assert np.all(np.abs(r_vg - r_gv) <= 1e-14 * den + 1e-300)
    assert np.allclose(den, den2, rtol=1e-14, atol=0)
    a, c = 0.75, -2.5
    r_lin, _ = oracle.causal_conv(a * v + c * w, g, lib=lib)
    r_w, den_w = oracle.causal_conv(w, g, lib=lib)
    assert np.all(np.abs(r_lin - (a * r_vg + c * r_w)) <= 1e-13 * (abs(a) * den + abs(c) * den_w) + 1e-300)
    # shift equivariance: delaying v by s delays r by s (bit-exact: only zero terms are added first)
    s = 7
    vs = np.zeros_like(v)
    vs[:, s:, :] = v[:, : L - s, :]
    r_s, _ = oracle.causal_conv(vs, g, lib=lib)
    assert np.array_equal(r_s[:, :s, :], np.zeros_like(r_s[:, :s, :]))
    assert np.array_equal(r_s[:, s:, :], r_vg[:, : L - s, :])
    # integer commutativity is exact
    vi = rng.integers(-128, 128, (B, L, D)).astype(np.int32)
    gi = rng.integers(-128, 128, (B, L, D)).astype(np.int32)
    assert np.array_equal(oracle.causal_conv_int(vi, gi, lib=lib), oracle.causal_conv_int(gi, vi, lib=lib))


def pin_causality(lib):
    B, L, D = 1, 100, 3
    rng = _rng(6)
    v = rng.standard_normal((B, L, D))
    g = rng.standard_normal((B, L, D))
    r, _ = oracle.causal_conv(v, g, lib=lib)
    for tc in (0, 31, 50, 98):
        v2, g2 = v.copy(), g.copy()
        v2[:, tc + 1:, :] = 1e4 * rng.standard_normal(v2[:, tc + 1:, :].shape)
        g2[:, tc + 1:, :] = 1e4 * rng.standard_normal(g2[:, tc + 1:, :].shape)
        r2, _ = oracle.causal_conv(v2, g2, lib=lib)
        assert np.array_equal(r[:, : tc + 1, :], r2[:, : tc + 1, :]), tc
        assert not np.array_equal(r[:, tc + 1:, :], r2[:, tc + 1:, :])


def pin_den(lib):
    B, L, D = 1, 50, 2
    rng = _rng(7)
    v = rng.standard_normal((B, L, D))
    g = rng.standard_normal((B, L, D))
    r, den = oracle.causal_conv(v, g, lib=lib)
    assert np.all(den >= np.abs(r))
    r, den = oracle.causal_conv(np.abs(v), np.abs(g), lib=lib)
    assert np.allclose(den, r, rtol=1e-15, atol=0)


def pin_points_match_full(lib):
    B, L, D = 2, 70, 5
    rng = _rng(8)
    v = rng.standard_normal((B, L, D)).astype(np.float32)
    g = rng.standard_normal((B, L, D)).astype(np.float32)
    r, den = oracle.causal_conv(v, g, lib=lib)
    pts = np.stack([rng.integers(0, B, 50), rng.integers(0, L, 50), rng.integers(0, D, 50)], 1)
    rp, dp = oracle.causal_conv_points(v, g, pts, lib=lib)
    assert np.array_equal(rp, r[pts[:, 0], pts[:, 1], pts[:, 2]])
    assert np.array_equal(dp, den[pts[:, 0], pts[:, 1], pts[:, 2]])
    vi = rng.integers(-128, 128, (B, L, D)).astype(np.int32)
    gi = rng.integers(-128, 128, (B, L, D)).astype(np.int32)
    ri = oracle.causal_conv_int(vi, gi, lib=lib)
    assert np.array_equal(oracle.causal_conv_int_points(vi, gi, pts, lib=lib), ri[pts[:, 0], pts[:, 1], pts[:, 2]])


# ---------------------------------------------------------- backward pins

def pin_bwd_adjoint(lib):
    """<dr, r(v, g)> = <dv, v> = <dg, g>: the gradient of the bilinear form
    sum_t dr_t r_t, checked against the (separately pinned) forward."""
    B, L, D = 2, 97, 3
    rng = _rng(20)
    dr, v, g = (rng.standard_normal((B, L, D)).astype(np.float32) for _ in range(3))
    r, _ = oracle.causal_conv(v, g, lib=lib)
    dv, _, dg, _ = oracle.causal_conv_bwd(dr, v, g, lib=lib)
    for b in range(B):
        for d in range(D):
            lhs = float(np.dot(dr[b, :, d].astype(np.float64), r[b, :, d]))
            assert abs(lhs - np.dot(dv[b, :, d], v[b, :, d].astype(np.float64))) <= 1e-11 * (1 + abs(lhs))
            assert abs(lhs - np.dot(dg[b, :, d], g[b, :, d].astype(np.float64))) <= 1e-11 * (1 + abs(lhs))


def pin_bwd_numpy_reversal(lib):
    """dv = rev(convolve(rev(dr), g)[:L]) with numpy's convolution."""
    B, L, D = 1, 64, 4
    rng = _rng(21)
    dr, v, g = (rng.standard_normal((B, L, D)).astype(np.float32) for _ in range(3))
    dv, den_dv, dg, _ = oracle.causal_conv_bwd(dr, v, g, lib=lib)
    for d in range(D):
        rdr = dr[0, ::-1, d].astype(np.float64)
        ref_v = np.convolve(rdr, g[0, :, d].astype(np.float64))[:L][::-1]
        ref_g = np.convolve(rdr, v[0, :, d].astype(np.float64))[:L][::-1]
        assert np.allclose(dv[0, :, d], ref_v, rtol=0, atol=1e-12 * den_dv.max())
        assert np.allclose(dg[0, :, d], ref_g, rtol=0, atol=1e-12 * den_dv.max() + 1e-12 * np.abs(ref_g).max())
        ad = np.convolve(np.abs(rdr), np.abs(g[0, :, d].astype(np.float64)))[:L][::-1]
        assert np.allclose(den_dv[0, :, d], ad, rtol=1e-13, atol=0)


def pin_bwd_autograd(lib):
    """torch autograd (fp64, CPU) through a forward built from torch's conv1d."""
    import torch
    B, L, D = 1, 40, 3
    rng = _rng(22)
    dr, v, g = (rng.standard_normal((B, L, D)).astype(np.float32) for _ in range(3))
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    tg = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    # r[b, t, d] = sum_j v[b, j, d] g[b, t-j, d]: depthwise conv1d of left-padded v with flipped g
    x = tv.permute(0, 2, 1).reshape(1, B * D, L)
    w = tg.permute(0, 2, 1).reshape(B * D, 1, L).flip(-1)
    r = torch.nn.functional.conv1d(torch.nn.functional.pad(x, (L - 1, 0)), w, groups=B * D)
    r = r.reshape(B, D, L).permute(0, 2, 1)
    (r * torch.tensor(dr, dtype=torch.float64)).sum().backward()
    dv, _, dg, _ = oracle.causal_conv_bwd(dr, v, g, lib=lib)
    assert np.allclose(dv, tv.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dg, tg.grad.numpy(), rtol=1e-12, atol=1e-12)


def pin_bwd_delta(lib):
    B, L, D = 1, 33, 2
    rng = _rng(23)
    v, g = (rng.standard_normal((B, L, D)).astype(np.float32) for _ in range(2))
    dr = np.zeros((B, L, D), np.float32)
    dr[:, L - 1, :] = 1.0  # only the last output matters: dv_j = g_{L-1-j}
    dv, _, dg, _ = oracle.causal_conv_bwd(dr, v, g, lib=lib)
    assert np.array_equal(dv, g[:, ::-1, :].astype(np.float64))
    assert np.array_equal(dg, v[:, ::-1, :].astype(np.float64))
    pts = np.array([(0, j, d) for j in range(L) for d in range(D)], np.int64)
    pv, _, pg, _ = oracle.causal_conv_bwd_points(dr, v, g, pts, lib=lib)
    assert np.array_equal(pv, dv.reshape(-1)) and np.array_equal(pg, dg.reshape(-1))


PINS = [pin_golden, pin_delta, pin_closed_forms, pin_numpy_convolve, pin_fft_independent,
        pin_symmetries, pin_causality, pin_den, pin_points_match_full,
        pin_bwd_adjoint, pin_bwd_numpy_reversal, pin_bwd_autograd, pin_bwd_delta]


def run_all(lib):
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    return failed
