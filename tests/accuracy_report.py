"""Accuracy and leakage report of the GPU paths, one JSON line per workload.

    python tests/accuracy_report.py [--workloads tiny_f32,small_f32,...] [--points N]

For each seeded workload (workloads.py) it runs the CUDA path through the
binding and compares with the oracle (the plain direct sum): on every output
where the oracle finishes in seconds, else on a stratified sample of (b, t, d)
points.  Reported per workload:

  * max_ratio: max over outputs of |r_gpu - r_exact| / (tol * den), with
    den = sum_j |v_j g_{t-j}| and tol = 1e-5 (fp32 I/O) or 2e-2 (bf16 I/O);
    for the NTT path the count of outputs that differ (must be 0);
  * violations: outputs with ratio > 1;
  * leakage: measured future-token leakage (the failure "Catastrophic Token
    Leakage in Convolutional Sequence Modeling and How to Mitigate It"
    describes for float FFT convolutions, and that its NTT primitive
    removes): max |r_{0..t_c}(perturbed) - r_{0..t_c}| when every v_j and
    g_j with j > t_c is replaced by fresh values (1e4 times larger for the
    float paths), at three cut points t_c; exactly 0 for the NTT path, > 0
    for a float transform outside the directly summed head (t < 32).

Test infrastructure (it calls the oracle); the GPU tests run it on the small
workloads.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import BF16_TOL, F32_TOL, as_f32, run_gpu  # noqa: E402

# outputs the oracle sums in full (else a sample of --points (b, t, d))
FULL_ORACLE_MAX_MACS = 6e10


def accuracy(w: workloads.Workload, v, g, r, n_points: int):
    macs = w.B * w.D * w.L * (w.L + 1) / 2
    full = macs <= FULL_ORACLE_MAX_MACS
    if w.dtype == "i32":
        if full:
            ref = oracle.causal_conv_int(v, g)
            diff = int(np.count_nonzero(r.astype(np.int64) != ref))
            return {"checked": "all", "outputs": int(ref.size), "differing": diff}
        pts = workloads.sample_points(w.B, w.L, w.D, n_points, seed=11)
        ref = oracle.causal_conv_int_points(v, g, pts)
        got = r[pts[:, 0], pts[:, 1], pts[:, 2]].astype(np.int64)
        return {"checked": "sample", "outputs": n_points, "differing": int(np.count_nonzero(got != ref))}
    vf, gf, rf = as_f32(v, w.dtype), as_f32(g, w.dtype), as_f32(r, w.dtype)
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    if full:
        ref, den = oracle.causal_conv(vf, gf)
        got, how, n = rf, "all", rf.size
    else:
        pts = workloads.sample_points(w.B, w.L, w.D, n_points, seed=11)
        ref, den = oracle.causal_conv_points(vf, gf, pts)
        got, how, n = rf[pts[:, 0], pts[:, 1], pts[:, 2]], "sample", n_points
    err = np.abs(np.asarray(got, np.float64) - ref)
    bound = tol * den
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    return {"checked": how, "outputs": int(n), "tol": tol, "max_ratio": float(ratio.max()),
            "violations": int((ratio > 1).sum())}


def leakage(w: workloads.Workload, v, g, r0, seed: int = 5):
    """max |Delta r_{0..t_c}| after replacing v_j, g_j for j > t_c, at three cuts."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    ref_scale = float(np.abs(as_f32(r0, w.dtype) if w.dtype != "i32" else r0).max()) or 1.0
    for t_c in (min(31, w.L - 2), w.L // 2, w.L - 2):
        v2, g2 = v.copy(), g.copy()
        if w.dtype == "i32":
            v2[:, t_c + 1:, :] = rng.integers(-128, 128, v2[:, t_c + 1:, :].shape)
            g2[:, t_c + 1:, :] = rng.integers(-128, 128, g2[:, t_c + 1:, :].shape)
        else:
            f = lambda shape: (1e4 * rng.standard_normal(shape)).astype(np.float32)  # noqa: E731
            v2[:, t_c + 1:, :] = f(v2[:, t_c + 1:, :].shape) if w.dtype == "f32" else \
                workloads.bf16_round(f(v2[:, t_c + 1:, :].shape))
            g2[:, t_c + 1:, :] = f(g2[:, t_c + 1:, :].shape) if w.dtype == "f32" else \
                workloads.bf16_round(f(g2[:, t_c + 1:, :].shape))
        r1 = run_gpu(v2, g2, w.dtype)
        a = r0[:, : t_c + 1, :] if w.dtype == "i32" else as_f32(r0[:, : t_c + 1, :], w.dtype)
        b = r1[:, : t_c + 1, :] if w.dtype == "i32" else as_f32(r1[:, : t_c + 1, :], w.dtype)
        leak = float(np.abs(b.astype(np.float64) - a.astype(np.float64)).max())
        out[str(t_c)] = {"max_abs": leak, "relative_to_max_r": leak / ref_scale}
    return out


def report(name: str, n_points: int):
    w = workloads.WORKLOADS[name]
    v, g = workloads.generate(w)
    t0 = time.perf_counter()
    r = run_gpu(v, g, w.dtype)
    line = {"workload": name, "shape": [w.B, w.L, w.D], "io_dtype": w.dtype,
            "path": "ntt" if w.dtype == "i32" else "fft"}
    line["accuracy"] = accuracy(w, v, g, r, n_points)
    line["leakage"] = leakage(w, v, g, r)
    line["seconds"] = round(time.perf_counter() - t0, 1)
    return line


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default=",".join(workloads.WORKLOADS))
    ap.add_argument("--points", type=int, default=4096)
    args = ap.parse_args(argv)
    lines = []
    for name in args.workloads.split(","):
        line = report(name, args.points)
        print(json.dumps(line), flush=True)
        lines.append(line)
    return lines


if __name__ == "__main__":
    main()
