"""Shared helpers for the GPU parity tests: move seeded numpy inputs to the
device, run the C-ABI path through the binding, and compare with the oracle."""
from __future__ import annotations

import numpy as np

import workloads

F32_TOL = 1e-5     # |r - r_ref| <= F32_TOL * sum_j |v_j g_{t-j}|  (fp32 I/O)
BF16_TOL = 2e-2    # same bound scaled by 2e-2 (bf16 I/O, fp32 arithmetic)


def to_dev(x: np.ndarray, dtype: str):
    import torch
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, np.int32)).cuda()


def from_dev(t, dtype: str) -> np.ndarray:
    import torch
    if dtype == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def run_gpu(v: np.ndarray, g: np.ndarray, dtype: str) -> np.ndarray:
    import torch
    import spectral_sequence_mixing_b200 as ssm
    tv, tg = to_dev(v, dtype), to_dev(g, dtype)
    fn = {"f32": ssm.causal_fftconv_f32, "bf16": ssm.causal_fftconv_bf16, "i32": ssm.causal_ntt_conv_i32}[dtype]
    r = fn(tv, tg)
    torch.cuda.synchronize()
    return from_dev(r, dtype)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """The exact float32 values the kernel sees."""
    return workloads.bf16_to_f32(x) if dtype == "bf16" else np.asarray(x, np.float32)


def float_violations(r_gpu, r_ref, den, tol, floor=0.0):
    """Elements breaking |r_gpu - r_ref| <= tol * den + floor; returns
    (count, worst ratio err / (tol*den + floor))."""
    err = np.abs(np.asarray(r_gpu, np.float64) - r_ref)
    bound = tol * den + floor
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    return int((err > bound).sum()), float(ratio.max() if ratio.size else 0.0)


def run_gpu_bwd(dr, v, g, dtype: str):
    import torch
    import spectral_sequence_mixing_b200 as ssm
    dv, dg = ssm.causal_conv_bwd(to_dev(dr, dtype), to_dev(v, dtype), to_dev(g, dtype))
    torch.cuda.synchronize()
    return from_dev(dv, dtype), from_dev(dg, dtype)


def run_gpu_gate(a: np.ndarray, w: np.ndarray, bias, n_head: int, dtype: str) -> np.ndarray:
    import torch
    import spectral_sequence_mixing_b200 as ssm
    tb = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias, np.float32)).cuda()
    g = ssm.mhf_gate(to_dev(a, dtype), torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda(), tb, n_head)
    torch.cuda.synchronize()
    return from_dev(g, dtype)


def run_gpu_gated_conv(v: np.ndarray, a: np.ndarray, w: np.ndarray, bias, n_head: int, dtype: str) -> np.ndarray:
    import torch
    import spectral_sequence_mixing_b200 as ssm
    tb = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias, np.float32)).cuda()
    r = ssm.mhf_gated_conv(to_dev(v, dtype), to_dev(a, dtype),
                           torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda(), tb, n_head)
    torch.cuda.synchronize()
    return from_dev(r, dtype)
