"""Parity of the MHF gate stream (tcgen05 tensor-core kernel) and of the gated
convolution with the oracle (oracle/mhf_gate.py), through the C ABI.

Bounds, from the arithmetic (the gate's contraction is fp32-exact up to the
fp16 hi/lo split, whose dropped lo*lo term and rounded lo parts stay below
2^-21 of |w| sigmoid(a) per term, and sigmoid is evaluated in fp32):
  gate, fp32 I/O:   |g - g_ref| <= 1e-5 * gabs,  gabs = |bias| + sum |w| sigmoid(a)
  gate, bf16 I/O:   |g - g_ref| <= 2e-2 * gabs   (g rounded to bf16: <= 2^-9 gabs)
  gated conv:       |r - r_ref| <= tol * sum_j |v_j| gabs_{t-j},  tol 1e-5 / 2e-2
"""
import numpy as np
import pytest

import oracle
import oracle.mhf_gate as mhf
import workloads
from conftest import cuda_available
from gpu_helpers import BF16_TOL, F32_TOL, as_f32, float_violations, from_dev, run_gpu_gate, run_gpu_gated_conv, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA GPU")]

# (B, L, D, H, K): ragged last tiles (L % 128 != 0), one-step rows, every head
# width (16, 32, 64) and tap count, more heads than SMs (200 x 16)
GATE_SHAPES = [(1, 1, 16, 1, 1), (1, 5, 32, 2, 3), (2, 130, 64, 1, 3), (3, 200, 96, 3, 2), (1, 129, 48, 3, 4),
               (2, 300, 128, 2, 1), (1, 1024, 768, 12, 3), (2, 257, 64, 4, 4), (1, 2000, 64, 1, 3),
               (1, 64, 1024, 64, 2), (1, 40, 3200, 200, 1), (1, 127, 64, 1, 4)]
_ids = lambda s: "x".join(map(str, s))  # noqa: E731


def _inputs(shape, dtype, seed):
    B, L, D, H, K = shape
    return workloads.generate_gate(B, L, D, H, K, dtype, seed)


@pytest.mark.parametrize("shape", GATE_SHAPES, ids=_ids)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_parity(dtype, shape):
    B, L, D, H, K = shape
    _, a, w, bias = _inputs(shape, dtype, seed=sum(shape))
    g = run_gpu_gate(a, w, bias, H, dtype)
    g_ref, gabs = mhf.mhf_gate(as_f32(a, dtype), w, bias, H)
    tol = F32_TOL if dtype == "f32" else BF16_TOL
    n_bad, worst = float_violations(as_f32(g, dtype), g_ref, gabs, tol)
    assert n_bad == 0, f"{n_bad} gate outputs beyond the bound, worst ratio {worst:.3g}"
    if dtype == "f32":  # the split contraction stays well inside the bound (worst case 3 * 2^-20)
        assert worst < 0.5, worst


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_without_bias(dtype):
    shape = (2, 200, 128, 4, 3)
    _, a, w, _ = _inputs(shape, dtype, seed=3)
    g = run_gpu_gate(a, w, None, 4, dtype)
    g_ref, gabs = mhf.mhf_gate(as_f32(a, dtype), w, None, 4)
    n_bad, worst = float_violations(as_f32(g, dtype), g_ref, gabs, F32_TOL if dtype == "f32" else BF16_TOL)
    assert n_bad == 0, worst


def test_gate_saturated_and_exact_inputs():
    """a = +-60 drives sigmoid to exactly 1 and (nearly) 0; a = 0 gives 1/2;
    w a power of two: g is exact in fp32 and must match bit for bit."""
    B, L, D, H, K = 1, 150, 64, 1, 2
    a = np.zeros((B, L, D), np.float32)
    a[:, ::3] = 60.0
    a[:, 1::3] = -60.0
    w = np.zeros((D, D, K), np.float32)
    w[:, :, 1] = 0.25
    w[:, :, 0] = -0.5
    bias = np.full(D, 0.125, np.float32)
    g = run_gpu_gate(a, w, bias, H, "f32")
    g_ref, gabs = mhf.mhf_gate(a, w, bias, H)
    n_bad, worst = float_violations(g, g_ref, gabs, F32_TOL)
    assert n_bad == 0, worst
    exact = (a[0, :, 0] == 0.0) | (a[0, :, 0] == 60.0)
    prev_exact = np.concatenate([[True], exact[:-1]])
    both = exact & prev_exact
    assert np.array_equal(g[0, both], g_ref[0, both].astype(np.float32))


@pytest.mark.parametrize("shape", [(2, 130, 64, 1, 3), (3, 200, 96, 3, 2), (2, 1024, 768, 12, 3), (1, 33, 16, 1, 4)],
                         ids=_ids)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gated_conv_parity_full_oracle(dtype, shape):
    B, L, D, H, K = shape
    v, a, w, bias = _inputs(shape, dtype, seed=11 + sum(shape))
    r = run_gpu_gated_conv(v, a, w, bias, H, dtype)
    r_ref, den = mhf.mhf_gated_conv(as_f32(v, dtype), as_f32(a, dtype), w, bias, H)
    n_bad, worst = float_violations(as_f32(r, dtype), r_ref, den, F32_TOL if dtype == "f32" else BF16_TOL)
    assert n_bad == 0, f"{n_bad} outputs beyond the bound, worst ratio {worst:.3g}"


def test_gated_conv_full_workload_sampled():
    """The benchmarked workload (mhf_small_f32): the whole gate against the
    oracle, and the convolution on a stratified sample of outputs."""
    w_ = workloads.GATE_WORKLOADS["mhf_small_f32"]
    v, a, w, bias = workloads.generate_gate(w_.B, w_.L, w_.D, w_.H, w_.K, w_.dtype, w_.seed)
    g = run_gpu_gate(a, w, bias, w_.H, "f32")
    g_ref, gabs = mhf.mhf_gate(a, w, bias, w_.H)
    n_bad, worst = float_violations(g, g_ref, gabs, F32_TOL)
    assert n_bad == 0 and worst < 0.5, worst
    r = run_gpu_gated_conv(v, a, w, bias, w_.H, "f32")
    pts = workloads.sample_points(w_.B, w_.L, w_.D, 4096, seed=21)
    r_ref, _ = oracle.causal_conv_points(v.astype(np.float64), g_ref, pts)
    den, _ = oracle.causal_conv_points(np.abs(v).astype(np.float64), gabs, pts)
    got = r[pts[:, 0], pts[:, 1], pts[:, 2]]
    n_bad, worst = float_violations(got, r_ref, den, F32_TOL)
    assert n_bad == 0, f"{n_bad} sampled outputs beyond the bound, worst ratio {worst:.3g}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_unaligned_pointers(dtype):
    """a and g starting one element past an allocation: no vector loads/stores."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D, H, K = 2, 200, 64, 2, 3
    _, a, w, bias = _inputs((B, L, D, H, K), dtype, seed=5)
    flat = to_dev(a, dtype).reshape(-1)
    buf = torch.empty(flat.numel() + 1, dtype=flat.dtype, device="cuda")
    buf[1:] = flat
    ta = buf[1:].view(B, L, D)
    out_buf = torch.empty_like(buf)
    tg = out_buf[1:].view(B, L, D)
    ssm.mhf_gate(ta, torch.from_numpy(w).cuda(), torch.from_numpy(bias).cuda(), H, out=tg)
    torch.cuda.synchronize()
    g = from_dev(tg.contiguous(), dtype)
    g_ref, gabs = mhf.mhf_gate(as_f32(a, dtype), w, bias, H)
    n_bad, worst = float_violations(as_f32(g, dtype), g_ref, gabs, F32_TOL if dtype == "f32" else BF16_TOL)
    assert n_bad == 0, worst


def test_gate_errors():
    import torch
    import spectral_sequence_mixing_b200 as ssm
    from spectral_sequence_mixing_b200 import CausalConvError
    from spectral_sequence_mixing_b200._lib import CC_ERR_ALIAS, CC_ERR_UNSUPPORTED, CC_ERR_WORKSPACE
    a = torch.zeros(1, 8, 96, device="cuda")
    with pytest.raises(CausalConvError) as e:  # head width 48
        ssm.mhf_gate(a, torch.zeros(96, 48, 1, device="cuda"), None, 2)
    assert e.value.status == CC_ERR_UNSUPPORTED
    with pytest.raises(CausalConvError) as e:  # 5 taps
        ssm.mhf_gate(a, torch.zeros(96, 32, 5, device="cuda"), None, 3)
    assert e.value.status == CC_ERR_UNSUPPORTED
    with pytest.raises(CausalConvError) as e:  # output = input
        ssm.mhf_gate(a, torch.zeros(96, 32, 1, device="cuda"), None, 3, out=a)
    assert e.value.status == CC_ERR_ALIAS
    v = torch.zeros_like(a)
    with pytest.raises(CausalConvError) as e:
        ssm.mhf_gated_conv(v, a, torch.zeros(96, 32, 1, device="cuda"), None, 3,
                           workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == CC_ERR_WORKSPACE
    assert ssm.fault_flags() == 0
