"""Parity of the causal depthwise convolution kernel with the oracle
(oracle/mhf_dwconv.py), through the C ABI.

Bound, from the arithmetic (K fused multiply-adds in fp32): |y - y_ref| <=
1e-6 * yabs with yabs = |bias| + sum |w| |x| for fp32 I/O, and 2^-8 * yabs for
bf16 I/O, where y is rounded to bf16 (2^-9 relative).
"""
import numpy as np
import pytest

import oracle.mhf_dwconv as dw
import workloads
from conftest import cuda_available
from gpu_helpers import as_f32, float_violations, from_dev, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA GPU")]

F32_DW_TOL = 1e-6
BF16_DW_TOL = 2.0 ** -8

# (B, L, D, K): runs with ragged tails (L % 16 != 0), L shorter than the taps,
# D not a multiple of 4 (scalar path), every K, a long row beyond any transform length
SHAPES = [(1, 1, 4, 3), (1, 2, 8, 4), (2, 17, 12, 3), (3, 100, 36, 3), (1, 1024, 768, 3), (2, 33, 7, 2),
          (1, 50, 5, 8), (2, 257, 64, 1), (1, 70000, 8, 3), (4, 31, 1536, 5)]
_ids = lambda s: "x".join(map(str, s))  # noqa: E731


def _run(x, w, bias, dtype, out_offset=0):
    import torch
    import spectral_sequence_mixing_b200 as ssm
    tx = to_dev(x, dtype)
    tb = None if bias is None else torch.from_numpy(bias).cuda()
    if out_offset:
        buf = torch.empty(tx.numel() + out_offset, dtype=tx.dtype, device="cuda")
        out = buf[out_offset:].view(tx.shape)
        ssm.causal_dwconv(tx, torch.from_numpy(w).cuda(), tb, out=out)
        y = out.contiguous()
    else:
        y = ssm.causal_dwconv(tx, torch.from_numpy(w).cuda(), tb)
    torch.cuda.synchronize()
    return from_dev(y, dtype)


@pytest.mark.parametrize("shape", SHAPES, ids=_ids)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dwconv_parity(dtype, shape):
    B, L, D, K = shape
    x, w, bias = workloads.generate_dwconv(B, L, D, K, dtype, seed=sum(shape))
    y = _run(x, w, bias, dtype)
    y_ref, yabs = dw.causal_dwconv(as_f32(x, dtype), w, bias)
    n_bad, worst = float_violations(as_f32(y, dtype), y_ref, yabs, F32_DW_TOL if dtype == "f32" else BF16_DW_TOL)
    assert n_bad == 0, f"{n_bad} outputs beyond the bound, worst ratio {worst:.3g}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dwconv_no_bias_and_unaligned_output(dtype):
    B, L, D, K = 2, 300, 64, 3
    x, w, _ = workloads.generate_dwconv(B, L, D, K, dtype, seed=3)
    y = _run(x, w, None, dtype, out_offset=1)   # misaligned y: the scalar path
    y_ref, yabs = dw.causal_dwconv(as_f32(x, dtype), w, None)
    n_bad, worst = float_violations(as_f32(y, dtype), y_ref, yabs, F32_DW_TOL if dtype == "f32" else BF16_DW_TOL)
    assert n_bad == 0, worst


def test_dwconv_exact_small_integers():
    """Integer-valued x, w, bias: every sum is exact in fp32, so y matches bit for bit."""
    B, L, D, K = 2, 70, 16, 3
    rng = np.random.Generator(np.random.PCG64(4))
    x = rng.integers(-8, 9, (B, L, D)).astype(np.float32)
    w = rng.integers(-4, 5, (D, K)).astype(np.float32)
    bias = rng.integers(-3, 4, D).astype(np.float32)
    y = _run(x, w, bias, "f32")
    y_ref, _ = dw.causal_dwconv(x, w, bias)
    assert np.array_equal(y, y_ref.astype(np.float32))


def test_dwconv_workload_full():
    wl = workloads.DWCONV_WORKLOADS["dwconv_small_f32"]
    x, w, bias = workloads.generate_dwconv(wl.B, wl.L, wl.D, wl.K, wl.dtype, wl.seed)
    y = _run(x, w, bias, "f32")
    y_ref, yabs = dw.causal_dwconv(x, w, bias)
    n_bad, worst = float_violations(y, y_ref, yabs, F32_DW_TOL)
    assert n_bad == 0, worst


def test_dwconv_errors():
    import torch
    import spectral_sequence_mixing_b200 as ssm
    from spectral_sequence_mixing_b200 import CausalConvError
    from spectral_sequence_mixing_b200._lib import CC_ERR_ALIAS, CC_ERR_UNSUPPORTED
    x = torch.zeros(1, 8, 16, device="cuda")
    with pytest.raises(CausalConvError) as e:
        ssm.causal_dwconv(x, torch.zeros(16, 9, device="cuda"))
    assert e.value.status == CC_ERR_UNSUPPORTED
    with pytest.raises(CausalConvError) as e:
        ssm.causal_dwconv(x, torch.zeros(16, 3, device="cuda"), out=x)
    assert e.value.status == CC_ERR_ALIAS
