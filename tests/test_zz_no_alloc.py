"""The allocation-free decode entry point, causal_conv_decode_f32_noalloc.

Some callers cannot allocate device memory: an engine that owns every byte of
device memory through its own pool and forbids allocations behind its back,
or a path that must not pay the device-wide synchronisation that cudaFree
implies.  For them the library offers one decode entry point whose scratch is
a fixed 8 MiB static device buffer instead of a caller workspace.

This file is named so that pytest collects it last.  Through the C ABI it
checks, on two calls in a row with different problems (a stale buffer would
show):
  * that the entry point returns the workspace-taking entry point's result
    bit for bit (both run the same fixed-order reduction);
  * that its result is within the fp32 bound of the oracle's exact sum;
  * that a call after the first one reserves no device memory;
and that it refuses problems beyond its buffer before doing anything.
"""
import numpy as np
import pytest

import oracle
from conftest import cuda_available
from gpu_helpers import F32_TOL, float_violations

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA GPU")]


def _inputs(B, Lcap, D, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.standard_normal((B, Lcap, D)).astype(np.float32)
    g = rng.standard_normal((B, Lcap, D)).astype(np.float32)
    return v, g


def _call_noalloc(lib, tv, tg, out, B, Lcap, D, t, stream):
    st = lib.causal_conv_decode_f32_noalloc(tv.data_ptr(), tg.data_ptr(), out.data_ptr(), B, Lcap, D, t, stream)
    assert st == 0, st


def test_noalloc_decode_matches_workspace_entry_point_and_oracle_on_two_calls():
    import torch
    from spectral_sequence_mixing_b200 import _lib, decode_workspace_bytes
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row with different problems sharing the fixed buffer
    for B, Lcap, D, t, seed in ((8, 1024, 768, 1023, 1), (3, 300, 37, 64, 2)):
        v, g = _inputs(B, Lcap, D, seed)
        tv, tg = torch.from_numpy(v).cuda(), torch.from_numpy(g).cuda()
        ws = torch.empty(decode_workspace_bytes(torch.float32, B, D, t), dtype=torch.uint8, device="cuda")
        r_ws = torch.empty((B, D), device="cuda")
        r_na = torch.full((B, D), float("nan"), device="cuda")
        st = lib.causal_conv_decode_f32(tv.data_ptr(), tg.data_ptr(), r_ws.data_ptr(), B, Lcap, D, t,
                                        ws.data_ptr(), ws.numel(), stream)
        assert st == 0, st
        _call_noalloc(lib, tv, tg, r_na, B, Lcap, D, t, stream)
        torch.cuda.synchronize()
        got = r_na.cpu().numpy().reshape(-1)
        same = r_ws.cpu().numpy().reshape(-1)
        # same kernels, same fixed summation order: identical bits
        assert np.array_equal(got.view(np.uint32), same.view(np.uint32)), \
            f"{(B, Lcap, D, t)}: the no-allocation result differs from the workspace entry point's"
        pts = np.array([(b, t, d) for b in range(B) for d in range(D)], np.int64)
        ref, den = oracle.causal_conv_points(v, g, pts)
        n_bad, worst = float_violations(got, ref, den, F32_TOL)
        assert n_bad == 0, f"{(B, Lcap, D, t)}: {n_bad} outputs beyond the oracle bound, worst ratio {worst:.3g}"


def test_noalloc_call_reserves_no_device_memory():
    import torch
    from spectral_sequence_mixing_b200 import _lib
    lib = _lib.load()
    B, Lcap, D, t = 4, 512, 256, 511
    v, g = _inputs(B, Lcap, D, 3)
    tv, tg = torch.from_numpy(v).cuda(), torch.from_numpy(g).cuda()
    out = torch.empty((B, D), device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    _call_noalloc(lib, tv, tg, out, B, Lcap, D, t, stream)  # warm-up: loads the module, looks the buffer up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        _call_noalloc(lib, tv, tg, out, B, Lcap, D, t, stream)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes across the calls"
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_refuses_problems_beyond_its_buffer():
    import torch
    from spectral_sequence_mixing_b200 import _lib
    lib = _lib.load()
    x = torch.zeros(4, device="cuda")
    y = torch.zeros(4, device="cuda")
    r = torch.zeros(4, device="cuda")
    D = 1 << 21  # one position, 2M channels: 16 MiB of partial sums > 8 MiB
    need = lib.causal_conv_decode_workspace_bytes(0, 1, D, 0)
    assert need > 8 << 20
    st = lib.causal_conv_decode_f32_noalloc(x.data_ptr(), y.data_ptr(), r.data_ptr(), 1, 1, D, 0, None)
    assert st == _lib.CC_ERR_SCRATCH_LIMIT
    assert "8 MiB" in _lib.strerror(st)
