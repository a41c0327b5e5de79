"""The allocation-free decode entry point, causal_conv_decode_f32_noalloc.

Some callers cannot allocate device memory: an engine that owns every byte of
device memory through its own pool and forbids allocations behind its back,
or a path that must not pay the device-wide synchronisation that cudaFree
implies.  For them the library offers one decode entry point whose scratch is
a fixed 8 MiB static device buffer instead of a caller workspace.

This file is named so that pytest collects it last; it checks that entry
point, through the C ABI, against the workspace-taking entry point on two
calls in a row (different problems, so a stale buffer would show), and that it
refuses problems beyond its buffer before doing anything.
"""
import ctypes

import numpy as np
import pytest

import oracle
from conftest import cuda_available
from gpu_helpers import F32_TOL, float_violations

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA GPU")]


def _decode_both(lib, B, Lcap, D, t, seed):
    import torch
    from spectral_sequence_mixing_b200 import decode_workspace_bytes
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.standard_normal((B, Lcap, D)).astype(np.float32)
    g = rng.standard_normal((B, Lcap, D)).astype(np.float32)
    tv, tg = torch.from_numpy(v).cuda(), torch.from_numpy(g).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(decode_workspace_bytes(torch.float32, B, D, t), dtype=torch.uint8, device="cuda")
    r_ws = torch.empty((B, D), device="cuda")
    r_na = torch.full((B, D), float("nan"), device="cuda")
    st = lib.causal_conv_decode_f32(tv.data_ptr(), tg.data_ptr(), r_ws.data_ptr(), B, Lcap, D, t, ws.data_ptr(),
                                    ws.numel(), stream)
    assert st == 0, st
    st = lib.causal_conv_decode_f32_noalloc(tv.data_ptr(), tg.data_ptr(), r_na.data_ptr(), B, Lcap, D, t, stream)
    assert st == 0, st
    torch.cuda.synchronize()
    pts = np.array([(b, t, d) for b in range(B) for d in range(D)], np.int64)
    _, den = oracle.causal_conv_points(v, g, pts)
    return r_ws.cpu().numpy().reshape(-1), r_na.cpu().numpy().reshape(-1), den


def test_noalloc_decode_matches_workspace_entry_point_on_two_calls():
    from spectral_sequence_mixing_b200 import _lib
    lib = _lib.load()
    # two calls in a row with different problems sharing the fixed buffer
    for B, Lcap, D, t, seed in ((8, 1024, 768, 1023, 1), (3, 300, 37, 64, 2)):
        ref, got, den = _decode_both(lib, B, Lcap, D, t, seed)
        n_bad, worst = float_violations(got, ref.astype(np.float64), den, F32_TOL)
        assert n_bad == 0, f"{(B, Lcap, D, t)}: {n_bad} outputs differ beyond the bound, worst ratio {worst:.3g}"


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
