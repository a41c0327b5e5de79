"""Parity of the sm_100a kernels (through the C ABI) with the CPU oracle.

Float paths: |r_gpu - r_ref| <= 1e-5 * sum_j |v_j g_{t-j}| per element (fp32
I/O) or 2e-2 of that (bf16 I/O), on the seeded workloads.  Integer path:
bit-exact.  The oracle computes the plain definition
r_t = sum_{j<=t} v_j g_{t-j} (Caracal, key designs 1 and 2).
"""
import numpy as np
import pytest

import oracle
import workloads
from conftest import cuda_available
from gpu_helpers import BF16_TOL, F32_TOL, as_f32, float_violations, run_gpu, to_dev, from_dev

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA GPU")]

P = 2013265921


def _rand_float(shape, seed, scale_g=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    return (rng.standard_normal(shape).astype(np.float32),
            (scale_g * rng.standard_normal(shape)).astype(np.float32))


# shapes spanning several tiles with ragged tails in L (vs N/2) and D (vs the channel tile)
# (D * element size a multiple of 16 bytes selects the TMA staging: (3, 200, 36)
# and (2, 130, 24) end in a partial channel group the copy engine zero-fills,
# (1, 513, 4) and (2, 700, 20) have many zero-filled time steps past L; in
# bf16, (2, 1000, 16) and (1, 513, 8) stage 8-channel rows for 4-channel tiles)
FLOAT_SHAPES = [(1, 1, 1), (1, 2, 3), (1, 3, 2), (2, 31, 5), (1, 32, 4), (1, 33, 7), (3, 200, 19), (1, 256, 8),
                (2, 257, 9), (2, 513, 5), (2, 1000, 37), (1, 1024, 12), (3, 200, 36), (2, 130, 24), (1, 513, 4),
                (2, 700, 20), (2, 1000, 16), (1, 513, 8)]


@pytest.mark.parametrize("shape", FLOAT_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_f32_parity_full_oracle(shape):
    v, g = _rand_float(shape, seed=sum(shape))
    r = run_gpu(v, g, "f32")
    r_ref, den = oracle.causal_conv(v, g)
    n_bad, worst = float_violations(r, r_ref, den, F32_TOL)
    assert n_bad == 0, f"{n_bad} elements beyond the fp32 bound, worst ratio {worst:.3g}"


@pytest.mark.parametrize("shape", FLOAT_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bf16_parity_full_oracle(shape):
    v, g = _rand_float(shape, seed=7 + sum(shape), scale_g=0.125)
    vb, gb = workloads.bf16_round(v), workloads.bf16_round(g)
    r = run_gpu(vb, gb, "bf16")
    r_ref, den = oracle.causal_conv(as_f32(vb, "bf16"), as_f32(gb, "bf16"))
    n_bad, worst = float_violations(as_f32(r, "bf16"), r_ref, den, BF16_TOL)
    assert n_bad == 0, f"{n_bad} elements beyond the bf16 bound, worst ratio {worst:.3g}"


@pytest.mark.parametrize("shape", [(2, 300, 16), (1, 2000, 16)], ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unaligned_base_pointers(dtype, shape):
    """Tensors starting 4 (f32) or 2 (bf16) bytes past an allocation: no tensor
    map (fused kernel) and no 16-byte group access (channel-group clusters)
    can describe them, so element-wise paths run."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    v, g = _rand_float(shape, seed=99, scale_g=0.125)
    if dtype == "bf16":
        v, g = workloads.bf16_round(v), workloads.bf16_round(g)
    n = int(np.prod(shape))
    tv, tg = to_dev(v.reshape(-1), dtype), to_dev(g.reshape(-1), dtype)
    bv = torch.empty(n + 1, dtype=tv.dtype, device="cuda")
    bg = torch.empty(n + 1, dtype=tv.dtype, device="cuda")
    bv[1:] = tv
    bg[1:] = tg
    r = ssm.causal_conv(bv[1:].view(shape), bg[1:].view(shape))
    torch.cuda.synchronize()
    r_ref, den = oracle.causal_conv(as_f32(v, dtype), as_f32(g, dtype))
    n_bad, worst = float_violations(as_f32(from_dev(r, dtype), dtype), r_ref, den,
                                    F32_TOL if dtype == "f32" else BF16_TOL)
    assert n_bad == 0, f"{n_bad} elements beyond the bound, worst ratio {worst:.3g}"


def test_fast_workspace_must_not_overlap_tensors():
    import torch
    import spectral_sequence_mixing_b200 as ssm
    from spectral_sequence_mixing_b200._lib import CausalConvError
    B, L, D = 1, 5000, 4
    v = torch.randn(B, L, D, device="cuda")
    g = torch.randn(B, L, D, device="cuda")
    n = ssm.fast_workspace_bytes(torch.float32, B, L, D)
    big = torch.empty(n + v.numel() * 4, dtype=torch.uint8, device="cuda")
    out = big[:v.numel() * 4].view(torch.float32).view(B, L, D)  # r inside the workspace
    with pytest.raises(CausalConvError) as e:
        ssm.causal_conv(v, g, out=out, workspace=big)
    assert e.value.status == 3


def test_no_kernel_wait_ran_out():
    """Every bounded wait in the kernels completed during the tests so far."""
    import spectral_sequence_mixing_b200 as ssm
    v, g = _rand_float((4, 1024, 64), seed=5)
    run_gpu(v, g, "f32")
    assert ssm.fault_flags() == 0


# clusters of 4 adjacent channels: partial groups, and whole groups with
# 16-byte accesses (D = 8, 12)
INT_SHAPES = [(1, 1, 1), (1, 2, 3), (2, 33, 5), (2, 1000, 37), (1, 4097, 3), (1, 8192, 2), (2, 1000, 8),
              (1, 8192, 12), (3, 500, 6)]


@pytest.mark.parametrize("shape", INT_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_ntt_bit_exact(shape):
    rng = np.random.Generator(np.random.PCG64(sum(shape)))
    v = rng.integers(-128, 128, shape).astype(np.int32)
    g = rng.integers(-128, 128, shape).astype(np.int32)
    r = run_gpu(v, g, "i32")
    assert np.array_equal(r.astype(np.int64), oracle.causal_conv_int(v, g))


@pytest.mark.parametrize("case", ["all_min", "all_max", "min_max", "alternating"])
def test_ntt_extremes(case):
    B, L, D = 1, 8192, 3
    if case == "all_min":
        v = np.full((B, L, D), -128, np.int32); g = v.copy()
    elif case == "all_max":
        v = np.full((B, L, D), 127, np.int32); g = v.copy()
    elif case == "min_max":
        v = np.full((B, L, D), -128, np.int32); g = np.full((B, L, D), 127, np.int32)
    else:
        s = np.where(np.arange(L) % 2 == 0, 127, -128).astype(np.int32).reshape(1, L, 1)
        v = np.broadcast_to(s, (B, L, D)).copy(); g = -v
    r = run_gpu(v, g, "i32").astype(np.int64)
    ref = oracle.causal_conv_int(v, g)
    assert np.array_equal(r, ref)
    if case == "all_min":
        assert r[0, -1, 0] == 2 ** 27


def test_ntt_wraps_to_centered_residue():
    """Sums beyond (p-1)/2 come back as the centered residue mod p."""
    rng = np.random.Generator(np.random.PCG64(11))
    B, L, D = 1, 512, 4
    v = rng.integers(-2 ** 31, 2 ** 31, (B, L, D), dtype=np.int64).astype(np.int32)
    g = rng.integers(-2 ** 31, 2 ** 31, (B, L, D), dtype=np.int64).astype(np.int32)
    r = run_gpu(v, g, "i32").astype(np.int64)
    # exact sums mod p: residues < 2^31, each product < 2^62, reduced before summing
    vm = v.astype(np.int64) % P
    gm = g.astype(np.int64) % P
    ref = np.zeros((B, L, D), np.int64)
    for t in range(L):
        ref[:, t, :] = ((vm[:, : t + 1, :] * gm[:, t::-1, :]) % P).sum(axis=1) % P
    ref = oracle.centered_mod(ref, P)
    assert np.array_equal(r, ref)


# rows longer than one fused tile: one row per CTA (L <= 4096) or per 8-CTA cluster (L <= 65536)
# rows of one CTA run in clusters of 8 adjacent channels: partial groups
# (D < 8, D = 12), whole groups with 16-byte accesses (D = 16, 24)
BIG_SHAPES = [(1, 1025, 3), (2, 2000, 5), (1, 4096, 4), (1, 2000, 16), (2, 1500, 24), (1, 4096, 12)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", BIG_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_big_rows_full_oracle(shape, dtype):
    v, g = _rand_float(shape, seed=100 + sum(shape), scale_g=0.125 if dtype == "bf16" else 1.0)
    if dtype == "bf16":
        v, g = workloads.bf16_round(v), workloads.bf16_round(g)
    r = run_gpu(v, g, dtype)
    r_ref, den = oracle.causal_conv(as_f32(v, dtype), as_f32(g, dtype))
    n_bad, worst = float_violations(as_f32(r, dtype) if dtype == "bf16" else r, r_ref, den,
                                    F32_TOL if dtype == "f32" else BF16_TOL)
    assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"


CLUSTER_SHAPES = [(1, 4097, 3), (2, 20000, 2), (1, 65536, 2), (2, 5000, 33)]


@pytest.mark.parametrize("two_pass", [True, False], ids=["two_pass", "single_pass"])
@pytest.mark.parametrize("shape", CLUSTER_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_cluster_rows_sampled_oracle(shape, two_pass):
    """Rows beyond one CTA: with the optional workspace (the four-step path)
    and without it (8-CTA cluster rows read straight from the channel-last
    tensors)."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = shape
    rng = np.random.Generator(np.random.PCG64(sum(shape)))
    v = rng.standard_normal(shape).astype(np.float32)
    g = (rng.standard_normal(shape) * (1.0 + np.arange(L).reshape(1, L, 1)) ** -0.75).astype(np.float32)
    n_ws = ssm.fast_workspace_bytes(torch.float32, B, L, D) if two_pass else 0
    assert (n_ws > 0) == two_pass
    ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
    r = ssm.causal_conv(to_dev(v, "f32"), to_dev(g, "f32"), workspace=ws)
    torch.cuda.synchronize()
    r = from_dev(r, "f32")
    pts = workloads.sample_points(B, L, D, 1024, seed=7)
    r_ref, den = oracle.causal_conv_points(v, g, pts)
    n_bad, worst = float_violations(r[pts[:, 0], pts[:, 1], pts[:, 2]], r_ref, den, F32_TOL)
    assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"


# Four-step shapes: ragged channel tiles ((3, 5000, 50), (5, 4097, 27)), a
# partial mid-pass group of rows ((1, 8192, 130), (16, 4100, 9) with 144
# rows), L past several 512-step columns and ragged in them; rows whose
# D * element size is a multiple of 16 bytes take the TMA forward pass and the
# 16-byte norm loads: (2, 6000, 72) (two batches, a partial 16-channel tile, a
# ragged last 512-step row read directly), (3, 4608, 20) (L a whole number of
# 512-step rows), (1, 8192, 40), (2, 65536, 16) (the longest rows, two batches).
FOUR_STEP_SHAPES = [(3, 5000, 50), (1, 8192, 130), (5, 4097, 27), (16, 4100, 9), (2, 6000, 72), (3, 4608, 20),
                    (1, 8192, 40), (2, 65536, 16)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", FOUR_STEP_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_cluster_rows_four_step_and_single_pass(shape, dtype):
    """The four-step path (workspace) and the single-pass cluster rows (no
    workspace) against the oracle on sampled outputs, fp32 and bf16."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = shape
    rng = np.random.Generator(np.random.PCG64(11 + sum(shape)))
    v = rng.standard_normal(shape).astype(np.float32)
    g = (rng.standard_normal(shape) * (1.0 + np.arange(L).reshape(1, L, 1)) ** -0.75).astype(np.float32)
    if dtype == "bf16":
        v, g = workloads.bf16_round(v), workloads.bf16_round(g)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    ws = torch.empty(ssm.fast_workspace_bytes(tdt, B, L, D), dtype=torch.uint8, device="cuda")
    vd, gd = to_dev(v, dtype), to_dev(g, dtype)
    r4 = ssm.causal_conv(vd, gd, workspace=ws)
    r1 = ssm.causal_conv(vd, gd, workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    pts = workloads.sample_points(B, L, D, 1024, seed=17)
    r_ref, den = oracle.causal_conv_points(as_f32(v, dtype), as_f32(g, dtype), pts)
    tol = F32_TOL if dtype == "f32" else BF16_TOL
    for r in (r4, r1):
        got = as_f32(from_dev(r, dtype), dtype) if dtype == "bf16" else from_dev(r, dtype)
        n_bad, worst = float_violations(got[pts[:, 0], pts[:, 1], pts[:, 2]], r_ref, den, tol)
        assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"


def test_four_step_misaligned_workspace_and_inputs():
    """A workspace that is not 16-byte aligned selects the single-pass path;
    inputs at a 4-byte offset (no tensor map) take the direct-load forward
    pass and the per-channel norm loads; both agree with the oracle."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = 1, 5000, 64
    rng = np.random.Generator(np.random.PCG64(77))
    v = rng.standard_normal((B, L, D)).astype(np.float32)
    g = (rng.standard_normal((B, L, D)) * (1.0 + np.arange(L).reshape(1, L, 1)) ** -0.75).astype(np.float32)
    n_ws = ssm.fast_workspace_bytes(torch.float32, B, L, D)
    big = torch.empty(n_ws + 64, dtype=torch.uint8, device="cuda")
    pts = workloads.sample_points(B, L, D, 1024, seed=19)
    r_ref, den = oracle.causal_conv_points(v, g, pts)
    vd, gd = to_dev(v, "f32"), to_dev(g, "f32")
    # unaligned inputs: the same values one float past a 16-byte boundary
    vbuf = torch.empty(v.size + 1, dtype=torch.float32, device="cuda")
    gbuf = torch.empty(v.size + 1, dtype=torch.float32, device="cuda")
    vu = vbuf[1:].view(B, L, D)
    gu = gbuf[1:].view(B, L, D)
    vu.copy_(vd)
    gu.copy_(gd)
    outs = [ssm.causal_conv(vd, gd, workspace=big[8:8 + n_ws]),      # misaligned workspace: single pass
            ssm.causal_conv(vu, gu, workspace=big[:n_ws]),          # four-step, direct loads
            ssm.causal_conv(vd, gd, workspace=big[:n_ws])]          # four-step, TMA forward pass
    torch.cuda.synchronize()
    for r in outs:
        got = from_dev(r, "f32")
        n_bad, worst = float_violations(got[pts[:, 0], pts[:, 1], pts[:, 2]], r_ref, den, F32_TOL)
        assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"


@pytest.mark.parametrize("scale", [1e-4, 1e4])
def test_four_step_imbalanced_streams(scale):
    """Streams whose norms differ by ~1e8 share one complex transform only
    after the per-row power-of-two balance (norm pass and alpha): the
    four-step path still meets the per-element bound on sampled outputs."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = 2, 5000, 16
    rng = np.random.Generator(np.random.PCG64(int(1 / scale) % 1000 + 3))
    v = (rng.standard_normal((B, L, D)) / scale).astype(np.float32)
    g = (rng.standard_normal((B, L, D)) * scale * (1.0 + np.arange(L).reshape(1, L, 1)) ** -0.75).astype(np.float32)
    ws = torch.empty(ssm.fast_workspace_bytes(torch.float32, B, L, D), dtype=torch.uint8, device="cuda")
    r = ssm.causal_conv(to_dev(v, "f32"), to_dev(g, "f32"), workspace=ws)
    torch.cuda.synchronize()
    r = from_dev(r, "f32")
    pts = workloads.sample_points(B, L, D, 1024, seed=23)
    r_ref, den = oracle.causal_conv_points(v, g, pts)
    n_bad, worst = float_violations(r[pts[:, 0], pts[:, 1], pts[:, 2]], r_ref, den, F32_TOL)
    assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"


def test_internal_workspace_on_a_side_stream_and_when_memory_is_short(monkeypatch):
    """Long rows with no workspace given: the binding takes one from the torch
    allocator and, when the call runs on another stream, records that stream
    on it (and on the output it allocates), so memory freed on return is not
    reused by the current stream while the call's kernels still run; when the
    allocator has no room for the four-step workspace the single-pass path
    runs instead.  Both agree with the oracle."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = 1, 6000, 32
    rng = np.random.Generator(np.random.PCG64(41))
    v = rng.standard_normal((B, L, D)).astype(np.float32)
    g = (rng.standard_normal((B, L, D)) * (1.0 + np.arange(L).reshape(1, L, 1)) ** -0.75).astype(np.float32)
    vd, gd = to_dev(v, "f32"), to_dev(g, "f32")
    pts = workloads.sample_points(B, L, D, 1024, seed=29)
    r_ref, den = oracle.causal_conv_points(v, g, pts)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    r_side = ssm.causal_conv(vd, gd, stream=s)  # workspace and output allocated here, used on s
    # fresh allocations on the current stream meanwhile, written at once
    junk = [torch.full((1 << 22,), 7.0, device="cuda") for _ in range(64)]
    s.synchronize()
    torch.cuda.synchronize()
    del junk
    real_empty = torch.empty

    def empty_or_oom(*args, **kw):
        if kw.get("dtype") is torch.uint8 and args and int(args[0]) > (1 << 24):
            raise torch.cuda.OutOfMemoryError("no room for the workspace")
        return real_empty(*args, **kw)
    monkeypatch.setattr(ssm.torch, "empty", empty_or_oom)
    r_short = ssm.causal_conv(vd, gd)  # single-pass path
    torch.cuda.synchronize()
    for r in (r_side, r_short):
        got = from_dev(r, "f32")
        n_bad, worst = float_violations(got[pts[:, 0], pts[:, 1], pts[:, 2]], r_ref, den, F32_TOL)
        assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"


def test_four_step_capture_side_stream_and_zero_rows():
    """The four-step path on a caller's side stream and replayed from a CUDA
    graph equals the eager default-stream call bit for bit (forward and the
    backward's time-reversed reads and writes); rows whose v or g is all zero
    come out exactly zero."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = 2, 6000, 72
    rng = np.random.Generator(np.random.PCG64(31))
    dr, v, g = (to_dev(rng.standard_normal((B, L, D)).astype(np.float32), "f32") for _ in range(3))
    v[0, :, 5] = 0.0
    g[1, :, 70] = 0.0
    ws = torch.empty(ssm.fast_workspace_bytes(torch.float32, B, L, D), dtype=torch.uint8, device="cuda")
    ref_dv, ref_dg = ssm.causal_conv_bwd(dr, v, g, workspace=ws)
    ref_r = ssm.causal_conv(v, g, workspace=ws)
    torch.cuda.synchronize()
    assert not ref_r[0, :, 5].any() and not ref_r[1, :, 70].any()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    dv, dg, r = torch.empty_like(dr), torch.empty_like(dr), torch.empty_like(dr)
    with torch.cuda.stream(s):
        ssm.causal_conv_bwd(dr, v, g, dv=dv, dg=dg, workspace=ws, stream=s)
        ssm.causal_conv(v, g, out=r, workspace=ws, stream=s)
        cv, cg, cr = dv.clone(), dg.clone(), r.clone()  # consumers on the caller's stream
    s.synchronize()
    assert torch.equal(cv, ref_dv) and torch.equal(cg, ref_dg) and torch.equal(cr, ref_r)
    graph = torch.cuda.CUDAGraph()
    dv.zero_()
    dg.zero_()
    r.zero_()
    with torch.cuda.graph(graph):
        ssm.causal_conv_bwd(dr, v, g, dv=dv, dg=dg, workspace=ws, stream=torch.cuda.current_stream())
        ssm.causal_conv(v, g, out=r, workspace=ws, stream=torch.cuda.current_stream())
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(dv, ref_dv) and torch.equal(dg, ref_dg) and torch.equal(r, ref_r)


@pytest.mark.parametrize("name", ["large_bf16", "long_f32"])
def test_config_sampled_oracle(name):
    """Full-size workloads in the launch configuration the benchmark times,
    checked on a stratified sample of outputs."""
    w = workloads.WORKLOADS[name]
    v, g = workloads.generate(w)
    r = run_gpu(v, g, w.dtype)
    pts = workloads.sample_points(w.B, w.L, w.D, 4096, seed=1000 + list(workloads.WORKLOADS).index(name))
    r_ref, den = oracle.causal_conv_points(as_f32(v, w.dtype), as_f32(g, w.dtype), pts)
    got = as_f32(r, w.dtype)[pts[:, 0], pts[:, 1], pts[:, 2]] if w.dtype == "bf16" else r[pts[:, 0], pts[:, 1], pts[:, 2]]
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    n_bad, worst = float_violations(got, r_ref, den, tol)
    assert n_bad == 0, f"{name}: {n_bad} violations, worst ratio {worst:.3g}"


CONFIGS_FULL = ["tiny_f32", "small_f32"]


@pytest.mark.parametrize("name", CONFIGS_FULL)
def test_config_full_oracle(name):
    w = workloads.WORKLOADS[name]
    v, g = workloads.generate(w)
    r = run_gpu(v, g, w.dtype)
    r_ref, den = oracle.causal_conv(as_f32(v, w.dtype), as_f32(g, w.dtype))
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    n_bad, worst = float_violations(as_f32(r, w.dtype) if w.dtype == "bf16" else r, r_ref, den, tol)
    assert n_bad == 0, f"{name}: {n_bad} violations, worst ratio {worst:.3g}"


def test_config_ntt_full_bit_exact():
    w = workloads.WORKLOADS["ntt_i32"]
    v, g = workloads.generate(w)
    r = run_gpu(v, g, "i32").astype(np.int64)
    pts = workloads.sample_points(w.B, w.L, w.D, 4096, seed=1004)
    # sampled check first (fast, informative), then every element
    ref_pts = oracle.causal_conv_int_points(v, g, pts)
    assert np.array_equal(r[pts[:, 0], pts[:, 1], pts[:, 2]], ref_pts)
    assert np.array_equal(r, oracle.causal_conv_int(v, g))


def _leak(dtype, v, g, t_c, scale, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    r0 = run_gpu(v, g, dtype)
    v2, g2 = v.copy(), g.copy()
    if dtype == "i32":
        v2[:, t_c + 1:, :] = rng.integers(-128, 128, v2[:, t_c + 1:, :].shape)
        g2[:, t_c + 1:, :] = rng.integers(-128, 128, g2[:, t_c + 1:, :].shape)
    else:
        v2[:, t_c + 1:, :] = scale * rng.standard_normal(v2[:, t_c + 1:, :].shape)
        g2[:, t_c + 1:, :] = scale * rng.standard_normal(g2[:, t_c + 1:, :].shape)
    r1 = run_gpu(v2, g2, dtype)
    return float(np.abs(r1[:, : t_c + 1, :].astype(np.float64) - r0[:, : t_c + 1, :]).max())


# one representative shape per kernel: fused, channel groups, long rows (the
# binding takes the four-step path; D = 8 and 16 with TMA-staged inputs), and
# the NTT
DEGENERATE_CASES = [("f32", (2, 1000, 5)), ("bf16", (1, 700, 8)), ("f32", (1, 3000, 9)), ("bf16", (2, 4096, 8)),
                    ("f32", (1, 5000, 3)), ("f32", (1, 5000, 8)), ("bf16", (1, 6000, 16)), ("i32", (2, 3000, 5))]


@pytest.mark.parametrize("dtype,shape", DEGENERATE_CASES, ids=lambda c: str(c))
def test_degenerate_inputs(dtype, shape):
    """Zero inputs give exactly zero; an impulse v = delta_0 returns g (and
    g = delta_0 returns v): exactly for the NTT, within 1e-5 (fp32) or 2e-2
    (bf16) of max|g| for the float paths (the float error is spread over the
    row, so a per-element bound cannot hold where |g_t| is tiny)."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = shape
    rng = np.random.Generator(np.random.PCG64(L + D))
    if dtype == "i32":
        x = rng.integers(-128, 128, shape).astype(np.int32)
    else:
        x = rng.standard_normal(shape).astype(np.float32)
        if dtype == "bf16":
            x = workloads.bf16_round(x)
    zero = np.zeros_like(x)
    delta = np.zeros_like(x)
    delta[:, 0, :] = 1 if dtype != "bf16" else workloads.bf16_round(np.ones((B, D), np.float32))

    def conv(a, b):
        r = ssm.causal_conv(to_dev(a, dtype), to_dev(b, dtype))
        torch.cuda.synchronize()
        return as_f32(from_dev(r, dtype), dtype) if dtype != "i32" else from_dev(r, dtype)

    assert not np.any(conv(zero, zero)) and not np.any(conv(zero, x)) and not np.any(conv(x, zero))
    for a, b in ((delta, x), (x, delta)):
        r = conv(a, b)
        if dtype == "i32":
            assert np.array_equal(r, x)
        else:
            xf = as_f32(x, dtype)
            tol = (F32_TOL if dtype == "f32" else BF16_TOL) * np.abs(xf).max()
            assert np.abs(r - xf).max() <= tol


def test_leakage_ntt_is_exactly_zero():
    rng = np.random.Generator(np.random.PCG64(5))
    v = rng.integers(-128, 128, (2, 8192, 8)).astype(np.int32)
    g = rng.integers(-128, 128, (2, 8192, 8)).astype(np.int32)
    for t_c in (31, 4096, 8190):
        assert _leak("i32", v, g, t_c, 1, seed=t_c) == 0.0


def test_leakage_f32_measured():
    """Float transforms leak future tokens through rounding (the TL;DR of
    "Catastrophic Token Leakage in Convolutional Sequence Modeling"): the
    prefix moves when only the future changes.  The directly summed head
    (t < 32) is exactly causal."""
    v, g = _rand_float((1, 1024, 16), seed=3)
    assert _leak("f32", v, g, 31, 1e4, seed=1) == 0.0
    leak_mid = _leak("f32", v, g, 512, 1e4, seed=2)
    assert np.isfinite(leak_mid) and leak_mid > 0.0


def test_from_host_matches_device_path():
    """Host buffers in and out (batches pipelined in pieces over two streams
    when B >= 2; B = 5 splits unevenly, B = 1 takes the single-stream path)."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    rng = np.random.Generator(np.random.PCG64(2))
    for dtype, (v, g) in (("f32", _rand_float((2, 1000, 12), 1)),
                          ("f32", _rand_float((5, 300, 8), 3)),
                          ("f32", _rand_float((1, 5000, 4), 4)),
                          ("f32", _rand_float((3, 4500, 8), 6)),  # long rows in batch pieces: four-step per piece
                          ("i32", tuple(rng.integers(-128, 128, (2, 700, 8)).astype(np.int32) for _ in range(2))),
                          ("i32", tuple(rng.integers(-128, 128, (7, 100, 4)).astype(np.int32) for _ in range(2)))):
        tv, tg = to_dev(v, dtype), to_dev(g, dtype)
        ref = from_dev(ssm.causal_conv(tv, tg), dtype)
        hv = torch.from_numpy(v).pin_memory()
        hg = torch.from_numpy(g).pin_memory()
        hr = torch.empty_like(hv).pin_memory()
        dv, dg, dr = torch.empty_like(tv), torch.empty_like(tg), torch.empty_like(tv)
        ssm.causal_conv_from_host(hv, hg, hr, dv, dg, dr)
        torch.cuda.synchronize()
        assert np.array_equal(hr.numpy(), ref)


def test_side_stream_and_determinism():
    import torch
    import spectral_sequence_mixing_b200 as ssm
    v, g = _rand_float((2, 1024, 64), 9)
    tv, tg = to_dev(v, "f32"), to_dev(g, "f32")
    ref = ssm.causal_fftconv_f32(tv, tg)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = ssm.causal_fftconv_f32(tv, tg, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("shape", [(2, 1024, 64), (1, 4096, 16), (1, 8192, 8)], ids=lambda s: "x".join(map(str, s)))
def test_cuda_graph_capture_and_replay(shape):
    """Every launch path is stream-ordered with no host synchronisation or
    allocation inside the call, so it can be captured into a CUDA graph and
    replayed: the replay equals the eager call bit for bit."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    dtype = "i32" if shape[1] == 8192 else "f32"
    if dtype == "i32":
        rng = np.random.Generator(np.random.PCG64(3))
        v = rng.integers(-128, 128, shape).astype(np.int32)
        g = rng.integers(-128, 128, shape).astype(np.int32)
    else:
        v, g = _rand_float(shape, 11)
    tv, tg = to_dev(v, dtype), to_dev(g, dtype)
    ref = ssm.causal_conv(tv, tg)
    out = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ssm.causal_conv(tv, tg, out=out, stream=s)  # warm-up (per-device tables) outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(graph):
        ssm.causal_conv(tv, tg, out=out, stream=torch.cuda.current_stream())
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_bwd_fork_join_capture_and_side_stream():
    """The backward of fused-kernel rows forks its dg launch onto a library
    stream and joins it back: on a caller's side stream and inside a CUDA
    graph capture the results equal the eager default-stream call bit for
    bit, and the caller's stream sees both outputs complete."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    rng = np.random.Generator(np.random.PCG64(21))
    dr, v, g = (to_dev(rng.standard_normal((3, 777, 24)).astype(np.float32), "f32") for _ in range(3))
    ref_dv, ref_dg = ssm.causal_conv_bwd(dr, v, g)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    dv, dg = torch.empty_like(dr), torch.empty_like(dr)
    with torch.cuda.stream(s):
        ssm.causal_conv_bwd(dr, v, g, dv=dv, dg=dg, stream=s)
        # consumers on the caller's stream: both halves are complete here
        cv, cg = dv.clone(), dg.clone()
    s.synchronize()
    assert torch.equal(dv, ref_dv) and torch.equal(dg, ref_dg)
    assert torch.equal(cv, ref_dv) and torch.equal(cg, ref_dg)
    graph = torch.cuda.CUDAGraph()
    dv.zero_()
    dg.zero_()
    with torch.cuda.graph(graph):
        ssm.causal_conv_bwd(dr, v, g, dv=dv, dg=dg, stream=torch.cuda.current_stream())
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(dv, ref_dv) and torch.equal(dg, ref_dg)


def test_rejects_host_pointer_on_device_entry():
    import torch
    from spectral_sequence_mixing_b200 import _lib
    lib = _lib.load()
    h = torch.zeros(1, 16, 4)
    d = torch.zeros(1, 16, 4, device="cuda")
    d2 = torch.zeros(1, 16, 4, device="cuda")
    assert lib.causal_fftconv_f32(h.data_ptr(), d.data_ptr(), d2.data_ptr(), 1, 16, 4, None, 0, None) == 6
    assert lib.causal_fftconv_f32(d.data_ptr(), d2.data_ptr(), h.data_ptr(), 1, 16, 4, None, 0, None) == 6


# ---------------------------------------------------------------- backward
from gpu_helpers import run_gpu_bwd  # noqa: E402

BWD_SHAPES = [(1, 1, 1), (2, 33, 5), (3, 200, 19), (2, 1000, 37), (1, 1024, 8), (1, 2000, 3), (1, 4096, 2)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", BWD_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bwd_parity_full_oracle(shape, dtype):
    """dv_j = sum_{t>=j} dr_t g_{t-j}, dg_k = sum_{t>=k} dr_t v_{t-k} (training gradients)."""
    rng = np.random.Generator(np.random.PCG64(300 + sum(shape)))
    dr, v, g = (rng.standard_normal(shape).astype(np.float32) for _ in range(3))
    tol = F32_TOL
    if dtype == "bf16":
        dr, v, g = (workloads.bf16_round(x) for x in (dr, v, g))
        tol = BF16_TOL
    dv, dg = run_gpu_bwd(dr, v, g, dtype)
    ref_dv, den_dv, ref_dg, den_dg = oracle.causal_conv_bwd(*(as_f32(x, dtype) for x in (dr, v, g)))
    for name, got, ref, den in (("dv", dv, ref_dv, den_dv), ("dg", dg, ref_dg, den_dg)):
        n_bad, worst = float_violations(as_f32(got, dtype) if dtype == "bf16" else got, ref, den, tol)
        assert n_bad == 0, f"{name}: {n_bad} violations, worst ratio {worst:.3g}"


@pytest.mark.parametrize("shape", [(1, 20000, 2), (8, 1024, 768)], ids=lambda s: "x".join(map(str, s)))
def test_bwd_sampled_oracle(shape):
    """Cluster path (L > 4096) and the small_f32 shape, on sampled outputs."""
    B, L, D = shape
    rng = np.random.Generator(np.random.PCG64(400 + L))
    dr, v, g = (rng.standard_normal(shape).astype(np.float32) for _ in range(3))
    dv, dg = run_gpu_bwd(dr, v, g, "f32")
    pts = workloads.sample_points(B, L, D, 2048, seed=8)
    ref_dv, den_dv, ref_dg, den_dg = oracle.causal_conv_bwd_points(dr, v, g, pts)
    ix = (pts[:, 0], pts[:, 1], pts[:, 2])
    for name, got, ref, den in (("dv", dv[ix], ref_dv, den_dv), ("dg", dg[ix], ref_dg, den_dg)):
        n_bad, worst = float_violations(got, ref, den, F32_TOL)
        assert n_bad == 0, f"{name}: {n_bad} violations, worst ratio {worst:.3g}"


@pytest.mark.parametrize("two_pass", [True, False], ids=["four_step", "single_pass"])
@pytest.mark.parametrize("shape", [(1, 4099, 3), (2, 9001, 2), (2, 5001, 8), (1, 4608, 16)],
                         ids=lambda s: "x".join(map(str, s)))
def test_bwd_cluster_rows_odd_length(shape, two_pass):
    """Backward on long rows (v read and r written reversed in time), with
    and without the workspace (four-step path / cluster rows): odd lengths cut
    the last output pair of the real-output inverse in half; D = 8 and 16
    take the TMA forward pass with reversed reads, at a ragged length (the
    row of the last 512 time steps read directly) and at a whole number of
    512-step rows."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = shape
    rng = np.random.Generator(np.random.PCG64(500 + L))
    dr, v, g = (rng.standard_normal(shape).astype(np.float32) for _ in range(3))
    n_ws = ssm.fast_workspace_bytes(torch.float32, B, L, D) if two_pass else 0
    ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
    dv, dg = ssm.causal_conv_bwd(to_dev(dr, "f32"), to_dev(v, "f32"), to_dev(g, "f32"), workspace=ws)
    torch.cuda.synchronize()
    dv, dg = from_dev(dv, "f32"), from_dev(dg, "f32")
    pts = workloads.sample_points(B, L, D, 1024, seed=9)
    # the first and last time steps of every row, where the reversal and the cut pair meet
    ends = np.array([[b, t, d] for b in range(B) for d in range(D) for t in (0, 1, L - 2, L - 1)], dtype=pts.dtype)
    pts = np.concatenate([pts, ends])
    ref_dv, den_dv, ref_dg, den_dg = oracle.causal_conv_bwd_points(dr, v, g, pts)
    ix = (pts[:, 0], pts[:, 1], pts[:, 2])
    for name, got, ref, den in (("dv", dv[ix], ref_dv, den_dv), ("dg", dg[ix], ref_dg, den_dg)):
        n_bad, worst = float_violations(got, ref, den, F32_TOL)
        assert n_bad == 0, f"{name}: {n_bad} violations, worst ratio {worst:.3g}"


def test_bwd_consistent_with_forward_adjoint():
    """<dr, r(v, g)> = <dv, v> = <dg, g> with the GPU forward and backward."""
    import spectral_sequence_mixing_b200 as ssm
    rng = np.random.Generator(np.random.PCG64(5))
    shape = (2, 700, 16)
    dr, v, g = (rng.standard_normal(shape).astype(np.float32) for _ in range(3))
    r = run_gpu(v, g, "f32").astype(np.float64)
    dv, dg = run_gpu_bwd(dr, v, g, "f32")
    lhs = np.einsum("btd,btd->bd", dr.astype(np.float64), r)
    for grad, x in ((dv, v), (dg, g)):
        rhs = np.einsum("btd,btd->bd", grad.astype(np.float64), x.astype(np.float64))
        assert np.allclose(lhs, rhs, rtol=1e-4, atol=1e-3)


# ---------------------------------------------------------------- decode step
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [(2, 64, 5, 0), (2, 64, 5, 1), (3, 300, 37, 63), (3, 300, 37, 64),
                                  (1, 5000, 19, 4999), (8, 1024, 768, 1023), (8, 1024, 768, 500),
                                  (2, 3000, 260, 2999), (1, 40, 12, 15)],
                         ids=lambda c: "x".join(map(str, c)))
def test_decode_step_matches_oracle(case, dtype):
    """One decode step equals the causal sum at position t, bit-identically
    across calls (fixed-order fp64 reduction)."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, Lcap, D, t = case
    rng = np.random.Generator(np.random.PCG64(sum(case)))
    v = rng.standard_normal((B, Lcap, D)).astype(np.float32)
    g = rng.standard_normal((B, Lcap, D)).astype(np.float32)
    tol = F32_TOL
    if dtype == "bf16":
        v, g = workloads.bf16_round(v), workloads.bf16_round(g)
        tol = BF16_TOL
    tv, tg = to_dev(v, dtype), to_dev(g, dtype)
    r1 = ssm.causal_conv_decode(tv, tg, t)
    r2 = ssm.causal_conv_decode(tv, tg, t)
    torch.cuda.synchronize()
    assert torch.equal(r1.view(torch.int16) if dtype == "bf16" else r1, r2.view(torch.int16) if dtype == "bf16" else r2)
    got = as_f32(from_dev(r1, dtype), dtype)
    pts = np.array([(b, t, d) for b in range(B) for d in range(D)], np.int64)
    ref, den = oracle.causal_conv_points(as_f32(v, dtype), as_f32(g, dtype), pts)
    n_bad, worst = float_violations(got.reshape(-1), ref, den, tol)
    assert n_bad == 0, f"{n_bad} violations, worst ratio {worst:.3g}"
    if dtype == "f32":  # fp64 accumulation, one rounding to float at the end
        assert np.all(np.abs(got.reshape(-1) - ref) <= 6.0e-8 * np.abs(ref) + 1e-12 * den)


def test_accuracy_report_runs():
    """The accuracy / leakage report (tests/accuracy_report.py) on the small
    workloads: no bound violation, the directly summed head does not leak."""
    import accuracy_report
    for line in accuracy_report.main(["--workloads", "tiny_f32,small_f32"]):
        assert line["accuracy"]["violations"] == 0
        assert line["leakage"]["31"]["max_abs"] == 0.0


@pytest.mark.parametrize("case", [(1, 5000, 24, "f32", 2), (1, 1024, 768, "f32", 3), (4, 300, 40, "bf16", 3),
                                  (3, 4096, 16, "i32", 2)], ids=lambda c: "x".join(map(str, c)))
def test_partitioned_call_equals_whole_call(case):
    """The multi-GPU split, run rank after rank on one GPU: every rank's slab
    (batches, or channels when B is smaller than the rank count) convolved by
    the library and placed back gives the unsplit call's result bit for bit,
    and a sampled set of its outputs matches the oracle."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    from spectral_sequence_mixing_b200 import partition
    B, L, D, dtype, world = case
    rng = np.random.Generator(np.random.PCG64(B * L + D))
    if dtype == "i32":
        v, g = (rng.integers(-128, 128, (B, L, D)).astype(np.int32) for _ in range(2))
    else:
        v, g = _rand_float((B, L, D), seed=L + D, scale_g=0.125)
        if dtype == "bf16":
            v, g = workloads.bf16_round(v), workloads.bf16_round(g)
    tv, tg = to_dev(v, dtype), to_dev(g, dtype)
    whole = ssm.causal_conv(tv, tg)
    pieced = torch.empty_like(whole)
    for rank in range(world):
        s = partition.shard_for(B, D, world, rank)
        partition.place(pieced, ssm.causal_conv(partition.take(tv, s), partition.take(tg, s)), s)
    torch.cuda.synchronize()
    a, b = from_dev(whole, dtype), from_dev(pieced, dtype)
    assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), "split call differs from the whole call"
    pts = np.stack([rng.integers(0, B, 512), rng.integers(0, L, 512), rng.integers(0, D, 512)], axis=1)
    if dtype == "i32":
        ref = oracle.causal_conv_int_points(v, g, pts)
        assert np.array_equal(b[pts[:, 0], pts[:, 1], pts[:, 2]].astype(np.int64), ref)
    else:
        ref, den = oracle.causal_conv_points(as_f32(v, dtype), as_f32(g, dtype), pts)
        got = as_f32(b, dtype)[pts[:, 0], pts[:, 1], pts[:, 2]]
        n_bad, worst = float_violations(got, ref, den, F32_TOL if dtype == "f32" else BF16_TOL)
        assert n_bad == 0, f"{n_bad} sampled outputs beyond the bound, worst ratio {worst:.3g}"


# bf16 rows with 2048 < L <= 4096 run on the tensor cores (clusters of 8 channels):
# whole groups, ragged last groups (D not a multiple of 8), single channels,
# and bases that are not 16-byte aligned (element-wise group accesses)
TC_SHAPES = [(2, 2049, 8), (1, 3000, 13), (1, 4096, 24), (3, 2500, 1), (1, 4095, 40)]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("offset", [0, 1])
def test_tensor_core_rows_bf16(shape, offset):
    import torch
    import spectral_sequence_mixing_b200 as ssm
    B, L, D = shape
    v, g = _rand_float(shape, seed=300 + L + D, scale_g=0.125)
    vb, gb = workloads.bf16_round(v), workloads.bf16_round(g)
    n = B * L * D

    def place(x):  # a bf16 tensor starting `offset` elements into its allocation
        buf = torch.zeros(n + offset, dtype=torch.bfloat16, device="cuda")
        buf[offset:] = to_dev(x, "bf16").reshape(-1)
        return buf[offset:].view(B, L, D)

    out = torch.empty(n + offset, dtype=torch.bfloat16, device="cuda")[offset:].view(B, L, D)
    ssm.causal_fftconv_bf16(place(vb), place(gb), out=out)
    torch.cuda.synchronize()
    r = as_f32(from_dev(out, "bf16"), "bf16")
    r_ref, den = oracle.causal_conv(as_f32(vb, "bf16"), as_f32(gb, "bf16"))
    n_bad, worst = float_violations(r, r_ref, den, BF16_TOL)
    assert n_bad == 0, f"{n_bad} elements beyond the bf16 bound, worst ratio {worst:.3g}"
