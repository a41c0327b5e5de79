"""Oracle for the causal sequence convolution -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product library (``spectral_sequence_mixing_b200``) never imports it, and the
two share no code: this package wraps ``causal_conv_oracle.c`` (plain C, fp64
and int64 direct sums) through ctypes and adds nothing but marshalling.

What it computes (Caracal: Causal Architecture via Spectral Mixing, "Key design
1" and "Key design 2"): for every (batch b, channel d) row of channel-last
[B, L, D] arrays,

    r[b, t, d]   = sum_{j=0..t} v[b, j, d] * g[b, t - j, d]
    den[b, t, d] = sum_{j=0..t} |v[b, j, d] * g[b, t - j, d]|   (float only)

The pages state that pad-to-2L -> FFT -> pointwise product -> inverse FFT ->
truncate-to-L equals this sum exactly, so the oracle is the sum itself.  The
integer variant (number-theoretic transform mod p, "Catastrophic Token Leakage
in Convolutional Sequence Modeling", abstract) is exact, so its oracle is the
same sum in int64; ``centered_mod`` gives what an exact mod-p transform returns
when the true sum does not fit in (-p/2, p/2).

The submodule ``oracle.mhf_gate`` adds the gate stream of the same block
(sigmoid and the head-grouped causal Conv1d_G2, float64 numpy) and composes it
with this sum; its pins are in tests/test_oracle_mhf_pins.py.  The submodule
``oracle.mhf_dwconv`` is the block's first step, the causal depthwise
convolution (kernel size 3 on the page); pins in tests/test_oracle_dwconv_pins.py.

Pins (tests/test_oracle_pins.py): hand-computed fixtures in tests/golden/,
delta inputs, closed-form sums, numpy.convolve on single rows, an fp64 FFT
convolution (independent algorithm), commutativity, bilinearity, shift
equivariance, strict causality, wrap-around, integer extremes, and mutants of
this C source that each pin set must reject.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "causal_conv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_I64 = ctypes.c_int64
_PTR = ctypes.c_void_p


def build(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP) into a shared library."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", out, src, "-lm"]
        subprocess.check_call(cmd)
    return out


def _bind(lib):
    sig_f = [_PTR, _PTR, _I64, _I64, _I64, _PTR, _PTR]
    sig_fp = [_PTR, _PTR, _I64, _I64, _I64, _PTR, _I64, _PTR, _PTR]
    for name in ("oracle_conv_f64", "oracle_conv_f32in"):
        getattr(lib, name).argtypes = sig_f
        getattr(lib, name).restype = None
    for name in ("oracle_conv_f64_points", "oracle_conv_f32in_points"):
        getattr(lib, name).argtypes = sig_fp
        getattr(lib, name).restype = None
    lib.oracle_conv_i32in.argtypes = [_PTR, _PTR, _I64, _I64, _I64, _PTR]
    lib.oracle_conv_i32in.restype = None
    lib.oracle_conv_i32in_points.argtypes = [_PTR, _PTR, _I64, _I64, _I64, _PTR, _I64, _PTR]
    lib.oracle_conv_i32in_points.restype = None
    lib.oracle_conv_bwd_f32in.argtypes = [_PTR, _PTR, _PTR, _I64, _I64, _I64, _PTR, _PTR, _PTR, _PTR]
    lib.oracle_conv_bwd_f32in.restype = None
    lib.oracle_conv_bwd_f32in_points.argtypes = [_PTR, _PTR, _PTR, _I64, _I64, _I64, _PTR, _I64, _PTR, _PTR,
                                                 _PTR, _PTR]
    lib.oracle_conv_bwd_f32in_points.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library.  ``path`` loads another
    build of the same source (the pin tests use it for mutants)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check3(v: np.ndarray, g: np.ndarray):
    if v.shape != g.shape or v.ndim != 3:
        raise ValueError(f"v and g must be [B, L, D] of equal shape, got {v.shape} and {g.shape}")
    return v.shape


def num_threads() -> int:
    return int(load().oracle_num_threads())


def causal_conv(v: np.ndarray, g: np.ndarray, lib=None):
    """Full r and den, float64 [B, L, D].  Accepts float64, float32 (widened
    exactly) or any float array representable in float32 (e.g. bf16 values
    already widened to float32)."""
    lib = lib or load()
    B, L, D = _check3(v, g)
    r = np.empty((B, L, D), np.float64)
    den = np.empty((B, L, D), np.float64)
    if v.dtype == np.float32 and g.dtype == np.float32:
        v = np.ascontiguousarray(v)
        g = np.ascontiguousarray(g)
        lib.oracle_conv_f32in(_ptr(v), _ptr(g), B, L, D, _ptr(r), _ptr(den))
    else:
        v = np.ascontiguousarray(v, np.float64)
        g = np.ascontiguousarray(g, np.float64)
        lib.oracle_conv_f64(_ptr(v), _ptr(g), B, L, D, _ptr(r), _ptr(den))
    return r, den


def causal_conv_points(v: np.ndarray, g: np.ndarray, pts: np.ndarray, lib=None):
    """r and den at the (b, t, d) triples in ``pts`` (shape [n, 3])."""
    lib = lib or load()
    B, L, D = _check3(v, g)
    pts = np.ascontiguousarray(pts, np.int64).reshape(-1, 3)
    if pts.size and ((pts.min(0) < 0).any() or (pts.max(0) >= np.array([B, L, D])).any()):
        raise ValueError("sample point out of range")
    n = pts.shape[0]
    r = np.empty(n, np.float64)
    den = np.empty(n, np.float64)
    if v.dtype == np.float32 and g.dtype == np.float32:
        v = np.ascontiguousarray(v)
        g = np.ascontiguousarray(g)
        lib.oracle_conv_f32in_points(_ptr(v), _ptr(g), B, L, D, _ptr(pts), n, _ptr(r), _ptr(den))
    else:
        v = np.ascontiguousarray(v, np.float64)
        g = np.ascontiguousarray(g, np.float64)
        lib.oracle_conv_f64_points(_ptr(v), _ptr(g), B, L, D, _ptr(pts), n, _ptr(r), _ptr(den))
    return r, den


def causal_conv_int(v: np.ndarray, g: np.ndarray, lib=None) -> np.ndarray:
    """Exact integer r (int64 [B, L, D]) for int32 inputs."""
    lib = lib or load()
    B, L, D = _check3(v, g)
    v = np.ascontiguousarray(v, np.int32)
    g = np.ascontiguousarray(g, np.int32)
    r = np.empty((B, L, D), np.int64)
    lib.oracle_conv_i32in(_ptr(v), _ptr(g), B, L, D, _ptr(r))
    return r


def causal_conv_int_points(v: np.ndarray, g: np.ndarray, pts: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    B, L, D = _check3(v, g)
    pts = np.ascontiguousarray(pts, np.int64).reshape(-1, 3)
    if pts.size and ((pts.min(0) < 0).any() or (pts.max(0) >= np.array([B, L, D])).any()):
        raise ValueError("sample point out of range")
    v = np.ascontiguousarray(v, np.int32)
    g = np.ascontiguousarray(g, np.int32)
    r = np.empty(pts.shape[0], np.int64)
    lib.oracle_conv_i32in_points(_ptr(v), _ptr(g), B, L, D, _ptr(pts), pts.shape[0], _ptr(r))
    return r


def causal_conv_bwd(dr: np.ndarray, v: np.ndarray, g: np.ndarray, lib=None):
    """Gradients of the causal convolution (float inputs widened exactly to
    double): returns (dv, den_dv, dg, den_dg), each float64 [B, L, D], with
    dv_j = sum_{t>=j} dr_t g_{t-j} and dg_k = sum_{t>=k} dr_t v_{t-k}."""
    lib = lib or load()
    B, L, D = _check3(v, g)
    if dr.shape != v.shape:
        raise ValueError("dr must have the shape of v")
    dr, v, g = (np.ascontiguousarray(x, np.float32) for x in (dr, v, g))
    out = [np.empty((B, L, D), np.float64) for _ in range(4)]
    lib.oracle_conv_bwd_f32in(_ptr(dr), _ptr(v), _ptr(g), B, L, D, *(_ptr(o) for o in out))
    return tuple(out)


def causal_conv_bwd_points(dr, v, g, pts, lib=None):
    lib = lib or load()
    B, L, D = _check3(v, g)
    pts = np.ascontiguousarray(pts, np.int64).reshape(-1, 3)
    if pts.size and ((pts.min(0) < 0).any() or (pts.max(0) >= np.array([B, L, D])).any()):
        raise ValueError("sample point out of range")
    dr, v, g = (np.ascontiguousarray(x, np.float32) for x in (dr, v, g))
    out = [np.empty(pts.shape[0], np.float64) for _ in range(4)]
    lib.oracle_conv_bwd_f32in_points(_ptr(dr), _ptr(v), _ptr(g), B, L, D, _ptr(pts), pts.shape[0],
                                     *(_ptr(o) for o in out))
    return tuple(out)


def centered_mod(x: np.ndarray, p: int) -> np.ndarray:
    """The representative of x mod p in (-p/2, p/2] ... for odd p this is
    [-(p-1)/2, (p-1)/2]: what an exact transform mod p followed by the
    centered lift returns for a true integer result x."""
    x = np.asarray(x, np.int64)
    m = np.mod(x, p)
    return np.where(m > (p - 1) // 2, m - p, m)
