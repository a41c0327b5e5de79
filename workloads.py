"""Seeded synthetic inputs for the causal convolution -- shared by the tests,
the benchmark and the smoke check.

This module holds no part of the convolution's arithmetic: it only draws
random numbers and rounds them to the I/O type, so both the CUDA path and the
oracle may take their inputs from it.

Shapes follow the workloads the pages describe (Caracal: Causal Architecture
via Spectral Mixing: Caracal-Small ~120M and Caracal-Large ~724M models, a
4096-token context for the 345M comparison, the "100k+ context" limitation;
and the integer-transform variant of "Catastrophic Token Leakage in
Convolutional Sequence Modeling").  The pages train on public text suites,
which these synthetic arrays stand in for.

Recipe (every array [B, L, D] channel-last, drawn in C order from
numpy.random.Generator(PCG64(seed)) in float64, v first, then g's factors in
the order listed, then rounded to the I/O type):

  tiny_f32      [1, 256, 64]    fp32  v ~ N(0,1); g ~ N(0,1)                      seed 0
  small_f32     [8, 1024, 768]  fp32  v ~ N(0,1); g = sigmoid(z1)*exp(-t/128)*sign(z2)  seed 1
  large_bf16    [4, 4096, 1536] bf16  v ~ N(0,1); g ~ N(0, 1/64)                  seed 2
  long_f32      [1, 65536, 1024] fp32 v ~ N(0,1); g = z*(1+t)^-0.75               seed 3
  ntt_i32       [4, 8192, 256]  int32 v, g uniform integers in [-128, 127]        seed 4

The gate stream of the same block (x_g = Conv1d_G2(sigmoid(a)), grouped by
head) takes a = Linear_G1(x_norm) and the Conv1d weights instead of g
(``generate_gate``; v, then a, then w, then bias from one generator):

  mhf_small_f32 [8, 1024, 768]  fp32  12 heads of 64, K = 3 taps               seed 5
  v, a ~ N(0,1); w, bias ~ U(-1/sqrt(C K), 1/sqrt(C K)) (a default Conv1d's
  initialisation range, fan-in C K), w float32 [D, C, K], bias float32 [D].

The block's causal depthwise convolution (``generate_dwconv``; x, then w,
then bias):

  dwconv_small_f32 [8, 1024, 768] fp32  K = 3 taps                             seed 6
  x ~ N(0,1); w, bias ~ U(-1/sqrt(K), 1/sqrt(K)) (a default depthwise Conv1d's
  range, fan-in K), w float32 [D, K], bias float32 [D].
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    D: int
    dtype: str  # "f32" | "bf16" | "i32"
    seed: int
    description: str

    @property
    def units(self) -> int:
        """Outputs r[b, t, d] per call."""
        return self.B * self.L * self.D

    @property
    def elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2, "i32": 4}[self.dtype]

    @property
    def algorithmic_bytes(self) -> int:
        """Read v + read g + write r, once each."""
        return 3 * self.units * self.elem_bytes


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 256, 64, "f32", 0,
                         "tiny fp32 causal conv, v,g ~ N(0,1)"),
    "small_f32": Workload("small_f32", 8, 1024, 768, "f32", 1,
                          "Caracal-Small-shaped MHF conv (12 heads x 64), decaying signed gate kernel"),
    "large_bf16": Workload("large_bf16", 4, 4096, 1536, "bf16", 2,
                           "Caracal-Large-shaped MHF conv (24 heads x 64), bf16 I/O"),
    "long_f32": Workload("long_f32", 1, 65536, 1024, "f32", 3,
                         "long-context fp32 conv, N = 2L = 131072, power-law gate kernel"),
    "ntt_i32": Workload("ntt_i32", 4, 8192, 256, "i32", 4,
                        "exact integer conv, values in [-128, 127], N = 16384"),
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); returns the
    16-bit patterns as uint16.  Inputs here are finite."""
    bits = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((bits >> 16) & 1)
    return ((bits + bias) >> 16).astype(np.uint16)


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _t_axis(L: int) -> np.ndarray:
    return np.arange(L, dtype=np.float64).reshape(1, L, 1)


def generate(w: Workload | str, B: int | None = None, L: int | None = None, D: int | None = None,
             seed: int | None = None):
    """Draw (v, g) for a workload recipe, optionally at other sizes / seed.

    Returns numpy arrays: float32 for "f32", uint16 bf16 patterns for "bf16",
    int32 for "i32".
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    B = w.B if B is None else B
    L = w.L if L is None else L
    D = w.D if D is None else D
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (B, L, D)
    if w.dtype == "i32":
        v = rng.integers(-128, 128, size=shape, dtype=np.int64).astype(np.int32)
        g = rng.integers(-128, 128, size=shape, dtype=np.int64).astype(np.int32)
        return v, g
    v = rng.standard_normal(shape)
    if w.name == "small_f32":
        z1 = rng.standard_normal(shape)
        z2 = rng.standard_normal(shape)
        g = (1.0 / (1.0 + np.exp(-z1))) * np.exp(-_t_axis(L) / 128.0) * np.sign(z2)
    elif w.name == "long_f32":
        z = rng.standard_normal(shape)
        g = z * (1.0 + _t_axis(L)) ** -0.75
    elif w.name == "large_bf16":
        g = rng.standard_normal(shape) * 0.125
    else:
        g = rng.standard_normal(shape)
    if w.dtype == "bf16":
        return bf16_round(v.astype(np.float32)), bf16_round(g.astype(np.float32))
    return v.astype(np.float32), g.astype(np.float32)


def sample_points(B: int, L: int, D: int, n: int, seed: int) -> np.ndarray:
    """Stratified (b, t, d) sample: a quarter with t < 64, a quarter with
    t >= L - 64, half uniform over t.  Shape [n, 3], int64."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = n // 4
    parts = [
        rng.integers(0, min(64, L), size=q),
        rng.integers(max(0, L - 64), L, size=q),
        rng.integers(0, L, size=n - 2 * q),
    ]
    t = np.concatenate(parts)
    b = rng.integers(0, B, size=n)
    d = rng.integers(0, D, size=n)
    return np.stack([b, t, d], axis=1).astype(np.int64)


@dataclass(frozen=True)
class GateWorkload:
    name: str
    B: int
    L: int
    D: int
    H: int
    K: int
    dtype: str  # "f32" | "bf16"
    seed: int
    description: str

    @property
    def units(self) -> int:
        return self.B * self.L * self.D


GATE_WORKLOADS = {
    "mhf_small_f32": GateWorkload("mhf_small_f32", 8, 1024, 768, 12, 3, "f32", 5,
                                  "Caracal-Small-shaped MHF gate + conv (12 heads x 64, 3 taps)"),
}


def generate_gate(B: int, L: int, D: int, H: int, K: int, dtype: str, seed: int):
    """(v, a, w, bias): v, a [B, L, D] in the I/O type (float32, or bf16 bit
    patterns as uint16); w float32 [D, D/H, K]; bias float32 [D]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    C = D // H
    v = rng.standard_normal((B, L, D)).astype(np.float32)
    a = rng.standard_normal((B, L, D)).astype(np.float32)
    bound = 1.0 / np.sqrt(C * K)
    w = rng.uniform(-bound, bound, (D, C, K)).astype(np.float32)
    bias = rng.uniform(-bound, bound, D).astype(np.float32)
    if dtype == "bf16":
        return bf16_round(v), bf16_round(a), w, bias
    return v, a, w, bias


@dataclass(frozen=True)
class DwconvWorkload:
    name: str
    B: int
    L: int
    D: int
    K: int
    dtype: str
    seed: int
    description: str

    @property
    def units(self) -> int:
        return self.B * self.L * self.D


DWCONV_WORKLOADS = {
    "dwconv_small_f32": DwconvWorkload("dwconv_small_f32", 8, 1024, 768, 3, "f32", 6,
                                       "Caracal-Small-shaped causal depthwise conv, kernel size 3"),
}


def generate_dwconv(B: int, L: int, D: int, K: int, dtype: str, seed: int):
    """(x, w, bias): x [B, L, D] in the I/O type (float32, or bf16 bit
    patterns as uint16); w float32 [D, K]; bias float32 [D]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((B, L, D)).astype(np.float32)
    bound = 1.0 / np.sqrt(K)
    w = rng.uniform(-bound, bound, (D, K)).astype(np.float32)
    bias = rng.uniform(-bound, bound, D).astype(np.float32)
    return (bf16_round(x) if dtype == "bf16" else x), w, bias
