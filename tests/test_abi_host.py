"""C-ABI library: loads, exports every declared symbol, and rejects bad
arguments on the host before touching a GPU (CPU only; no compute calls)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER_DIR = os.path.join(ROOT, "include")


def declared_symbols():
    names = []
    for f in sorted(os.listdir(HEADER_DIR)):
        if f.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, f)).read()
            names += re.findall(r"CC_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


@pytest.fixture(scope="module")
def lib():
    from spectral_sequence_mixing_b200 import build
    build.build()
    from spectral_sequence_mixing_b200 import _lib
    return _lib.load()


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ("causal_fftconv_f32", "causal_fftconv_bf16", "causal_ntt_conv_i32", "causal_conv_from_host",
              "causal_conv_workspace_bytes", "causal_conv_max_len", "causal_conv_strerror", "causal_ntt_params"):
        assert n in names, n


def test_library_exports_every_declared_symbol(lib):
    from spectral_sequence_mixing_b200 import _lib
    for n in declared_symbols():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no ctypes signature in the binding"


def test_strerror(lib):
    from spectral_sequence_mixing_b200 import strerror
    seen = set()
    for st in range(7):
        s = strerror(st)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 7
    assert strerror(99) == "unknown status"


def test_max_len_and_workspace(lib):
    assert lib.causal_conv_max_len(0) >= 1024
    assert lib.causal_conv_max_len(2) == 8192
    assert lib.causal_conv_max_len(7) == 0
    assert lib.causal_conv_workspace_bytes(0, 8, 1024, 768) == 0
    assert lib.causal_conv_workspace_bytes(9, 8, 1024, 768) == ctypes.c_size_t(-1).value
    assert lib.causal_conv_workspace_bytes(0, 0, 1024, 768) == ctypes.c_size_t(-1).value


def test_ntt_params_number_theory(lib):
    """The transform constants against number theory done here in Python."""
    from spectral_sequence_mixing_b200 import ntt_params
    p = 2013265921
    assert p == 15 * 2 ** 27 + 1
    # 31 is a primitive root: 31^((p-1)/q) != 1 for each prime q | p-1 = 2^27 * 3 * 5
    for q in (2, 3, 5):
        assert pow(31, (p - 1) // q, p) != 1
    for N in (2, 1024, 16384, 2 ** 27):
        c = ntt_params(N)
        assert c["p"] == p
        w = c["omega"]
        assert pow(w, N, p) == 1 and pow(w, N // 2, p) == p - 1  # order exactly N
        assert w * c["omega_inv"] % p == 1
        assert N * c["n_inv"] % p == 1
        assert p * c["p_inv_mod_2_32"] % 2 ** 32 == 1
        assert c["r2_mod_p"] == 2 ** 64 % p
    assert ntt_params(16384)["omega"] == pow(31, (p - 1) // 16384, p)


@pytest.mark.parametrize("N", [0, 1, 3, 12, 2 ** 28])
def test_ntt_params_rejects_bad_n(lib, N):
    out = (ctypes.c_uint32 * 6)()
    assert lib.causal_ntt_params(N, out) == 1


# Fake (never dereferenced) addresses: every check below fails before the
# library makes any CUDA call.
A, B_, C = 0x10000000, 0x20000000, 0x30000000


@pytest.mark.parametrize("fn", ["causal_fftconv_f32", "causal_fftconv_bf16", "causal_ntt_conv_i32"])
def test_host_side_argument_errors(lib, fn):
    f = getattr(lib, fn)
    INVALID, UNSUP, ALIAS, WS = 1, 2, 3, 4
    assert f(None, B_, C, 1, 16, 4, None, 0, None) == INVALID
    assert f(A, None, C, 1, 16, 4, None, 0, None) == INVALID
    assert f(A, B_, None, 1, 16, 4, None, 0, None) == INVALID
    for shape in [(0, 16, 4), (1, 0, 4), (1, 16, 0), (-1, 16, 4), (2 ** 40, 2 ** 20, 2 ** 10)]:
        assert f(A, B_, C, *shape, None, 0, None) == INVALID, shape
    assert f(A, B_, C, 1, 10 ** 7, 4, None, 0, None) == UNSUP
    assert f(A, B_, A + 8, 1, 16, 4, None, 0, None) == ALIAS   # r overlaps v
    assert f(A, B_, B_ - 8, 1, 16, 4, None, 0, None) == ALIAS  # r overlaps g
    # workspace: none required today, so any size passes that check; a
    # too-small workspace can only be tested once a path needs one.
    assert lib.causal_conv_workspace_bytes(0, 1, 16, 4) == 0
    _ = WS


def test_from_host_rejects_null_host_pointers(lib):
    assert lib.causal_conv_from_host(0, None, B_, C, A, B_, C, 1, 16, 4, None, 0, None) == 1
    assert lib.causal_conv_from_host(9, A, B_, C, A + 0x1000000, B_ + 0x1000000, C + 0x1000000, 1, 16, 4, None, 0,
                                     None) == 1


def test_bwd_host_side_argument_errors(lib):
    f = lib.causal_fftconv_bwd_f32
    D_, E_ = 0x40000000, 0x50000000
    assert f(A, B_, C, None, E_, 1, 16, 4, None, 0, None) == 1        # null dv
    assert f(A, B_, C, D_, None, 1, 16, 4, None, 0, None) == 1        # null dg
    assert f(A, B_, C, D_, E_, 0, 16, 4, None, 0, None) == 1          # B < 1
    assert f(A, B_, C, A + 8, E_, 1, 16, 4, None, 0, None) == 3       # dv overlaps dr
    assert f(A, B_, C, D_, B_ + 8, 1, 16, 4, None, 0, None) == 3      # dg overlaps v
    assert f(A, B_, C, D_, D_ + 8, 1, 16, 4, None, 0, None) == 3      # dv overlaps dg


def test_decode_host_side_checks(lib):
    f = lib.causal_conv_decode_f32
    ws = lib.causal_conv_decode_workspace_bytes(0, 8, 768, 1023)
    assert 0 < ws < 2 ** 32 and ws % (8 * 768 * 8) == 0
    assert lib.causal_conv_decode_workspace_bytes(0, 8, 768, -1) == ctypes.c_size_t(-1).value
    big = 1 << 30
    W = 0x60000000
    assert f(None, B_, C, 1, 16, 4, 3, W, big, None) == 1            # null cache
    assert f(A, B_, C, 1, 16, 4, 16, W, big, None) == 1              # t >= Lcap
    assert f(A, B_, C, 1, 16, 4, -1, W, big, None) == 1              # t < 0
    assert f(A, B_, C, 70000, 16, 4, 3, W, big, None) == 1           # B > 65535
    assert f(A, B_, A + 8, 1, 16, 4, 3, W, big, None) == 3           # output inside a cache
    assert f(A, B_, C, 1, 16, 4, 3, None, 0, None) == 4              # workspace missing
    assert f(A, B_, C, 1, 16, 4, 3, W, 8, None) == 4                 # workspace too small
    assert lib.causal_conv_decode_bf16(A, B_, C, 1, 16, 4, 3, W, 8, None) == 4


def test_decode_alias_is_range_exact(lib):
    """An output just past the end of a cache is not an overlap; one inside is."""
    f = lib.causal_conv_decode_f32
    B, L, D = 1, 16, 4
    cache = B * L * D * 4
    W = 0x60000000
    assert f(A, B_, A + cache, B, L, D, 3, W, 8, None) == 4      # passes the alias check, fails on workspace
    assert f(A, B_, A + cache - 4, B, L, D, 3, W, 8, None) == 3  # last cache element overlaps
    assert f(A, B_, A - B * D * 4, B, L, D, 3, W, 8, None) == 4  # output right before the cache


def test_fault_flags_host_checks(lib):
    import ctypes
    assert lib.causal_conv_fault_flags(0, None, 0) == 1                      # NULL flags
    out = ctypes.c_uint(7)
    assert lib.causal_conv_fault_flags(-1, ctypes.byref(out), 0) == 1       # bad device


def test_fast_workspace_bytes(lib):
    f = lib.causal_conv_fast_workspace_bytes

    def four_step(rows):  # partial transforms [131072][rows] float2, 64 norm partials and a scale pair per row
        return 131072 * rows * 8 + 64 * rows * 8 + rows * 8
    assert f(0, 1, 4096, 8) == 0                       # rows of one CTA: no workspace path
    assert f(0, 1, 4097, 8) == four_step(8)
    assert f(1, 2, 65536, 16) == four_step(32)          # bf16 keeps fp32 partial transforms
    assert f(2, 1, 5000, 8) == 0                       # NTT path
    assert f(0, 1, 65537, 8) == 0                      # beyond the longest row
    assert f(0, 70000, 5000, 8) == four_step(560000)
    assert f(0, 2 ** 20, 5000, 2 ** 12) == 0           # B * D rows beyond int
    assert f(0, 1, 5000, 0) == 0 and f(7, 1, 5000, 8) == 0


@pytest.mark.parametrize("fn", ["causal_mhf_gate_f32", "causal_mhf_gate_bf16"])
def test_gate_host_side_argument_errors(lib, fn):
    """Every check of the gate entry that needs no device (dummy pointers)."""
    f = getattr(lib, fn)
    W_, G_ = 0x40000000, 0x50000000
    INVALID, UNSUP, ALIAS = 1, 2, 3
    ok = (1, 16, 64, 2, 3)  # B, L, D, H, K: head width 32
    assert f(None, W_, None, G_, *ok, None) == INVALID
    assert f(A, None, None, G_, *ok, None) == INVALID
    assert f(A, W_, None, None, *ok, None) == INVALID
    for shape in [(0, 16, 64, 2, 3), (1, 0, 64, 2, 3), (1, 16, 0, 2, 3), (1, 16, 64, 0, 3), (1, 16, 64, 2, 0),
                  (1, 16, 64, 3, 1), (1, 16, 64, -2, 1)]:
        assert f(A, W_, None, G_, *shape, None) == INVALID, shape
    for shape in [(1, 16, 96, 2, 1), (1, 16, 256, 2, 1), (1, 16, 8, 1, 1), (1, 16, 64, 2, 5)]:
        assert f(A, W_, None, G_, *shape, None) == UNSUP, shape       # head width 48 / 128 / 8, 5 taps
    assert f(A, W_, None, A + 8, *ok, None) == ALIAS                    # g overlaps a
    assert f(A, W_, None, W_ - 8, *ok, None) == ALIAS                   # g overlaps w
    assert f(A, W_, G_ + 16, G_, *ok, None) == ALIAS                    # g overlaps bias


def test_gated_conv_host_side_checks(lib):
    f = lib.causal_mhf_gated_conv_f32
    V_, W_, R_, S_ = 0x40000000, 0x50000000, 0x60000000, 0x70000000
    need = lib.causal_mhf_gated_conv_workspace_bytes(0, 1, 16, 64)
    assert need == 16 * 64 * 4
    assert lib.causal_mhf_gated_conv_workspace_bytes(1, 1, 16, 64) == 16 * 64 * 2
    assert lib.causal_mhf_gated_conv_workspace_bytes(2, 1, 16, 64) == ctypes.c_size_t(-1).value
    ok = (1, 16, 64, 2, 3)
    assert f(None, A, W_, None, R_, *ok, S_, need, None) == 1           # null v
    assert f(V_, A, W_, None, R_, *ok, None, need, None) == 1           # null workspace
    assert f(V_, A, W_, None, R_, *ok, S_, need - 1, None) == 4         # workspace too small
    assert f(V_, A, W_, None, V_ + 4, *ok, S_, need, None) == 3         # r overlaps v
    assert f(V_, A, W_, None, R_, *ok, A + 64, need, None) == 3         # workspace overlaps a
    assert f(V_, A, W_, None, R_, *ok, V_ + 64, need, None) == 3        # workspace overlaps v
    assert f(V_, A, W_, None, R_, *ok, R_ - 64, need, None) == 3        # workspace overlaps r
    assert f(V_, A, W_, None, R_, 1, 16, 96, 2, 1, S_, 16 * 96 * 4, None) == 2  # head width 48


@pytest.mark.parametrize("fn", ["causal_dwconv_f32", "causal_dwconv_bf16"])
def test_dwconv_host_side_argument_errors(lib, fn):
    f = getattr(lib, fn)
    W_, Y_ = 0x40000000, 0x50000000
    ok = (1, 16, 64, 3)
    assert f(None, W_, None, Y_, *ok, None) == 1
    assert f(A, None, None, Y_, *ok, None) == 1
    assert f(A, W_, None, None, *ok, None) == 1
    for shape in [(0, 16, 64, 3), (1, 0, 64, 3), (1, 16, 0, 3), (1, 16, 64, 0), (2 ** 40, 2 ** 20, 2 ** 10, 3)]:
        assert f(A, W_, None, Y_, *shape, None) == 1, shape
    assert f(A, W_, None, Y_, 1, 16, 64, 9, None) == 2          # more than 8 taps
    assert f(A, W_, None, A + 64, *ok, None) == 3               # y overlaps x
    assert f(A, W_, None, W_ - 64, *ok, None) == 3              # y overlaps w
    assert f(A, W_, Y_ + 8, Y_, *ok, None) == 3                 # y overlaps bias


def test_probe_library_builds_and_exports_its_entry():
    """The rate probes behind `bench.py --probe` build with the library
    (their own .so, outside the C ABI) and export ccp_run; a bad kind is
    refused before any CUDA call."""
    from spectral_sequence_mixing_b200 import build
    build.build()
    assert os.path.exists(build.PROBE_LIB)
    probe = ctypes.CDLL(build.PROBE_LIB)
    assert hasattr(probe, "ccp_run")
    probe.ccp_run.restype = ctypes.c_int
    probe.ccp_run.argtypes = [ctypes.c_int] * 4 + [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double)]
    ms, units = ctypes.c_float(0), ctypes.c_double(0)
    assert probe.ccp_run(99, 1, 32, 1, ctypes.byref(ms), ctypes.byref(units)) != 0
    assert probe.ccp_run(0, 0, 32, 1, ctypes.byref(ms), ctypes.byref(units)) != 0
