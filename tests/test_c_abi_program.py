"""The C ABI from a C program (tests/c_abi/abi_check.c): the header compiles
as C99 with warnings as errors, the host-only entry points answer from C, and
on a GPU a float32 convolution called from C matches the oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from conftest import ROOT, cuda_available

SRC = os.path.join(ROOT, "tests", "c_abi", "abi_check.c")
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "spectral_sequence_mixing_b200")
CUDA = "/usr/local/cuda"
BUILD = os.path.join(ROOT, "tests", "c_abi", "_build")  # in-tree, git-ignored


def _compile(cuda: bool):
    from spectral_sequence_mixing_b200 import build
    build.build()
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    os.makedirs(BUILD, exist_ok=True)
    exe = os.path.join(BUILD, "abi_check_cuda" if cuda else "abi_check")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, SRC, "-o", exe,
           "-L", PKG, "-lcausalconv", f"-Wl,-rpath,{PKG}", "-lm"]
    if cuda:
        cmd[1:1] = ["-DABI_CHECK_CUDA", "-I", os.path.join(CUDA, "include")]
        cmd += ["-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_header_is_c99_and_host_queries_answer_from_c():
    exe = _compile(cuda=False)
    out = subprocess.run([exe, "host"], check=True, capture_output=True, text=True).stdout.splitlines()
    got = {line.split()[0]: line.split()[1:] for line in out}
    st, p, w, winv, ninv, pinv, r2 = (int(x) for x in got["ntt_params"])
    P = 2013265921
    assert st == 0 and p == P
    assert pow(w, 16384, P) == 1 and pow(w, 8192, P) == P - 1      # order exactly 16384
    assert w * winv % P == 1 and 16384 * ninv % P == 1
    assert (P * pinv) % 2 ** 32 == 1 and r2 == pow(2, 64, P)
    assert got["max_len"] == ["65536", "65536", "8192"]
    assert got["workspace"] == ["0"]
    assert got["fast_workspace"] == ["0", str(8 * (131072 * 8 + 64 * 8 + 8))]  # 8 rows of the four-step path
    assert got["strerror"] and got["null_args"] == ["1"]


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA GPU")
def test_device_convolution_called_from_c():
    import oracle
    from gpu_helpers import F32_TOL, float_violations
    exe = _compile(cuda=True)
    B, L, D = 2, 300, 8
    base = os.path.join(BUILD, "conv_out")
    subprocess.run([exe, "run", str(B), str(L), str(D), base], check=True, capture_output=True, text=True)
    rd = lambda ext: np.fromfile(f"{base}.{ext}", dtype=np.float32).reshape(B, L, D)  # noqa: E731
    v, g, r = rd("v"), rd("g"), rd("r")
    ref, den = oracle.causal_conv(v, g)
    n_bad, worst = float_violations(r, ref, den, F32_TOL)
    assert n_bad == 0, f"{n_bad} elements beyond the fp32 bound, worst ratio {worst:.3g}"
