"""ctypes loader for ``libcausalconv.so`` (the sm_100a C-ABI library).

Fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcausalconv.so")

CC_OK, CC_ERR_INVALID_ARG, CC_ERR_UNSUPPORTED, CC_ERR_ALIAS, CC_ERR_WORKSPACE, CC_ERR_CUDA, CC_ERR_NOT_DEVICE = range(7)
CC_ERR_SCRATCH_LIMIT = 7
CC_DTYPE_F32, CC_DTYPE_BF16, CC_DTYPE_I32 = 0, 1, 2

# name -> (restype, argtypes); every symbol include/causalconv.h declares.
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_CONV = [_P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]
SIGNATURES = {
    "causal_fftconv_f32": (ctypes.c_int, _CONV),
    "causal_fftconv_bf16": (ctypes.c_int, _CONV),
    "causal_ntt_conv_i32": (ctypes.c_int, _CONV),
    "causal_fftconv_bwd_f32": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_fftconv_bwd_bf16": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_conv_decode_f32": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_conv_decode_bf16": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_conv_decode_workspace_bytes": (_SZ, [ctypes.c_int, _I64, _I64, _I64]),
    "causal_conv_decode_f32_noalloc": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "causal_conv_from_host": (ctypes.c_int, [ctypes.c_int, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_conv_workspace_bytes": (_SZ, [ctypes.c_int, _I64, _I64, _I64]),
    "causal_conv_fast_workspace_bytes": (_SZ, [ctypes.c_int, _I64, _I64, _I64]),
    "causal_conv_max_len": (_I64, [ctypes.c_int]),
    "causal_conv_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "causal_ntt_params": (ctypes.c_int, [_I64, ctypes.POINTER(ctypes.c_uint32)]),
    "causal_conv_fault_flags": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_uint), ctypes.c_int]),
    "causal_mhf_gate_f32": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P]),
    "causal_mhf_gate_bf16": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P]),
    "causal_mhf_gated_conv_f32": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_mhf_gated_conv_bf16": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "causal_mhf_gated_conv_workspace_bytes": (_SZ, [ctypes.c_int, _I64, _I64, _I64]),
    "causal_dwconv_f32": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "causal_dwconv_bf16": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
}

_lib = None


class CausalConvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} (status {status})")


def load(path: str = LIB_PATH):
    """Load the library once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m spectral_sequence_mixing_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return load().causal_conv_strerror(int(status)).decode()
