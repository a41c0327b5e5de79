"""B200 (sm_100a) causal sequence convolution.

    r[b, t, d] = sum_{j<=t} v[b, j, d] * g[b, t-j, d]

computed as in Caracal: Causal Architecture via Spectral Mixing (Multi-Head
Fourier module: zero-pad to 2L, FFT, pointwise product, inverse FFT,
truncate to L), the gate stream of the same block (sigmoid and the head-grouped causal
Conv1d_G2, on the tensor cores), plus the exact number-theoretic variant of "Catastrophic
Token Leakage in Convolutional Sequence Modeling and How to Mitigate It".

This module is argument marshalling only: every step of the computation runs
in the CUDA kernels of ``libcausalconv.so`` behind the C ABI declared in
``include/causalconv.h``.  PyTorch supplies device memory and the stream.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (CC_DTYPE_BF16, CC_DTYPE_F32, CC_DTYPE_I32, CausalConvError, load, strerror)

__all__ = [
    "causal_fftconv_f32", "causal_fftconv_bf16", "causal_ntt_conv_i32", "causal_conv", "causal_conv_bwd",
    "causal_conv_decode", "decode_workspace_bytes",
    "causal_conv_from_host", "workspace_bytes", "fast_workspace_bytes", "max_len", "ntt_params", "strerror",
    "fault_flags", "mhf_gate", "mhf_gated_conv", "mhf_gated_conv_workspace_bytes", "causal_dwconv",
    "CausalConvError", "CC_DTYPE_F32", "CC_DTYPE_BF16", "CC_DTYPE_I32",
]

_DT = {torch.float32: CC_DTYPE_F32, torch.bfloat16: CC_DTYPE_BF16, torch.int32: CC_DTYPE_I32}
_FN = {CC_DTYPE_F32: "causal_fftconv_f32", CC_DTYPE_BF16: "causal_fftconv_bf16", CC_DTYPE_I32: "causal_ntt_conv_i32"}


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != 3:
        raise ValueError(f"{name} must be [B, L, D], got shape {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} shape {tuple(t.shape)} != {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous ([B, L, D] row-major)")


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def fast_workspace_bytes(dtype: torch.dtype, B: int, L: int, D: int) -> int:
    """Bytes of the optional workspace that lets long rows (4096 < L <= 65536)
    take the four-step path through device memory; 0 where it does not apply."""
    return int(load().causal_conv_fast_workspace_bytes(_DT[dtype], B, L, D))


_ONE_CTA_ROW = 4096  # rows up to this length never use the optional workspace


def _workspace(workspace, dtype_code: int, B: int, L: int, D: int, device):
    """(pointer, bytes, tensor allocated here or None) of the workspace: the
    caller's; with none given, one of the optional four-step size taken from
    the torch allocator when that path applies (the single-pass path when the
    allocator has no room for it).  A tensor of 0 bytes selects the
    single-pass path."""
    own = None
    if workspace is None:
        if L <= _ONE_CTA_ROW or dtype_code == CC_DTYPE_I32:
            return None, 0, None
        n = int(load().causal_conv_fast_workspace_bytes(dtype_code, B, L, D))
        if n == 0:
            return None, 0, None
        try:
            workspace = own = torch.empty(n, dtype=torch.uint8, device=device)
        except torch.cuda.OutOfMemoryError:
            return None, 0, None
    nbytes = workspace.numel() * workspace.element_size()
    return (workspace.data_ptr() if nbytes else None), nbytes, own


def _record(stream, *tensors):
    """Tensors allocated here (on the current stream) and handed to the
    library's work on `stream`: tell the caching allocator, so their memory is
    not given out again before that stream has finished with it."""
    if stream is None:
        return
    for t in tensors:
        if t is not None and stream != torch.cuda.current_stream(t.device):
            t.record_stream(stream)


def _run(dtype_code: int, v: torch.Tensor, g: torch.Tensor, out, workspace, stream):
    dtype = v.dtype
    _check(v, "v", dtype)
    _check(g, "g", dtype, v.shape)
    if not v.is_cuda or not g.is_cuda or v.device != g.device:
        raise ValueError("v and g must be CUDA tensors on the same device")
    B, L, D = v.shape
    own_out = out is None
    if own_out:
        out = torch.empty_like(v)
    _check(out, "out", dtype, v.shape)
    ws_ptr, ws_bytes, own_ws = _workspace(workspace, dtype_code, B, L, D, v.device)
    fn = getattr(load(), _FN[dtype_code])
    if v.device.index == torch.cuda.current_device():
        st = fn(v.data_ptr(), g.data_ptr(), out.data_ptr(), B, L, D, ws_ptr, ws_bytes, _stream_ptr(stream))
    else:  # the library works on the current device: switch to the tensors' one (and its stream)
        with torch.cuda.device(v.device):
            st = fn(v.data_ptr(), g.data_ptr(), out.data_ptr(), B, L, D, ws_ptr, ws_bytes, _stream_ptr(stream))
    _record(stream, own_ws, out if own_out else None)
    if st != 0:
        raise CausalConvError(st, _FN[dtype_code])
    return out


def causal_fftconv_f32(v: torch.Tensor, g: torch.Tensor, out: torch.Tensor | None = None, workspace=None,
                       stream=None) -> torch.Tensor:
    """float32 [B, L, D] -> float32 [B, L, D] causal convolution (fused FFT kernel)."""
    return _run(CC_DTYPE_F32, v, g, out, workspace, stream)


def causal_fftconv_bf16(v: torch.Tensor, g: torch.Tensor, out: torch.Tensor | None = None, workspace=None,
                        stream=None) -> torch.Tensor:
    """bfloat16 [B, L, D] in/out, float32 transform arithmetic."""
    return _run(CC_DTYPE_BF16, v, g, out, workspace, stream)


def causal_ntt_conv_i32(v: torch.Tensor, g: torch.Tensor, out: torch.Tensor | None = None, workspace=None,
                        stream=None) -> torch.Tensor:
    """int32 [B, L, D] exact causal convolution (NTT mod 2013265921, centered residue)."""
    return _run(CC_DTYPE_I32, v, g, out, workspace, stream)


def causal_conv(v: torch.Tensor, g: torch.Tensor, out=None, workspace=None, stream=None) -> torch.Tensor:
    """Dispatch on dtype: float32 / bfloat16 -> FFT path, int32 -> NTT path."""
    if v.dtype not in _DT:
        raise TypeError(f"unsupported dtype {v.dtype}")
    return _run(_DT[v.dtype], v, g, out, workspace, stream)


def causal_conv_bwd(dr: torch.Tensor, v: torch.Tensor, g: torch.Tensor, dv=None, dg=None, workspace=None,
                    stream=None):
    """Gradients (dv, dg) of the causal convolution given dr = dLoss/dr
    (float32 or bfloat16 [B, L, D]):  dv_j = sum_{t>=j} dr_t g_{t-j},
    dg_k = sum_{t>=k} dr_t v_{t-k}."""
    dtype = v.dtype
    if dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"unsupported dtype {dtype}")
    for name, t in (("dr", dr), ("v", v), ("g", g)):
        _check(t, name, dtype, v.shape)
        if not t.is_cuda or t.device != v.device:
            raise ValueError("dr, v, g must be CUDA tensors on the same device")
    own = [dv is None, dg is None]
    dv = torch.empty_like(v) if dv is None else dv
    dg = torch.empty_like(v) if dg is None else dg
    _check(dv, "dv", dtype, v.shape)
    _check(dg, "dg", dtype, v.shape)
    B, L, D = v.shape
    ws_ptr, ws_bytes, own_ws = _workspace(workspace, _DT[dtype], B, L, D, v.device)
    fn = "causal_fftconv_bwd_f32" if dtype == torch.float32 else "causal_fftconv_bwd_bf16"
    with torch.cuda.device(v.device):
        st = getattr(load(), fn)(dr.data_ptr(), v.data_ptr(), g.data_ptr(), dv.data_ptr(), dg.data_ptr(), B, L, D,
                                 ws_ptr, ws_bytes, _stream_ptr(stream))
    _record(stream, own_ws, dv if own[0] else None, dg if own[1] else None)
    if st != 0:
        raise CausalConvError(st, fn)
    return dv, dg


def decode_workspace_bytes(dtype: torch.dtype, B: int, D: int, t: int) -> int:
    return int(load().causal_conv_decode_workspace_bytes(_DT[dtype], B, D, t))


def causal_conv_decode(v_cache: torch.Tensor, g_cache: torch.Tensor, t: int, out=None, workspace=None,
                       stream=None) -> torch.Tensor:
    """Output [B, D] of position t from [B, Lcap, D] caches:
    r[b, d] = sum_{j<=t} v[b, j, d] g[b, t-j, d].  `workspace` (a uint8 CUDA
    tensor of decode_workspace_bytes bytes) is allocated here when not given."""
    dtype = v_cache.dtype
    if dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"unsupported dtype {dtype}")
    _check(v_cache, "v_cache", dtype)
    _check(g_cache, "g_cache", dtype, v_cache.shape)
    B, Lcap, D = v_cache.shape
    own_out, own_ws = out is None, workspace is None
    if own_out:
        out = torch.empty((B, D), dtype=dtype, device=v_cache.device)
    nbytes = decode_workspace_bytes(dtype, B, D, t)
    if own_ws:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=v_cache.device)
    fn = "causal_conv_decode_f32" if dtype == torch.float32 else "causal_conv_decode_bf16"
    with torch.cuda.device(v_cache.device):
        st = getattr(load(), fn)(v_cache.data_ptr(), g_cache.data_ptr(), out.data_ptr(), B, Lcap, D, int(t),
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream))
    _record(stream, workspace if own_ws else None, out if own_out else None)
    if st != 0:
        raise CausalConvError(st, fn)
    return out


def causal_conv_from_host(v_host: torch.Tensor, g_host: torch.Tensor, r_host: torch.Tensor, v_dev: torch.Tensor,
                          g_dev: torch.Tensor, r_dev: torch.Tensor, workspace=None, stream=None) -> None:
    """Host buffers in and out (pinned for overlap); the library enqueues the
    H2D copies, the convolution and the D2H copy on ``stream``.  Caller
    synchronises before reading ``r_host``."""
    dtype = v_host.dtype
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    for name, t in (("v_host", v_host), ("g_host", g_host), ("r_host", r_host), ("v_dev", v_dev), ("g_dev", g_dev),
                    ("r_dev", r_dev)):
        _check(t, name, dtype, v_host.shape)
    if v_host.is_cuda or g_host.is_cuda or r_host.is_cuda:
        raise ValueError("*_host tensors must live in host memory")
    B, L, D = v_host.shape
    ws_ptr, ws_bytes, own_ws = _workspace(workspace, _DT[dtype], B, L, D, v_dev.device)
    with torch.cuda.device(v_dev.device):
        st = load().causal_conv_from_host(_DT[dtype], v_host.data_ptr(), g_host.data_ptr(), r_host.data_ptr(),
                                          v_dev.data_ptr(), g_dev.data_ptr(), r_dev.data_ptr(), B, L, D, ws_ptr,
                                          ws_bytes, _stream_ptr(stream))
    _record(stream, own_ws)
    if st != 0:
        raise CausalConvError(st, "causal_conv_from_host")


def workspace_bytes(dtype: torch.dtype, B: int, L: int, D: int) -> int:
    return int(load().causal_conv_workspace_bytes(_DT[dtype], B, L, D))


def max_len(dtype: torch.dtype) -> int:
    return int(load().causal_conv_max_len(_DT[dtype]))


def ntt_params(N: int) -> dict:
    out = (ctypes.c_uint32 * 6)()
    st = load().causal_ntt_params(N, out)
    if st != 0:
        raise CausalConvError(st, "causal_ntt_params")
    return dict(zip(("p", "omega", "omega_inv", "n_inv", "p_inv_mod_2_32", "r2_mod_p"), list(out)))


def fault_flags(device: int | None = None, clear: bool = False) -> int:
    """The per-device word of kernel waits that ran out of time (0 = none);
    synchronises the device."""
    dev = torch.cuda.current_device() if device is None else int(device)
    out = ctypes.c_uint(0)
    st = load().causal_conv_fault_flags(dev, ctypes.byref(out), 1 if clear else 0)
    if st != 0:
        raise CausalConvError(st, "causal_conv_fault_flags")
    return int(out.value)


# ------------------------------------------------------------------ MHF gate stream
_GATE_FN = {torch.float32: "causal_mhf_gate_f32", torch.bfloat16: "causal_mhf_gate_bf16"}
_GATED_FN = {torch.float32: "causal_mhf_gated_conv_f32", torch.bfloat16: "causal_mhf_gated_conv_bf16"}


def _check_gate_params(w: torch.Tensor, bias, D: int, n_head: int, device):
    if not isinstance(w, torch.Tensor) or w.dtype != torch.float32 or w.dim() != 3:
        raise TypeError("w must be a float32 tensor [D, D/n_head, K]")
    if n_head < 1 or D % n_head or tuple(w.shape[:2]) != (D, D // n_head):
        raise ValueError(f"w shape {tuple(w.shape)} does not fit D={D}, n_head={n_head}")
    if not w.is_contiguous() or w.device != device:
        raise ValueError("w must be contiguous and on the device of a")
    if bias is not None:
        if not isinstance(bias, torch.Tensor) or bias.dtype != torch.float32 or tuple(bias.shape) != (D,):
            raise TypeError("bias must be a float32 tensor [D] or None")
        if not bias.is_contiguous() or bias.device != device:
            raise ValueError("bias must be contiguous and on the device of a")
    return int(w.shape[2])


def mhf_gate(a: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None, n_head: int, out=None,
             stream=None) -> torch.Tensor:
    """g = Conv1d_G2(sigmoid(a)): the head-grouped causal convolution of the
    gate stream (w: [D, D/n_head, K] float32, bias: [D] float32 or None);
    a and the result are [B, L, D] float32 or bfloat16."""
    if a.dtype not in _GATE_FN:
        raise TypeError(f"unsupported dtype {a.dtype}")
    _check(a, "a", a.dtype)
    if not a.is_cuda:
        raise ValueError("a must be a CUDA tensor")
    B, L, D = a.shape
    K = _check_gate_params(w, bias, D, n_head, a.device)
    own_out = out is None
    if own_out:
        out = torch.empty_like(a)
    _check(out, "out", a.dtype, a.shape)
    fn = getattr(load(), _GATE_FN[a.dtype])
    with torch.cuda.device(a.device):
        st = fn(a.data_ptr(), w.data_ptr(), bias.data_ptr() if bias is not None else None, out.data_ptr(), B, L, D,
                n_head, K, _stream_ptr(stream))
    _record(stream, out if own_out else None)
    if st != 0:
        raise CausalConvError(st, _GATE_FN[a.dtype])
    return out


def mhf_gated_conv_workspace_bytes(dtype: torch.dtype, B: int, L: int, D: int) -> int:
    return int(load().causal_mhf_gated_conv_workspace_bytes(_DT[dtype], B, L, D))


def mhf_gated_conv(v: torch.Tensor, a: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None, n_head: int,
                   out=None, workspace=None, stream=None) -> torch.Tensor:
    """r = causal_conv(v, mhf_gate(a, w, bias, n_head)); the gate goes through
    ``workspace`` (a device tensor of at least mhf_gated_conv_workspace_bytes
    bytes; taken from the torch allocator when None)."""
    if v.dtype not in _GATED_FN:
        raise TypeError(f"unsupported dtype {v.dtype}")
    _check(v, "v", v.dtype)
    _check(a, "a", v.dtype, v.shape)
    if not v.is_cuda or v.device != a.device:
        raise ValueError("v and a must be CUDA tensors on the same device")
    B, L, D = v.shape
    K = _check_gate_params(w, bias, D, n_head, v.device)
    own_out, own_ws = out is None, workspace is None
    if own_out:
        out = torch.empty_like(v)
    _check(out, "out", v.dtype, v.shape)
    if own_ws:
        workspace = torch.empty(mhf_gated_conv_workspace_bytes(v.dtype, B, L, D), dtype=torch.uint8,
                                device=v.device)
    nbytes = workspace.numel() * workspace.element_size()
    fn = getattr(load(), _GATED_FN[v.dtype])
    with torch.cuda.device(v.device):
        st = fn(v.data_ptr(), a.data_ptr(), w.data_ptr(), bias.data_ptr() if bias is not None else None,
                out.data_ptr(), B, L, D, n_head, K, workspace.data_ptr() if nbytes else None, nbytes,
                _stream_ptr(stream))
    _record(stream, workspace if own_ws else None, out if own_out else None)
    if st != 0:
        raise CausalConvError(st, _GATED_FN[v.dtype])
    return out


# ------------------------------------------------------------------ depthwise convolution
_DW_FN = {torch.float32: "causal_dwconv_f32", torch.bfloat16: "causal_dwconv_bf16"}


def causal_dwconv(x: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None = None, out=None,
                  stream=None) -> torch.Tensor:
    """y = the causal depthwise convolution of x ([B, L, D] float32 / bfloat16)
    with w ([D, K] or [D, 1, K] float32) and bias ([D] float32 or None)."""
    if x.dtype not in _DW_FN:
        raise TypeError(f"unsupported dtype {x.dtype}")
    _check(x, "x", x.dtype)
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    B, L, D = x.shape
    if not isinstance(w, torch.Tensor) or w.dtype != torch.float32:
        raise TypeError("w must be a float32 tensor [D, K] or [D, 1, K]")
    if w.dim() == 3 and w.shape[1] == 1:
        w = w.reshape(w.shape[0], w.shape[2])
    if w.dim() != 2 or w.shape[0] != D or not w.is_contiguous() or w.device != x.device:
        raise ValueError(f"w must be contiguous [D={D}, K] on the device of x, got {tuple(w.shape)}")
    if bias is not None and (not isinstance(bias, torch.Tensor) or bias.dtype != torch.float32
                             or tuple(bias.shape) != (D,) or not bias.is_contiguous() or bias.device != x.device):
        raise ValueError("bias must be a contiguous float32 tensor [D] on the device of x, or None")
    own_out = out is None
    if own_out:
        out = torch.empty_like(x)
    _check(out, "out", x.dtype, x.shape)
    fn = getattr(load(), _DW_FN[x.dtype])
    with torch.cuda.device(x.device):
        st = fn(x.data_ptr(), w.data_ptr(), bias.data_ptr() if bias is not None else None, out.data_ptr(), B, L, D,
                int(w.shape[1]), _stream_ptr(stream))
    _record(stream, out if own_out else None)
    if st != 0:
        raise CausalConvError(st, _DW_FN[x.dtype])
    return out
