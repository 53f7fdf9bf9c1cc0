"""Exact tiled attention for B200 (sm_100a): thin Python binding over libfa.so.

This module only marshals arguments: it takes device pointers and the current
CUDA stream from torch tensors and calls the C ABI declared in include/fa.h.
Every step of the computation runs in the library's CUDA kernels; there is no
Python or CPU fallback.  If libfa.so is missing the call raises.

    o, lse = forward(q, k, v, causal=True)            # q, k, v: [B, H, N, d] on cuda
    dq, dk, dv = backward(q, k, v, o, do, lse, causal=True)
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = ["forward", "backward", "forward_gqa", "backward_gqa", "forward_qk", "backward_qk",
           "backward_noalloc", "FAError", "library_path", "load_library", "check_device_status",
           "workspace_size", "SYMBOLS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

# Entry points declared in include/fa.h, with ctypes signatures.
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SYMBOLS = {
    "fa_forward": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_forward_gqa": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_forward_qk": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_forward_fp32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_workspace_size": (_Z, [_I, _I, _I, _I]),
    "fa_backward": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_gqa": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_qk": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_fp32": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_noalloc": (_I, [_P] * 9 + [_I, _I, _I, _I, _F, _I, _P]),
    "fa_debug_wait_timeout": (_I, [_P]),
    "fa_check_device_status": (_I, [_P]),
    "fa_last_error": (ctypes.c_char_p, []),
    "fa_status_string": (ctypes.c_char_p, [_I]),
}


class FAError(RuntimeError):
    """A nonzero fa_status returned by the library."""

    def __init__(self, code, where):
        self.code = code
        detail = ""
        if code == 5:  # FA_ERR_CUDA
            detail = ": " + load_library().fa_last_error().decode()
        super().__init__(f"{where}: {status_string(code)}{detail} (fa_status {code})")


def library_path():
    return os.path.join(_HERE, "libfa.so")


def load_library():
    """Loads libfa.so (built in-tree by exact_tiled_attention_35_b200.build)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is not built; run `python -m exact_tiled_attention_35_b200.build`"
            )
        lib = ctypes.CDLL(path)
        for name, (res, args) in SYMBOLS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def status_string(code):
    return load_library().fa_status_string(int(code)).decode()


def _check(code, where):
    if code != 0:
        raise FAError(code, where)


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _require(ts, dtype, shape):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if t.dtype != dtype:
            raise ValueError(f"expected dtype {dtype}, got {t.dtype}")
        if tuple(t.shape) != shape:
            raise ValueError(f"expected shape {shape}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")


def forward(q, k, v, causal=False, scale=None, out=None, lse=None):
    """O = softmax(scale * Q K^T) V and the per-row logsumexp, via fa_forward.

    bf16 tensors run the tcgen05 kernel; fp32 tensors run fa_forward_fp32.
    Returns (o, lse) with lse float32 [B, H, N].
    """
    B, H, N, d = _shape(q)
    _require((q, k, v), q.dtype, (B, H, N, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _require((out,), q.dtype, (B, H, N, d))
    lib = load_library()
    fn = lib.fa_forward if q.dtype == torch.bfloat16 else lib.fa_forward_fp32
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q, k, v must be bfloat16 or float32")
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, scale, int(bool(causal)),
              _stream(q)), "fa_forward")
    return out, lse


def forward_gqa(q, k, v, causal=False, scale=None, out=None, lse=None):
    """Grouped-query / multi-query forward via fa_forward_gqa (bf16).

    q: [B, H, N, d]; k, v: [B, Hkv, N, d] with Hkv dividing H."""
    B, H, N, d = _shape(q)
    Hkv = int(k.shape[1])
    _require((q,), torch.bfloat16, (B, H, N, d))
    _require((k, v), torch.bfloat16, (B, Hkv, N, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(load_library().fa_forward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, N,
                                         d, scale, int(bool(causal)), _stream(q)), "fa_forward_gqa")
    return out, lse


def backward_gqa(q, k, v, o, do, lse, causal=False, scale=None, workspace=None):
    """dQ [B,H,N,d], dK and dV [B,Hkv,N,d] via fa_backward_gqa (bf16)."""
    B, H, N, d = _shape(q)
    Hkv = int(k.shape[1])
    _require((q, o, do), torch.bfloat16, (B, H, N, d))
    _require((k, v), torch.bfloat16, (B, Hkv, N, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(max(int(lib.fa_backward_workspace_size(B, H, N, d)), 16),
                                dtype=torch.uint8, device=q.device)
    _check(lib.fa_backward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), B, H, Hkv, N, d, scale,
                               int(bool(causal)), _stream(q)), "fa_backward_gqa")
    return dq, dk, dv


def forward_qk(q, k, v, causal=False, scale=None, out=None, lse=None):
    """Forward with separate query and key lengths via fa_forward_qk (bf16).

    q: [B, H, Nq, d]; k, v: [B, Hkv, Nk, d] with Hkv dividing H.  The causal
    mask is aligned at the bottom right (key j visible to query i iff
    j <= i + Nk - Nq); a query that sees no key gets O = 0 and LSE = -inf."""
    B, H, Nq, d = _shape(q)
    Hkv, Nk = int(k.shape[1]), int(k.shape[2])
    _require((q,), torch.bfloat16, (B, H, Nq, d))
    _require((k, v), torch.bfloat16, (B, Hkv, Nk, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _require((out,), torch.bfloat16, (B, H, Nq, d))
    _require((lse,), torch.float32, (B, H, Nq))
    _check(load_library().fa_forward_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, Nq,
                                        Nk, d, scale, int(bool(causal)), _stream(q)), "fa_forward_qk")
    return out, lse


def backward_qk(q, k, v, o, do, lse, causal=False, scale=None, workspace=None):
    """dQ [B,H,Nq,d], dK and dV [B,Hkv,Nk,d] via fa_backward_qk (bf16)."""
    B, H, Nq, d = _shape(q)
    Hkv, Nk = int(k.shape[1]), int(k.shape[2])
    _require((q, o, do), torch.bfloat16, (B, H, Nq, d))
    _require((k, v), torch.bfloat16, (B, Hkv, Nk, d))
    _require((lse,), torch.float32, (B, H, Nq))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(max(int(lib.fa_backward_workspace_size(B, H, Nq, d)), 16),
                                dtype=torch.uint8, device=q.device)
    _check(lib.fa_backward_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                              _ptr(dk), _ptr(dv), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), B, H, Hkv, Nq, Nk, d, scale,
                              int(bool(causal)), _stream(q)), "fa_backward_qk")
    return dq, dk, dv


def workspace_size(B, H, N, d):
    return int(load_library().fa_backward_workspace_size(B, H, N, d))


def backward(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None,
             workspace=None):
    """dQ, dK, dV of sum(O * dO) via fa_backward (bf16) or fa_backward_fp32."""
    B, H, N, d = _shape(q)
    _require((q, k, v, o, do), q.dtype, (B, H, N, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    lib = load_library()
    ws_bytes = int(lib.fa_backward_workspace_size(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    fn = lib.fa_backward if q.dtype == torch.bfloat16 else lib.fa_backward_fp32
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
              _ptr(workspace), workspace.numel() * workspace.element_size(), B, H, N, d, scale,
              int(bool(causal)), _stream(q)), "fa_backward")
    return dq, dk, dv


def backward_noalloc(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV via fa_backward_noalloc: no workspace, the library's fixed scratch array."""
    B, H, N, d = _shape(q)
    _require((q, k, v, o, do), torch.bfloat16, (B, H, N, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(load_library().fa_backward_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, N, d, scale, int(bool(causal)), _stream(q)), "fa_backward_noalloc")
    return dq, dk, dv


def check_device_status(device=None):
    """Synchronises the current stream and raises if a kernel's bounded wait ran out."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(load_library().fa_check_device_status(
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)), "fa_check_device_status")
