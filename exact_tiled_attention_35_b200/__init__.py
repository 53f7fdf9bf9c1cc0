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

__all__ = ["forward", "forward_fp8", "backward", "forward_gqa", "backward_gqa", "forward_qk", "backward_qk",
           "backward_stages", "backward_deterministic", "backward_noalloc", "STAGE_PREPROCESS",
           "STAGE_MAIN", "STAGE_DQ_CONVERT", "STAGE_DETERMINISTIC", "FAError", "library_path", "load_library", "check_device_status",
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
    "fa_forward_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _F, _F, _I, _P]),
    "fa_backward_workspace_size": (_Z, [_I, _I, _I, _I]),
    "fa_backward": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_gqa": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_qk": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_fp32": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_stages": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_backward_deterministic": (_I, [_P] * 9 + [_P, _Z, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_backward_noalloc": (_I, [_P] * 9 + [_I, _I, _I, _I, _F, _I, _P]),
    "fa_debug_wait_timeout": (_I, [_P]),
    "fa_debug_hold_scheduler": (_I, [_P]),
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
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _require(ts, dtype, shape, what="tensor"):
    """Every tensor in ts: a contiguous tensor of this dtype and shape."""
    for t in ts:
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{what}: expected a torch tensor")
        if t.dtype != dtype:
            raise ValueError(f"{what}: expected dtype {dtype}, got {t.dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{what}: tensors must be contiguous")


def _on_device(*ts):
    """All tensors on one CUDA device (checked after every shape and dtype)."""
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _out(t, like, shape=None, dtype=None):
    if t is not None:
        return t
    if shape is None:
        return torch.empty_like(like)
    return torch.empty(shape, dtype=dtype, device=like.device)


def _workspace(workspace, need, device):
    if workspace is None:
        return torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or workspace.device != device:
        raise ValueError(f"workspace: expected a CUDA tensor on {device}")
    if not workspace.is_contiguous():
        raise ValueError("workspace: must be contiguous")
    return workspace


def _nbytes(t):
    return t.numel() * t.element_size()


def forward(q, k, v, causal=False, scale=None, out=None, lse=None):
    """O = softmax(scale * Q K^T) V and the per-row logsumexp, via fa_forward.

    bf16 tensors run the tcgen05 kernel; fp32 tensors run fa_forward_fp32.
    Returns (o, lse) with lse float32 [B, H, N].
    """
    B, H, N, d = _shape(q)
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q, k, v must be bfloat16 or float32")
    _require((q, k, v), q.dtype, (B, H, N, d), "q, k, v")
    scale = _scale(scale, d)
    out = _out(out, q)
    lse = _out(lse, q, (B, H, N), torch.float32)
    _require((out,), q.dtype, (B, H, N, d), "out")
    _require((lse,), torch.float32, (B, H, N), "lse")
    _on_device(q, k, v, out, lse)
    lib = load_library()
    fn = lib.fa_forward if q.dtype == torch.bfloat16 else lib.fa_forward_fp32
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, scale, int(bool(causal)),
              _stream(q)), "fa_forward")
    return out, lse


def forward_gqa(q, k, v, causal=False, scale=None, out=None, lse=None):
    """Grouped-query / multi-query forward via fa_forward_gqa (bf16).

    q: [B, H, N, d]; k, v: [B, Hkv, N, d] with Hkv dividing H."""
    B, H, N, d = _shape(q)
    Hkv = int(_shape(k)[1])
    _require((q,), torch.bfloat16, (B, H, N, d), "q")
    _require((k, v), torch.bfloat16, (B, Hkv, N, d), "k, v")
    scale = _scale(scale, d)
    out = _out(out, q)
    lse = _out(lse, q, (B, H, N), torch.float32)
    _require((out,), torch.bfloat16, (B, H, N, d), "out")
    _require((lse,), torch.float32, (B, H, N), "lse")
    _on_device(q, k, v, out, lse)
    _check(load_library().fa_forward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, N,
                                         d, scale, int(bool(causal)), _stream(q)), "fa_forward_gqa")
    return out, lse


def forward_qk(q, k, v, causal=False, scale=None, out=None, lse=None):
    """Forward with separate query and key lengths via fa_forward_qk (bf16).

    q: [B, H, Nq, d]; k, v: [B, Hkv, Nk, d] with Hkv dividing H.  The causal
    mask is aligned at the bottom right (key j visible to query i iff
    j <= i + Nk - Nq); a query that sees no key gets O = 0 and LSE = -inf."""
    B, H, Nq, d = _shape(q)
    _, Hkv, Nk, _ = _shape(k)
    _require((q,), torch.bfloat16, (B, H, Nq, d), "q")
    _require((k, v), torch.bfloat16, (B, Hkv, Nk, d), "k, v")
    scale = _scale(scale, d)
    out = _out(out, q)
    lse = _out(lse, q, (B, H, Nq), torch.float32)
    _require((out,), torch.bfloat16, (B, H, Nq, d), "out")
    _require((lse,), torch.float32, (B, H, Nq), "lse")
    _on_device(q, k, v, out, lse)
    _check(load_library().fa_forward_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, Nq,
                                        Nk, d, scale, int(bool(causal)), _stream(q)), "fa_forward_qk")
    return out, lse


def forward_fp8(q, k, v, q_descale, k_descale, v_descale, causal=False, scale=None, out=None,
                lse=None):
    """FP8 forward via fa_forward_fp8: q [B,H,Nq,d], k and v [B,Hkv,Nk,d] stored as
    torch.float8_e4m3fn with per-tensor descales (the values they stand for are
    descale * stored).  Returns (o bf16 [B,H,Nq,d], lse float32 [B,H,Nq])."""
    B, H, Nq, d = _shape(q)
    _, Hkv, Nk, _ = _shape(k)
    f8 = torch.float8_e4m3fn
    _require((q,), f8, (B, H, Nq, d), "q")
    _require((k, v), f8, (B, Hkv, Nk, d), "k, v")
    scale = _scale(scale, d)
    out = _out(out, q, (B, H, Nq, d), torch.bfloat16)
    lse = _out(lse, q, (B, H, Nq), torch.float32)
    _require((out,), torch.bfloat16, (B, H, Nq, d), "out")
    _require((lse,), torch.float32, (B, H, Nq), "lse")
    _on_device(q, k, v, out, lse)
    _check(load_library().fa_forward_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, Nq,
                                         Nk, d, scale, float(q_descale), float(k_descale),
                                         float(v_descale), int(bool(causal)), _stream(q)),
           "fa_forward_fp8")
    return out, lse


def _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, dtype):
    """Shapes of a backward call, checked; returns (B, H, Hkv, Nq, Nk, d, dq, dk, dv)."""
    B, H, Nq, d = _shape(q)
    _, Hkv, Nk, _ = _shape(k)
    dev = q.device
    _require((q, o, do), dtype, (B, H, Nq, d), "q, o, do")
    _require((k, v), dtype, (B, Hkv, Nk, d), "k, v")
    _require((lse,), torch.float32, (B, H, Nq), "lse")
    dq, dk, dv = _out(dq, q), _out(dk, k), _out(dv, v)
    _require((dq,), dtype, (B, H, Nq, d), "dq")
    _require((dk, dv), dtype, (B, Hkv, Nk, d), "dk, dv")
    _on_device(q, k, v, o, do, lse, dq, dk, dv)
    return B, H, Hkv, Nq, Nk, d, dq, dk, dv


def backward(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None,
             workspace=None):
    """dQ, dK, dV of sum(O * dO) via fa_backward (bf16) or fa_backward_fp32."""
    if not isinstance(q, torch.Tensor) or q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q must be a bfloat16 or float32 tensor")
    B, H, Hkv, Nq, Nk, d, dq, dk, dv = _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, q.dtype)
    if Hkv != H or Nk != Nq:
        raise ValueError("k, v must have the shape of q (use backward_gqa / backward_qk)")
    scale = _scale(scale, d)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_backward_workspace_size(B, H, Nq, d)), q.device)
    fn = lib.fa_backward if q.dtype == torch.bfloat16 else lib.fa_backward_fp32
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
              _ptr(workspace), _nbytes(workspace), B, H, Nq, d, scale, int(bool(causal)), _stream(q)),
           "fa_backward")
    return dq, dk, dv


def backward_gqa(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None,
                 workspace=None):
    """dQ [B,H,N,d], dK and dV [B,Hkv,N,d] via fa_backward_gqa (bf16)."""
    B, H, Hkv, Nq, Nk, d, dq, dk, dv = _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, torch.bfloat16)
    if Nk != Nq:
        raise ValueError("k, v must have the length of q (use backward_qk)")
    scale = _scale(scale, d)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_backward_workspace_size(B, H, Nq, d)), q.device)
    _check(lib.fa_backward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(workspace), _nbytes(workspace), B, H, Hkv, Nq, d,
                               scale, int(bool(causal)), _stream(q)), "fa_backward_gqa")
    return dq, dk, dv


def backward_qk(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None,
                workspace=None):
    """dQ [B,H,Nq,d], dK and dV [B,Hkv,Nk,d] via fa_backward_qk (bf16)."""
    B, H, Hkv, Nq, Nk, d, dq, dk, dv = _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, torch.bfloat16)
    scale = _scale(scale, d)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_backward_workspace_size(B, H, Nq, d)), q.device)
    _check(lib.fa_backward_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                              _ptr(dk), _ptr(dv), _ptr(workspace), _nbytes(workspace), B, H, Hkv, Nq, Nk,
                              d, scale, int(bool(causal)), _stream(q)), "fa_backward_qk")
    return dq, dk, dv


STAGE_PREPROCESS, STAGE_MAIN, STAGE_DQ_CONVERT, STAGE_DETERMINISTIC = 1, 2, 4, 8


def backward_deterministic(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None,
                           workspace=None):
    """dQ [B,H,Nq,d], dK and dV [B,Hkv,Nk,d] via fa_backward_deterministic (bf16):
    the same results as backward_qk, reproducible bit for bit (dQ by a separate
    pass over the key tiles in a fixed order)."""
    B, H, Hkv, Nq, Nk, d, dq, dk, dv = _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, torch.bfloat16)
    scale = _scale(scale, d)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_backward_workspace_size(B, H, Nq, d)), q.device)
    _check(lib.fa_backward_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                                         _ptr(dk), _ptr(dv), _ptr(workspace), _nbytes(workspace), B, H, Hkv,
                                         Nq, Nk, d, scale, int(bool(causal)), _stream(q)),
           "fa_backward_deterministic")
    return dq, dk, dv


def backward_stages(stages, q, k, v, o, do, lse, dq, dk, dv, workspace, causal=False, scale=None):
    """Runs the selected stages of the bf16 backward pass via fa_backward_stages.

    stages: OR of STAGE_PREPROCESS, STAGE_MAIN, STAGE_DQ_CONVERT; run them in that
    order with the same tensors and workspace (fa_backward runs all three)."""
    B, H, Hkv, Nq, Nk, d, dq, dk, dv = _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, torch.bfloat16)
    scale = _scale(scale, d)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_backward_workspace_size(B, H, Nq, d)), q.device)
    _check(lib.fa_backward_stages(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                                  _ptr(dk), _ptr(dv), _ptr(workspace), _nbytes(workspace), B, H, Hkv, Nq,
                                  Nk, d, scale, int(bool(causal)), int(stages), _stream(q)),
           "fa_backward_stages")
    return dq, dk, dv


def workspace_size(B, H, N, d):
    return int(load_library().fa_backward_workspace_size(B, H, N, d))


def backward_noalloc(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV via fa_backward_noalloc: no workspace, the library's fixed scratch array."""
    B, H, Hkv, Nq, Nk, d, dq, dk, dv = _bwd_tensors(q, k, v, o, do, lse, dq, dk, dv, torch.bfloat16)
    if Hkv != H or Nk != Nq:
        raise ValueError("k, v must have the shape of q")
    scale = _scale(scale, d)
    _check(load_library().fa_backward_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, Nq, d, scale, int(bool(causal)), _stream(q)), "fa_backward_noalloc")
    return dq, dk, dv


def check_device_status(device=None):
    """Synchronises the current stream and raises if a kernel's bounded wait ran out."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(load_library().fa_check_device_status(
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)), "fa_check_device_status")
