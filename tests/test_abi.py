"""Host-only checks of the C ABI: the library loads, exports every entry point
declared in include/fa.h, and rejects bad arguments before touching a device."""

import ctypes
import os
import re

import pytest

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA, TIMEOUT = range(7)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert set(declared_functions()) == set(fa.SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(7):
        assert fa.status_string(code)
    assert fa.status_string(99) == "unknown status"


P = ctypes.c_void_p
GOOD = [P(0x10000), P(0x20000), P(0x30000), P(0x40000), P(0x50000)]


def fwd(lib, ptrs, B=1, H=1, N=128, d=128, scale=0.125, causal=0, fn="fa_forward"):
    return getattr(lib, fn)(*ptrs, B, H, N, d, scale, causal, None)


@pytest.mark.parametrize("fn", ["fa_forward", "fa_forward_fp32"])
def test_forward_rejects_bad_arguments(lib, fn):
    for i in range(5):
        ptrs = list(GOOD)
        ptrs[i] = None
        assert fwd(lib, ptrs, fn=fn) == INVALID
    ptrs = list(GOOD)
    ptrs[2] = P(0x30008)
    assert fwd(lib, ptrs, fn=fn) == MISALIGNED
    assert fwd(lib, GOOD, d=96, fn=fn) == UNSUPPORTED
    assert fwd(lib, GOOD, d=256, fn=fn) == UNSUPPORTED
    assert fwd(lib, GOOD, N=0, fn=fn) == INVALID
    assert fwd(lib, GOOD, B=0, fn=fn) == INVALID
    assert fwd(lib, GOOD, H=-1, fn=fn) == INVALID
    assert fwd(lib, GOOD, scale=0.0, fn=fn) == INVALID
    assert fwd(lib, GOOD, scale=float("nan"), fn=fn) == INVALID
    assert fwd(lib, GOOD, scale=float("inf"), fn=fn) == INVALID


def test_workspace_size(lib):
    # LSE*log2(e) and D padded to 128-row tiles, an fp32 dQ accumulator and the
    # main kernel's work-item counters, each segment rounded up to 256 bytes
    def expect(B, H, N, d):
        up = lambda x: (x + 255) // 256 * 256
        npad = (N + 127) // 128 * 128
        return 2 * up(B * H * npad * 4) + up(B * H * N * d * 4) + 256

    assert lib.fa_backward_workspace_size(2, 16, 2048, 128) == expect(2, 16, 2048, 128)
    assert lib.fa_backward_workspace_size(2, 16, 2048, 128) == 2 * 32 * 2048 * 4 + 32 * 2048 * 128 * 4 + 256
    assert lib.fa_backward_workspace_size(1, 1, 3, 64) == expect(1, 1, 3, 64) == 512 + 512 + 768 + 256
    assert lib.fa_backward_workspace_size(1, 1, 3, 96) == 0
    assert lib.fa_backward_workspace_size(0, 1, 3, 64) == 0


@pytest.mark.parametrize("fn", ["fa_backward", "fa_backward_fp32"])
def test_backward_rejects_bad_arguments(lib, fn):
    ptrs = [P(0x10000 * (i + 1)) for i in range(9)]
    ws = P(0x100000)
    need = lib.fa_backward_workspace_size(1, 2, 300, 64)
    f = getattr(lib, fn)
    assert f(*ptrs, ws, need - 1, 1, 2, 300, 64, 0.125, 0, None) == WORKSPACE
    assert f(*ptrs, None, need, 1, 2, 300, 64, 0.125, 0, None) == WORKSPACE
    assert f(*ptrs, P(0x100004), need, 1, 2, 300, 64, 0.125, 0, None) == MISALIGNED
    for i in range(9):
        bad = list(ptrs)
        bad[i] = None
        assert f(*bad, ws, need, 1, 2, 300, 64, 0.125, 0, None) == INVALID
    assert f(*ptrs, ws, need, 1, 2, 300, 80, 0.125, 0, None) == UNSUPPORTED


def test_unequal_length_entry_points_reject_bad_arguments(lib):
    # host-side checks only: no CUDA call is reached
    f = lib.fa_forward_qk
    assert f(*GOOD, 1, 4, 2, 0, 128, 64, 0.125, 1, None) == INVALID  # Nq = 0
    assert f(*GOOD, 1, 4, 2, 128, 0, 64, 0.125, 1, None) == INVALID  # Nk = 0
    assert f(*GOOD, 1, 4, 3, 128, 256, 64, 0.125, 1, None) == INVALID  # Hkv does not divide H
    assert f(*GOOD, 1, 4, 2, 128, 256, 96, 0.125, 1, None) == UNSUPPORTED
    for i in range(5):
        ptrs = list(GOOD)
        ptrs[i] = None
        assert f(*ptrs, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == INVALID
    b = lib.fa_backward_qk
    ptrs = [P(0x10000 * (i + 1)) for i in range(9)]
    ws = P(0x100000)
    need = lib.fa_backward_workspace_size(1, 4, 100, 64)  # sized by the query rows
    assert b(*ptrs, ws, need - 1, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == WORKSPACE
    assert b(*ptrs, P(0x100004), need, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == MISALIGNED
    assert b(*ptrs, ws, need, 1, 4, 2, 100, 0, 64, 0.125, 1, None) == INVALID
    assert b(*ptrs, ws, need, 1, 4, 2, 0, 300, 64, 0.125, 1, None) == INVALID
    for i in range(9):
        bad = list(ptrs)
        bad[i] = None
        assert b(*bad, ws, need, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == INVALID


def test_status_codes_have_strings(lib):
    for code in range(8):
        assert fa.status_string(code) != "unknown status", code


def test_backward_stages_rejects_bad_arguments(lib):
    f = lib.fa_backward_stages
    ptrs = [P(0x10000 * (i + 1)) for i in range(9)]
    ws = P(0x100000)
    need = lib.fa_backward_workspace_size(1, 4, 100, 64)
    for stages in (0, 8, -1, 16, 24, 0x107):
        assert f(*ptrs, ws, need, 1, 4, 2, 100, 300, 64, 0.125, 1, stages, None) == INVALID
    assert f(*ptrs, ws, need - 1, 1, 4, 2, 100, 300, 64, 0.125, 1, 2, None) == WORKSPACE
    assert f(*ptrs, P(0x100004), need, 1, 4, 2, 100, 300, 64, 0.125, 1, 2, None) == MISALIGNED
    assert f(*ptrs, ws, need, 1, 4, 3, 100, 300, 64, 0.125, 1, 7, None) == INVALID
    for i in range(9):
        bad = list(ptrs)
        bad[i] = None
        assert f(*bad, ws, need, 1, 4, 2, 100, 300, 64, 0.125, 1, 1, None) == INVALID


def test_binding_checks_every_tensor_before_the_library():
    # Shapes and dtypes of every argument are checked in the binding before any
    # pointer reaches the library (CPU tensors: the checks run without a GPU and
    # fail on the bad argument first).
    import torch

    B, H, N, d = 1, 2, 64, 64
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    lse_ok = torch.zeros(B, H, N)
    with pytest.raises(ValueError, match="lse"):
        fa.forward(q, q, q, lse=torch.zeros(B, H, N + 1))
    with pytest.raises(ValueError, match="lse"):
        fa.forward(q, q, q, lse=torch.zeros(B, H, N, dtype=torch.float64))
    with pytest.raises(ValueError, match="out"):
        fa.forward(q, q, q, out=torch.zeros(B, H, N, d + 1, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="lse"):
        fa.backward(q, q, q, q, q, torch.zeros(B, H, N - 1))
    with pytest.raises(ValueError, match="dq"):
        fa.backward(q, q, q, q, q, lse_ok, dq=torch.zeros(B, H, N, d))
    with pytest.raises(ValueError, match="dk, dv"):
        fa.backward(q, q, q, q, q, lse_ok, dv=torch.zeros(B, H, 2 * N, d, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="q, o, do"):
        fa.backward(q, q, q, q[:, :, :32].contiguous(), q, lse_ok)
    with pytest.raises(ValueError, match="contiguous"):
        fa.backward(q, q, q, q, q, lse_ok, dq=q.transpose(2, 3).contiguous().transpose(2, 3))
    with pytest.raises(ValueError, match="lse"):
        fa.backward_gqa(q, q[:, :1].contiguous(), q[:, :1].contiguous(), q, q, torch.zeros(B, H, N, 2))
    with pytest.raises(ValueError, match="lse"):
        fa.backward_noalloc(q, q, q, q, q, torch.zeros(B, H + 1, N))
    with pytest.raises(ValueError, match="lse"):
        fa.backward_stages(fa.STAGE_MAIN, q, q, q, q, q, torch.zeros(1), None, None, None, None)
    with pytest.raises(ValueError, match="CUDA"):
        fa.forward(q, q, q)  # well-formed, but on the host


def test_noalloc_rejects_oversized_shapes_without_cuda(lib):
    ptrs = [P(0x10000 * (i + 1)) for i in range(9)]
    B, H, N, d = 4, 16, 4096, 128
    assert lib.fa_backward_workspace_size(B, H, N, d) > 64 << 20
    assert lib.fa_backward_noalloc(*ptrs, B, H, N, d, 0.088, 1, None) == WORKSPACE


def test_fp8_forward_rejects_bad_arguments(lib):
    f = lib.fa_forward_fp8
    good = (1.0, 1.0, 1.0)
    for qs, ks, vs in ((0.0, 1.0, 1.0), (1.0, -1.0, 1.0), (1.0, 1.0, float("nan")), (float("inf"), 1.0, 1.0),
                       (1e-30, 1e-30, 1.0)):
        assert f(*GOOD, 1, 2, 1, 16, 16, 64, 0.125, qs, ks, vs, 0, None) == INVALID, (qs, ks, vs)
    assert f(*GOOD, 1, 2, 3, 16, 16, 64, 0.125, *good, 0, None) == INVALID  # Hkv does not divide H
    assert f(*GOOD, 1, 2, 1, 0, 16, 64, 0.125, *good, 0, None) == INVALID
    assert f(*GOOD, 1, 2, 1, 16, 16, 96, 0.125, *good, 0, None) == UNSUPPORTED
    for i in range(5):
        ptrs = list(GOOD)
        ptrs[i] = None
        assert f(*ptrs, 1, 2, 1, 16, 16, 64, 0.125, *good, 0, None) == INVALID
    ptrs = list(GOOD)
    ptrs[1] = P(0x20001)
    assert f(*ptrs, 1, 2, 1, 16, 16, 64, 0.125, *good, 0, None) == MISALIGNED


def test_deterministic_backward_rejects_bad_arguments(lib):
    f = lib.fa_backward_deterministic
    ptrs = [P(0x10000 * (i + 1)) for i in range(9)]
    ws = P(0x100000)
    need = lib.fa_backward_workspace_size(1, 4, 100, 64)
    assert f(*ptrs, ws, need - 1, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == WORKSPACE
    assert f(*ptrs, P(0x100004), need, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == MISALIGNED
    assert f(*ptrs, ws, need, 1, 4, 3, 100, 300, 64, 0.125, 1, None) == INVALID
    assert f(*ptrs, ws, need, 1, 4, 2, 100, 300, 96, 0.125, 1, None) == UNSUPPORTED
    for i in range(9):
        bad = list(ptrs)
        bad[i] = None
        assert f(*bad, ws, need, 1, 4, 2, 100, 300, 64, 0.125, 1, None) == INVALID
