"""fa_backward_noalloc: the backward pass for callers that cannot allocate device
memory (their device memory is owned by a host framework that only hands them
input and output buffers, or they must not call cudaMalloc/cudaFree because
those calls can synchronise the whole device).  Its scratch is a fixed array
inside the library instead of a caller workspace.

GPU only.  Called through the C ABI twice in a row (the second call finds the
array as the first one left it) and checked two ways: against the fp64 oracle
within the gradient bound of the parity tests, and against fa_backward on the
same inputs, where dK and dV come from the same kernel and must agree bit for
bit (dQ is summed by reduce-adds in an order that varies, so it is held to fp32
rounding).  This file is named so that pytest collects it last.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import make_inputs, to_f64
from oracle import attention_bwd_ref
from parity import check_bwd

pytestmark = pytest.mark.gpu

MAX_BYTES = 64 << 20  # FA_BACKWARD_NOALLOC_MAX_BYTES in include/fa.h


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return fa.load_library()


def call_noalloc(lib, q, k, v, o, do, lse, causal):
    B, H, N, d = q.shape
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.fa_backward_noalloc(P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv),
                                 B, H, N, d, 1.0 / math.sqrt(d), int(causal),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, fa.status_string(st)
    return dq, dk, dv


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 4, 1000, 128, True), (2, 3, 384, 64, False)])
def test_noalloc_matches_oracle_and_workspace_backward_twice(lib, B, H, N, d, causal):
    assert lib.fa_backward_workspace_size(B, H, N, d) <= MAX_BYTES
    for call in range(2):
        q, k, v, do = make_inputs(B, H, N, d, seed=100 + call, with_do=True)
        qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
        o, lse = fa.forward(qd, kd, vd, causal=causal)
        got = call_noalloc(lib, qd, kd, vd, o, dod, lse, causal)
        fa.check_device_status()
        ref = attention_bwd_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), 1 / math.sqrt(d), causal)
        check_bwd([to_f64(g) for g in got], ref, ("noalloc", call))
        ws = fa.backward(qd, kd, vd, o, dod, lse, causal=causal)
        fa.check_device_status()
        assert torch.equal(got[1], ws[1]) and torch.equal(got[2], ws[2]), call  # dK, dV
        rel = float((got[0].float() - ws[0].float()).norm() / ws[0].float().norm())
        assert rel < 1e-3, (call, rel)


def test_noalloc_rejects_shapes_beyond_its_array(lib):
    B, H, N, d = 4, 16, 4096, 128  # needs about 135 MB of scratch
    assert lib.fa_backward_workspace_size(B, H, N, d) > MAX_BYTES
    dummy = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(9)]
    st = lib.fa_backward_noalloc(*dummy, B, H, N, d, 0.088, 1, None)
    assert st == 4  # FA_ERR_WORKSPACE
