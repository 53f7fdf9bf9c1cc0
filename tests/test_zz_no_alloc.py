"""fa_backward_noalloc: the backward pass for callers that cannot allocate device
memory (their device memory is owned by a host framework that only hands them
input and output buffers, or they must not call cudaMalloc/cudaFree because
those calls can synchronise the whole device).  Its scratch is a fixed array
inside the library instead of a caller workspace.

GPU only.  Called through the C ABI and compared with fa_backward on the same
inputs, twice in a row (the second call reuses the array the first one left
behind), within the gradient tolerance of the parity tests.  This file is named
so that pytest collects it last.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import make_inputs, to_f64

pytestmark = pytest.mark.gpu

GRAD_RELL2 = 2e-2  # the dQ/dK/dV bound of the parity tests
MAX_BYTES = 64 << 20  # FA_BACKWARD_NOALLOC_MAX_BYTES in include/fa.h


def rel_l2(x, ref):
    return float(np.linalg.norm((x - ref).ravel()) / np.linalg.norm(ref.ravel()))


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return fa.load_library()


def call_noalloc(lib, q, k, v, o, do, lse, causal):
    B, H, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.fa_backward_noalloc(P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv),
                                 B, H, N, d, 1.0 / math.sqrt(d), int(causal),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, fa.status_string(st)
    return dq, dk, dv


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 4, 1000, 128, True), (2, 3, 384, 64, False)])
def test_noalloc_matches_workspace_backward_twice(lib, B, H, N, d, causal):
    for call in range(2):
        q, k, v, do = (t.cuda() for t in make_inputs(B, H, N, d, seed=100 + call, with_do=True))
        o, lse = fa.forward(q, k, v, causal=causal)
        ref = fa.backward(q, k, v, o, do, lse, causal=causal)
        got = call_noalloc(lib, q, k, v, o, do, lse, causal)
        fa.check_device_status()
        for g, r in zip(got, ref):
            g64, r64 = to_f64(g), to_f64(r)
            assert np.all(np.isfinite(g64))
            assert rel_l2(g64, r64) <= GRAD_RELL2, (call, rel_l2(g64, r64))


def test_noalloc_rejects_shapes_beyond_its_array(lib):
    B, H, N, d = 4, 16, 4096, 128  # needs about 135 MB of scratch
    assert lib.fa_backward_workspace_size(B, H, N, d) > MAX_BYTES
    dummy = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(9)]
    st = lib.fa_backward_noalloc(*dummy, B, H, N, d, 0.088, 1, None)
    assert st == 4  # FA_ERR_WORKSPACE
