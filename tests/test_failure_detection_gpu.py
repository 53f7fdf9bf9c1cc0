"""Failure detection without a GPU fault: a kernel waits on a barrier that nothing
completes, its bounded wait runs out (about 2 s), it records a timeout in the
device status word and returns.  The host must see FA_ERR_DEVICE_TIMEOUT, and the
context must stay usable (a normal forward right after matches the oracle)."""

import ctypes
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import make_inputs, to_f64
from oracle import attention_fwd_ref

pytestmark = pytest.mark.gpu

FA_ERR_DEVICE_TIMEOUT = 6


def test_bounded_wait_reports_timeout_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = fa.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fa_check_device_status(stream) == 0  # starts clean
    assert lib.fa_debug_wait_timeout(stream) == 0
    assert lib.fa_check_device_status(stream) == FA_ERR_DEVICE_TIMEOUT
    assert lib.fa_check_device_status(stream) == 0  # reading clears it
    q, k, v = (t.cuda() for t in make_inputs(1, 2, 200, 64, seed=5))
    o, lse = fa.forward(q, k, v, causal=True)
    fa.check_device_status()
    o_ref, _ = attention_fwd_ref(to_f64(q.cpu()), to_f64(k.cpu()), to_f64(v.cpu()), 1 / math.sqrt(64), True)
    assert np.max(np.abs(to_f64(o) - o_ref)) < 1e-2
