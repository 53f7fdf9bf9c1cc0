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


FA_ERR_DEVICE_STATE = 7


def test_stale_scheduler_slot_is_reported_not_used():
    # A launch that never finished would leave its scheduler slot held.  The
    # diagnostic marks every slot that way; the next forward must stop drawing
    # work and report FA_ERR_DEVICE_STATE instead of handing out stale items,
    # and after the status has been read (which frees the slots) the forward
    # must be correct again.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = fa.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fa_check_device_status(stream) == 0
    q, k, v = (t.cuda() for t in make_inputs(2, 16, 2048, 64, seed=6))  # 256 items > one per SM
    assert lib.fa_debug_hold_scheduler(stream) == 0
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), device="cuda")
    fa.forward(q, k, v, causal=True, out=o, lse=lse)
    assert lib.fa_check_device_status(stream) == FA_ERR_DEVICE_STATE
    assert bool(torch.isnan(o).any())  # items past each CTA's first were skipped, visibly
    assert lib.fa_check_device_status(stream) == 0
    o, lse = fa.forward(q, k, v, causal=True, out=o, lse=lse)
    fa.check_device_status()
    sl = (slice(1, 2), slice(15, 16))  # one head checked against the oracle
    o_ref, _ = attention_fwd_ref(to_f64(q[sl].cpu()), to_f64(k[sl].cpu()), to_f64(v[sl].cpu()),
                                 1 / math.sqrt(64), True)
    assert not bool(torch.isnan(o).any())
    assert np.max(np.abs(to_f64(o[sl]) - o_ref)) < 1e-2
