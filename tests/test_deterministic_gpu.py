"""The deterministic backward (fa_backward_deterministic: dK/dV per key tile as
in fa_backward, dQ by a separate pass over the key tiles in a fixed order).
GPU only.  Checked against the fp64 oracle (gradient bound of tests/parity.py),
run twice for bitwise equal results, and against fa_backward: dK and dV come
from the same per-key-tile arithmetic and must agree bit for bit; fa_backward's
dQ (reduce-adds in a varying order) must agree to fp32 rounding."""

import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import WORKLOADS, make_inputs, to_f64
from oracle import attention_bwd_gqa_ref, attention_bwd_ref
from parity import check_bwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load_library()


def _inputs(B, H, Hkv, Nq, Nk, d, seed):
    q, do = make_inputs(B, H, Nq, d, seed=seed, with_do=True)[0::3]
    k, v = make_inputs(B, Hkv, Nk, d, seed=seed + 100)[1:3]
    return q, k, v, do


def _run(q, k, v, do, causal):
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward_qk(qd, kd, vd, causal=causal)
    outs = []
    for _ in range(2):
        g = tuple(torch.full_like(t, float("nan")) for t in (qd, kd, vd))
        fa.backward_deterministic(qd, kd, vd, o, dod, lse, causal=causal, dq=g[0], dk=g[1], dv=g[2])
        outs.append(g)
    ref_run = fa.backward_qk(qd, kd, vd, o, dod, lse, causal=causal)
    fa.check_device_status()
    return outs, ref_run


def _compare(outs, ref_run, ref, what):
    (dq, dk, dv), again = outs
    for a, b in zip((dq, dk, dv), again):
        assert torch.equal(a, b), what  # run to run, bit for bit
    assert torch.equal(dk, ref_run[1]) and torch.equal(dv, ref_run[2]), what
    if float(ref_run[0].float().norm()) > 0:
        rel = float((dq.float() - ref_run[0].float()).norm() / ref_run[0].float().norm())
        assert rel < 1e-3, (what, rel)
    check_bwd([to_f64(x) for x in (dq, dk, dv)], ref, what)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 256, 384, 700])
def test_deterministic_backward_sweep(N, causal, d):
    q, k, v, do = _inputs(1, 2, 2, N, N, d, seed=N + 3)
    outs, ref_run = _run(q, k, v, do, causal)
    ref = attention_bwd_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), 1 / math.sqrt(d), causal)
    _compare(outs, ref_run, ref, (N, causal, d))


@pytest.mark.parametrize("H,Hkv,Nq,Nk,causal,d", [(8, 2, 300, 300, True, 128), (4, 1, 256, 640, True, 64),
                                                  (4, 4, 640, 200, True, 128), (6, 3, 129, 1000, False, 64),
                                                  (4, 2, 1000, 1, True, 128)])
def test_deterministic_backward_grouped_heads_and_unequal_lengths(H, Hkv, Nq, Nk, causal, d):
    q, k, v, do = _inputs(1, H, Hkv, Nq, Nk, d, seed=H + Nq)
    outs, ref_run = _run(q, k, v, do, causal)
    ref = attention_bwd_gqa_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), 1 / math.sqrt(d), causal)
    _compare(outs, ref_run, ref, (H, Hkv, Nq, Nk, causal, d))


def test_deterministic_backward_fwdbwd_workload_every_head():
    w = WORKLOADS["fwdbwd_b2h16n2048d128_causal"]
    q, k, v, do = make_inputs(w.B, w.H, w.N, w.d, seed=0, with_do=True)
    outs, ref_run = _run(q, k, v, do, w.causal)
    got = [to_f64(x) for x in outs[0]]
    for b in range(w.B):
        for h in range(w.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            ref = attention_bwd_ref(to_f64(q[sl]), to_f64(k[sl]), to_f64(v[sl]), to_f64(do[sl]), w.scale, w.causal)
            check_bwd([g[sl] for g in got], ref, (w.name, b, h))
    for a, b_ in zip(outs[0], outs[1]):
        assert torch.equal(a, b_)
