"""Parity of the FP8 forward (fa_forward_fp8: e4m3 Q, K, V with per-tensor
scales, e4m3 P) with the fp64 oracle evaluated on the values the stored e4m3
tensors stand for.  GPU only.  Bounds: tests/parity.py (check_fwd_fp8), built on
oracle.e4m3_p_rounding_bound.  Outputs are NaN-filled before every call.
"""

import json
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import WORKLOADS, fp8_values, make_fp8_inputs, sample_rows, to_f64
from oracle import attention_fwd_gqa_ref, attention_rows_ref, e4m3_p_rounding_bound
from parity import check_fwd_fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load_library()


def run_fp8(B, H, Hkv, Nq, Nk, d, causal, seed, gain=1.0):
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(B, H, Nq, d, seed=seed, qk_gain=gain,
                                             Hkv=None if (Hkv == H and Nk == Nq) else Hkv,
                                             Nk=None if (Hkv == H and Nk == Nq) else Nk)
    qd, kd, vd = (t.cuda() for t in (q8, k8, v8))
    o = torch.full((B, H, Nq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, Nq), float("nan"), device="cuda")
    fa.forward_fp8(qd, kd, vd, qs, ks, vs, causal=causal, out=o, lse=lse)
    fa.check_device_status()
    vals = (fp8_values(q8, qs), fp8_values(k8, ks), fp8_values(v8, vs))
    return vals, to_f64(o), to_f64(lse)


def _ref(vals, scale, causal):
    q, k, v = vals
    g = q.shape[1] // k.shape[1]
    o_ref, lse_ref = attention_fwd_gqa_ref(q, k, v, scale, causal)
    bound = e4m3_p_rounding_bound(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), scale, causal)
    return o_ref, lse_ref, bound


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 77, 128, 300, 640, 1000])
def test_fp8_forward_sweep(N, causal, d):
    vals, o, lse = run_fp8(1, 3, 3, N, N, d, causal, seed=N + d)
    o_ref, lse_ref, bound = _ref(vals, 1 / math.sqrt(d), causal)
    check_fwd_fp8(o, lse, o_ref, lse_ref, bound, (N, causal, d))


@pytest.mark.parametrize("H,Hkv,Nq,Nk,causal,d", [(8, 2, 300, 300, True, 128), (4, 1, 256, 640, True, 64),
                                                  (4, 4, 640, 200, True, 128), (6, 3, 129, 1000, False, 64)])
def test_fp8_forward_grouped_heads_and_unequal_lengths(H, Hkv, Nq, Nk, causal, d):
    vals, o, lse = run_fp8(1, H, Hkv, Nq, Nk, d, causal, seed=H + Nq)
    o_ref, lse_ref, bound = _ref(vals, 1 / math.sqrt(d), causal)
    check_fwd_fp8(o, lse, o_ref, lse_ref, bound, (H, Hkv, Nq, Nk, causal, d))


@pytest.mark.parametrize("name", ["fwd_b4h16n1024d64", "fwd_b2h32n4096d128_causal"])
def test_fp8_forward_workload_every_row(name):
    w = WORKLOADS[name]
    vals, o, lse = run_fp8(w.B, w.H, w.H, w.N, w.N, w.d, w.causal, seed=0)
    figs = []
    for b in range(w.B):
        for h in range(w.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            o_ref, lse_ref, bound = _ref(tuple(x[sl] for x in vals), w.scale, w.causal)
            figs.append(check_fwd_fp8(o[sl], lse[sl], o_ref, lse_ref, bound, (name, b, h)))
    worst = {k: max(f[k] for f in figs) for k in ("o_max_abs", "o_rel_l2", "lse_max_abs", "o_max_err_over_bound")}
    print("PARITY " + json.dumps({"workload": name + "_fp8", "checked": "every row", **worst}))


def test_fp8_forward_long_context_sampled_rows():
    w = WORKLOADS["fwd_b1h8n32768d128_causal_x4"]
    vals, o, lse = run_fp8(w.B, w.H, w.H, w.N, w.N, w.d, w.causal, seed=0, gain=w.qk_gain)
    rows = [sample_rows(w.N, w.sampled_rows, 0, h) for h in range(w.H)]
    o_ref, lse_ref = attention_rows_ref(*vals, rows, w.scale, w.causal)
    bound = e4m3_p_rounding_bound(*vals, w.scale, w.causal, rows=rows)
    o = np.stack([o[:, h, rows[h]] for h in range(w.H)], axis=1)
    lse = np.stack([lse[:, h, rows[h]] for h in range(w.H)], axis=1)
    fig = check_fwd_fp8(o, lse, o_ref, lse_ref, bound, w.name)
    print("PARITY " + json.dumps({"workload": w.name + "_fp8", "checked": "512 sampled rows per head", **fig}))


def test_fp8_descales_enter_exactly():
    # doubling a tensor's descale while halving nothing else is the same as
    # doubling the values it stands for: V's scale multiplies O, Q's and K's
    # scales multiply the scores (so LSE moves with them)
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 2, 384, 128, seed=9)
    qd, kd, vd = (t.cuda() for t in (q8, k8, v8))
    o1, l1 = fa.forward_fp8(qd, kd, vd, qs, ks, vs, causal=True)
    o2, l2 = fa.forward_fp8(qd, kd, vd, qs, ks, 2 * vs, causal=True)
    fa.check_device_status()
    assert torch.equal(o2.float(), (o1.float() * 2).bfloat16().float())
    assert torch.equal(l1, l2)
