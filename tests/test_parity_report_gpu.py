"""Parity figures of the CUDA path against the fp64 oracle, one line per
workload, for the measured table.  GPU only.

Each workload is checked against the same bounds as the parity tests (bf16
forward max-abs <= 1e-2 plus half the bf16 spacing of the reference value,
rel-L2 <= 5e-3; gradients rel-L2 <= 2e-2), and the figures themselves are
printed as ``PARITY {json}`` lines (visible with ``pytest -s``).  The oracle
covers every row for the small workloads, 64 sampled rows per head for the
4096-token one, the workload's own 512 sampled rows per head for the 32K one,
and four whole heads for the backward.
"""

import json
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import WORKLOADS, make_inputs, sample_rows, to_f64
from oracle import attention_bwd_ref, attention_fwd_ref, attention_rows_ref

pytestmark = pytest.mark.gpu


def _half_spacing(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0**-126)))
    return 0.5 * 2.0 ** (e - 7)


def _fwd_figures(o, lse, o_ref, lse_ref, bf16_out):
    err = np.abs(o - o_ref)
    bound = 1e-2 + (_half_spacing(o_ref) if bf16_out else 0.0)
    return {
        "o_max_abs": float(err.max()),
        "o_excess_over_bound": float((err - bound).max()),
        "o_rel_l2": float(np.linalg.norm((o - o_ref).ravel()) / np.linalg.norm(o_ref.ravel())),
        "lse_max_abs": float(np.abs(lse - lse_ref).max()),
    }


def _check_fwd(fig):
    assert fig["o_excess_over_bound"] <= 0 and fig["o_rel_l2"] <= 5e-3 and fig["lse_max_abs"] <= 1e-2, fig


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load_library()


@pytest.mark.parametrize("name", ["fwd_b1h1n256d64_fp32", "fwd_b4h16n1024d64", "fwd_b2h32n4096d128_causal",
                                  "fwd_b1h8n32768d128_causal_x4"])
def test_forward_parity_figures(name):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w.B, w.H, w.N, w.d, dtype=w.dtype, seed=0, qk_gain=w.qk_gain)
    o, lse = fa.forward(*(t.cuda() for t in (q, k, v)), causal=w.causal)
    fa.check_device_status()
    o, lse = to_f64(o), to_f64(lse)
    qd, kd, vd = to_f64(q), to_f64(k), to_f64(v)
    rows_per_head = w.sampled_rows or (64 if w.N >= 4096 else 0)
    if rows_per_head:
        rows = [sample_rows(w.N, rows_per_head, 0, h) for h in range(w.H)]
        o_ref, lse_ref = attention_rows_ref(qd, kd, vd, rows, w.scale, w.causal)
        o = np.stack([o[:, h, rows[h]] for h in range(w.H)], axis=1)
        lse = np.stack([lse[:, h, rows[h]] for h in range(w.H)], axis=1)
        checked = f"{rows_per_head} sampled rows per head"
    else:
        o_ref, lse_ref = attention_fwd_ref(qd, kd, vd, w.scale, w.causal)
        checked = "every row"
    fig = _fwd_figures(o, lse, o_ref, lse_ref, w.dtype == torch.bfloat16)
    print("PARITY " + json.dumps({"workload": name, "checked": checked, **fig}))
    _check_fwd(fig)


def test_backward_parity_figures():
    w = WORKLOADS["fwdbwd_b2h16n2048d128_causal"]
    q, k, v, do = make_inputs(w.B, w.H, w.N, w.d, seed=0, with_do=True)
    qg, kg, vg, dog = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qg, kg, vg, causal=w.causal)
    dq, dk, dv = fa.backward(qg, kg, vg, o, dog, lse, causal=w.causal)
    fa.check_device_status()
    got = [to_f64(x) for x in (dq, dk, dv)]
    worst = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for b, h in [(0, 0), (0, 7), (1, 3), (1, 15)]:
        sl = lambda x: to_f64(x)[b : b + 1, h : h + 1]
        ref = attention_bwd_ref(sl(q), sl(k), sl(v), sl(do), w.scale, w.causal)
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            g = g[b : b + 1, h : h + 1]
            worst[name] = max(worst[name], float(np.linalg.norm((g - r).ravel()) / np.linalg.norm(r.ravel())))
    print("PARITY " + json.dumps({"workload": w.name, "checked": "4 whole heads",
                                  **{f"{k}_rel_l2": v for k, v in worst.items()}}))
    assert max(worst.values()) <= 2e-2, worst
