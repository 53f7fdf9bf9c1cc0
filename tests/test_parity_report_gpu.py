"""The five workloads at their full sizes against the fp64 oracle, one PARITY
line per workload (visible with ``pytest -s``).  GPU only.

Every output element is compared for the first four workloads: the oracle runs
one (batch, head) at a time with the whole score matrix of that head.  The
long-context workload (32768 keys) is checked on its own definition, 512
seeded sampled query rows per head (``inputs.sample_rows``), each row against
all of its keys.  Bounds: tests/parity.py.  Outputs are NaN-filled before the
call, so an element the kernels never write fails.
"""

import json

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import WORKLOADS, make_inputs, sample_rows, to_f64
from oracle import attention_bwd_ref, attention_fwd_ref, attention_rows_ref
from parity import check_bwd, check_fwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load_library()


def _forward(w, q, k, v):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((w.B, w.H, w.N), float("nan"), device="cuda")
    fa.forward(qd, kd, vd, causal=w.causal, out=o, lse=lse)
    fa.check_device_status()
    return (qd, kd, vd, o, lse), to_f64(o), to_f64(lse)


def _per_head_fwd_ref(w, q, k, v):
    o_ref = np.empty((w.B, w.H, w.N, w.d))
    lse_ref = np.empty((w.B, w.H, w.N))
    for b in range(w.B):
        for h in range(w.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            o_ref[sl], lse_ref[sl] = attention_fwd_ref(to_f64(q[sl]), to_f64(k[sl]), to_f64(v[sl]),
                                                       w.scale, w.causal)
    return o_ref, lse_ref


def _report(name, checked, fig):
    print("PARITY " + json.dumps({"workload": name, "checked": checked, **fig}))


@pytest.mark.parametrize("name", ["fwd_b1h1n256d64_fp32", "fwd_b4h16n1024d64", "fwd_b2h32n4096d128_causal"])
def test_forward_every_row(name):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w.B, w.H, w.N, w.d, dtype=w.dtype, seed=0, qk_gain=w.qk_gain)
    _, o, lse = _forward(w, q, k, v)
    o_ref, lse_ref = _per_head_fwd_ref(w, q, k, v)
    fig = check_fwd(o, lse, o_ref, lse_ref, name, bf16_out=w.dtype == torch.bfloat16)
    _report(name, "every row", fig)


def test_forward_long_context_sampled_rows():
    w = WORKLOADS["fwd_b1h8n32768d128_causal_x4"]
    q, k, v = make_inputs(w.B, w.H, w.N, w.d, seed=0, qk_gain=w.qk_gain)
    _, o, lse = _forward(w, q, k, v)
    rows = [sample_rows(w.N, w.sampled_rows, 0, h) for h in range(w.H)]
    o_ref, lse_ref = attention_rows_ref(to_f64(q), to_f64(k), to_f64(v), rows, w.scale, w.causal)
    o = np.stack([o[:, h, rows[h]] for h in range(w.H)], axis=1)
    lse = np.stack([lse[:, h, rows[h]] for h in range(w.H)], axis=1)
    fig = check_fwd(o, lse, o_ref, lse_ref, w.name)
    _report(w.name, f"{w.sampled_rows} sampled rows per head", fig)


def test_forward_and_backward_every_head():
    w = WORKLOADS["fwdbwd_b2h16n2048d128_causal"]
    q, k, v, do = make_inputs(w.B, w.H, w.N, w.d, seed=0, with_do=True)
    (qd, kd, vd, o_dev, lse_dev), o, lse = _forward(w, q, k, v)
    dod = do.cuda()
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    fa.backward(qd, kd, vd, o_dev, dod, lse_dev, causal=w.causal, dq=dq, dk=dk, dv=dv)
    fa.check_device_status()
    got = [to_f64(x) for x in (dq, dk, dv)]
    o_ref, lse_ref = _per_head_fwd_ref(w, q, k, v)
    fig = check_fwd(o, lse, o_ref, lse_ref, w.name)
    ref = [np.empty_like(g) for g in got]
    for b in range(w.B):
        for h in range(w.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            for r, x in zip(ref, attention_bwd_ref(to_f64(q[sl]), to_f64(k[sl]), to_f64(v[sl]),
                                                   to_f64(do[sl]), w.scale, w.causal)):
                r[sl] = x
    errs = check_bwd(got, ref, w.name)
    # the bound also holds head by head, not only over the whole tensor
    worst = {n: 0.0 for n in ("dq", "dk", "dv")}
    for b in range(w.B):
        for h in range(w.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            e = check_bwd([g[sl] for g in got], [r[sl] for r in ref], (w.name, b, h))
            worst = {n: max(worst[n], e[n]) for n in worst}
    _report(w.name, "every row and every head, forward and backward",
            {**fig, **{f"{n}_rel_l2": e for n, e in errs.items()},
             **{f"{n}_rel_l2_worst_head": e for n, e in worst.items()}})
