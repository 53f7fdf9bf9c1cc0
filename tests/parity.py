"""Error measures and parity bounds shared by the GPU parity tests.

Bounds (from the method's task statement): bf16 forward O max-abs <= 1e-2 and
rel-L2 <= 5e-3; dQ/dK/dV rel-L2 <= 2e-2.  LSE max-abs <= 1e-2 is a reading (the
statement names no LSE bound; the forward's absolute bound is reused).

Max-abs on bf16 outputs.  O is stored in bf16, so the kernel's fp32 result x is
rounded to nearest-even before it reaches memory, and for |O| >= 2 one rounding
step (2^-6 or more) already exceeds 1e-2.  The bound is therefore applied to the
kernel's error before that rounding: the stored value must be the bf16 rounding
of some x with |x - o_ref| <= 1e-2.  Rounding is monotone, so this holds exactly
when rne(o_ref - 1e-2) <= o <= rne(o_ref + 1e-2) element by element (the "band"
check below).  It admits at most half a bf16 spacing beyond 1e-2 and nothing
else.  fp32 outputs are held to the plain |o - o_ref| <= 1e-2.
"""

from __future__ import annotations

import numpy as np

O_MAXABS, O_RELL2, LSE_MAXABS, GRAD_RELL2 = 1e-2, 5e-3, 1e-2, 2e-2


def rel_l2(x, ref):
    return float(np.linalg.norm((x - ref).ravel()) / np.linalg.norm(ref.ravel()))


def max_abs(x, ref):
    return float(np.max(np.abs(x - ref))) if np.size(x) else 0.0


def bf16_rne(x):
    """float64 -> nearest bf16 value (ties to even), returned as float64.

    bf16 keeps 8 significant bits: x is scaled by the spacing 2^(e-7) of its
    binade (exact in fp64), rounded half to even by numpy, and scaled back.
    Values below the normal range use the spacing of the smallest binade."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e - 1, -126)
    spacing = np.ldexp(1.0, e - 7)
    return np.round(x / spacing) * spacing


def bf16_band(o_ref, tol=O_MAXABS):
    """The bf16 values a kernel may store when its error before rounding is <= tol."""
    return bf16_rne(o_ref - tol), bf16_rne(o_ref + tol)


def fwd_figures(o, lse, o_ref, lse_ref, bf16_out=True):
    """Error figures of a forward result against the oracle."""
    fig = {
        "o_max_abs": max_abs(o, o_ref),
        "o_rel_l2": rel_l2(o, o_ref),
        "lse_max_abs": max_abs(lse, lse_ref),
        "finite": bool(np.all(np.isfinite(o)) and np.all(np.isfinite(lse))),
    }
    if bf16_out:
        lo, hi = bf16_band(o_ref)
        fig["o_outside_band"] = int(np.count_nonzero((o < lo) | (o > hi)))
        fig["o_max_abs_vs_rne_ref"] = max_abs(o, bf16_rne(o_ref))
    else:
        fig["o_outside_band"] = int(np.count_nonzero(np.abs(o - o_ref) > O_MAXABS))
    return fig


def check_fwd(o, lse, o_ref, lse_ref, what, bf16_out=True):
    fig = fwd_figures(o, lse, o_ref, lse_ref, bf16_out)
    ok = (fig["finite"] and fig["o_outside_band"] == 0 and fig["o_rel_l2"] <= O_RELL2
          and fig["lse_max_abs"] <= LSE_MAXABS)
    assert ok, (what, fig)
    return fig


def check_bwd(got, ref, what, bound=GRAD_RELL2):
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(g)), (what, name)
        if np.linalg.norm(r) < 1e-12:  # e.g. N == 1: dQ = dK = 0 exactly
            assert max_abs(g, r) <= 1e-3, (what, name)
            errs[name] = 0.0
            continue
        errs[name] = rel_l2(g, r)
        assert errs[name] <= bound, (what, name, errs[name])
    return errs


# FP8 forward (e4m3 Q, K, V and P; see oracle.e4m3_p_rounding_bound).  Reading
# of the tolerance: the rounding of P to e4m3 dominates; element by element the
# error must stay inside the oracle's worst-case bound for that rounding plus the
# bf16 rounding of the output and 2e-3 for the remaining fp32 arithmetic (the
# exponentials, accumulation order); over the tensor the relative L2 error must
# stay under 5e-2, about twice the ~2.6 % rounding noise e4m3's 3 mantissa bits
# give.  LSE does not see the rounding of P and keeps the bf16 bound.
FP8_O_RELL2, FP8_SLACK = 5e-2, 2e-3


def check_fwd_fp8(o, lse, o_ref, lse_ref, bound, what):
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), what
    assert np.all(o[empty] == 0.0), what
    full = ~empty
    o, lse, o_ref, lse_ref, bound = o[full], lse[full], o_ref[full], lse_ref[full], bound[full]
    _, e = np.frexp(o_ref)
    half_ulp = np.ldexp(1.0, np.maximum(e - 1, -126) - 8)
    fig = {
        "o_max_abs": max_abs(o, o_ref),
        "o_rel_l2": rel_l2(o, o_ref) if o.size else 0.0,
        "lse_max_abs": max_abs(lse, lse_ref),
        "o_over_bound": int(np.count_nonzero(np.abs(o - o_ref) > bound + half_ulp + FP8_SLACK)),
        "o_max_err_over_bound": float(np.max(np.abs(o - o_ref) / (bound + half_ulp + FP8_SLACK)))
        if o.size else 0.0,
        "finite": bool(np.all(np.isfinite(o)) and np.all(np.isfinite(lse))),
    }
    ok = (fig["finite"] and fig["o_over_bound"] == 0 and fig["o_rel_l2"] <= FP8_O_RELL2
          and fig["lse_max_abs"] <= LSE_MAXABS)
    assert ok, (what, fig)
    return fig
