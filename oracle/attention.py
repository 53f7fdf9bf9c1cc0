"""Plain, slow, fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
call it.  It shares no code with the CUDA path.

Sources (the three web pages on exact tiled attention):

* "Atención Flash: Revolucionando la Eficiencia de los Modelos de Transformador"
  (unite.ai), section "Atención Flash" / standard attention listing: the
  definition softmax(Q K^T / sqrt(d_k)) V, with the score tensor of shape
  (batch, seq, seq) materialised.  ``attention_fwd_ref`` is that definition,
  written out in fp64, one (batch, head) at a time.
* same page, section "La Matemática detrás de la Atención Flash", formula 1
  (softmax decomposition with the row maximum m) and formula 2 (the merge of two
  blocks with m = max(m_x, m_y)).  ``safe_softmax`` and ``softmax_merge``.
* same page, section "Detalles de Implementación" (the simplified tiled loop):
  running statistics M (max) and L (sum), query blocks outside, key/value blocks
  inside.  ``online_softmax_attention`` restates that loop with the output update
  corrected (the printed update drops the factor L of the old sum; here the old
  output is multiplied by L * exp(M - M_new) before the division by L_new).
* "FlashAttention algorithm part 3" (nisoo.com), sections "Softmax Sicura" and
  "SafeSoftmax con Calcolo Normalizzatore Online": subtract the maximum before
  exponentiating; keep a running normaliser corrected when the maximum moves.

Not on the pages, taken from the method's statement of the task: the causal mask
(key j visible to query i iff j <= i, square and top-left aligned), the per-row
log-sum-exp output (natural log, of the scaled scores) and the backward pass
(the closed-form softmax Jacobian).

Reading for unequal query and key lengths (Nq queries, Nk keys), which the pages
do not treat: the causal mask is aligned at the bottom right, key j visible to
query i iff j <= i + (Nk - Nq), so the last query sees every key and Nq = Nk is
the square mask above.  A query that sees no key (i < Nq - Nk) has O = 0 and
LSE = -inf.

All arrays are numpy float64 with layout [B, H, N, d] (LSE: [B, H, N]); K and V
may have their own length Nk.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "safe_softmax",
    "softmax_merge",
    "scores",
    "attention_fwd_ref",
    "attention_bwd_ref",
    "attention_rows_ref",
    "online_softmax_attention",
    "attention_fwd_gqa_ref",
    "attention_bwd_gqa_ref",
    "e4m3_p_rounding_bound",
]


def _as64(x):
    return np.asarray(x, dtype=np.float64)


def safe_softmax(x, axis=-1):
    """softmax(x) = exp(x - m) / sum(exp(x - m)), m = max(x).

    Softmax decomposition, formula 1 of the unite.ai page ("La Matemática detrás
    de la Atención Flash"); the nisoo.com page ("Softmax Sicura") gives the same
    rule in words.  Entries equal to -inf get probability 0.
    """
    x = _as64(x)
    m = np.max(x, axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def softmax_merge(fx, mx, lx, fy, my, ly):
    """Merge the partial softmax statistics of two blocks x and y.

    Formula 2 of the unite.ai page ("Fusión de Softmax"), whose printed form is
    garbled.  Reading used here: for a block z keep f(z) = exp(z - m_z) and
    l(z) = sum f(z).  With m = max(m_x, m_y):
        f(x u y) = [exp(m_x - m) f(x), exp(m_y - m) f(y)]
        l(x u y) = exp(m_x - m) l(x) + exp(m_y - m) l(y)
        softmax(x u y) = f(x u y) / l(x u y)
    Returns (softmax(x u y), m, l).
    """
    m = max(mx, my)
    ax = math.exp(mx - m)
    ay = math.exp(my - m)
    f = np.concatenate([ax * _as64(fx), ay * _as64(fy)])
    l = ax * lx + ay * ly
    return f / l, m, l


def scores(q, k, scale, causal):
    """S = scale * Q K^T per (batch, head), with the causal mask applied.

    The score tensor of the standard-attention listing (unite.ai page), here
    one [Nq, Nk] matrix per (b, h).  Masked entries are -inf: under the causal
    mask, key j is hidden from query i when j > i + (Nk - Nq).
    """
    q = _as64(q)
    k = _as64(k)
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))
    if causal:
        nq, nk = q.shape[2], k.shape[2]
        above = np.triu(np.ones((nq, nk), dtype=bool), k=nk - nq + 1)
        s = np.where(above, -np.inf, s)
    return s


def _softmax_rows(s):
    """Row-wise safe softmax of a score tensor and its log-sum-exp; a row with no
    visible key gets probabilities 0 and LSE -inf."""
    m = np.max(s, axis=-1, keepdims=True)
    empty = np.isneginf(m)
    m0 = np.where(empty, 0.0, m)
    e = np.exp(s - m0)
    l = np.sum(e, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(empty, 0.0, e / np.where(empty, 1.0, l))
        lse = np.where(empty, -np.inf, m0 + np.log(np.where(empty, 1.0, l)))
    return p, lse[..., 0]


def attention_fwd_ref(q, k, v, scale, causal):
    """O = softmax(scale * Q K^T) V and LSE = log sum_j exp(scale * q_i . k_j).

    The standard-attention definition of the unite.ai page, evaluated in fp64
    with the full score matrix materialised.  LSE_i = m_i + ln sum_j
    exp(S_ij - m_i) with m_i the row maximum (safe softmax).
    """
    v = _as64(v)
    p, lse = _softmax_rows(scores(q, k, scale, causal))
    o = np.matmul(p, v)
    return o, lse


def attention_bwd_ref(q, k, v, do, scale, causal):
    """Gradients of L = sum(O * dO) with respect to Q, K and V.

    Not on the pages; the closed form of the softmax Jacobian:
        P   = softmax(S)            (row-wise)
        dV  = P^T dO
        dP  = dO V^T
        dS  = P * (dP - rowsum(P * dP))
        dQ  = scale * dS K
        dK  = scale * dS^T Q
    """
    q = _as64(q)
    k = _as64(k)
    v = _as64(v)
    do = _as64(do)
    p, _ = _softmax_rows(scores(q, k, scale, causal))
    dv = np.matmul(np.swapaxes(p, -1, -2), do)
    dp = np.matmul(do, np.swapaxes(v, -1, -2))
    ds = p * (dp - np.sum(p * dp, axis=-1, keepdims=True))
    dq = scale * np.matmul(ds, k)
    dk = scale * np.matmul(np.swapaxes(ds, -1, -2), q)
    return dq, dk, dv


def attention_rows_ref(q, k, v, rows, scale, causal):
    """O and LSE for selected query rows only, without the full N x N matrix.

    Same definition as ``attention_fwd_ref``, evaluated row by row: for each
    (b, h) and each query index i in ``rows[h]`` (or ``rows`` when it is one
    list for all heads) the score row S[i, :] (keys 0..i + Nk - Nq when causal)
    is formed, then its safe softmax and the weighted sum of V.  A row with no
    visible key gets O = 0 and LSE = -inf.
    Returns (o [B, H, R, d], lse [B, H, R]).
    """
    q = _as64(q)
    k = _as64(k)
    v = _as64(v)
    b_, h_, n, d = q.shape
    off = k.shape[2] - n
    per_head = isinstance(rows, (list, tuple)) and len(rows) > 0 and np.ndim(rows[0]) == 1
    r = len(rows[0]) if per_head else len(rows)
    o = np.zeros((b_, h_, r, d))
    lse = np.zeros((b_, h_, r))
    for b in range(b_):
        for h in range(h_):
            sel = rows[h] if per_head else rows
            for t, i in enumerate(sel):
                i = int(i)
                last = i + off + 1 if causal else k.shape[2]
                if last <= 0:
                    lse[b, h, t] = -np.inf
                    continue
                kk = k[b, h, :last]
                vv = v[b, h, :last]
                srow = scale * (kk @ q[b, h, i])
                m = np.max(srow)
                e = np.exp(srow - m)
                l = np.sum(e)
                o[b, h, t] = (e / l) @ vv
                lse[b, h, t] = m + math.log(l)
    return o, lse


def online_softmax_attention(q, k, v, scale, causal, block_q=128, block_k=128):
    """The tiled loop of the unite.ai page ("Detalles de Implementación"), corrected.

    Query blocks outside, key/value blocks inside; running maximum M and running
    sum L per query row (initialised to -inf and 0), updated block by block with
    exp(M - M_new) (formula 2 of the same page; the online normaliser of the
    nisoo.com page).  The printed output update omits the factor L of the old
    sum; here O_new = (L * exp(M - M_new) * O + exp(S - M_new) V) / L_new.
    Returns (o, lse) so it can be compared with ``attention_fwd_ref``.
    """
    q = _as64(q)
    k = _as64(k)
    v = _as64(v)
    b_, h_, n, d = q.shape
    nk = k.shape[2]
    o = np.zeros_like(q)
    lse = np.zeros((b_, h_, n))
    for b in range(b_):
        for h in range(h_):
            for i0 in range(0, n, block_q):
                i1 = min(n, i0 + block_q)
                qb = q[b, h, i0:i1]
                ob = np.zeros((i1 - i0, d))
                mrow = np.full((i1 - i0, 1), -np.inf)
                lrow = np.zeros((i1 - i0, 1))
                for j0 in range(0, nk, block_k):
                    j1 = min(nk, j0 + block_k)
                    sb = scale * (qb @ k[b, h, j0:j1].T)
                    if causal:
                        qi = np.arange(i0, i1)[:, None]
                        kj = np.arange(j0, j1)[None, :]
                        sb = np.where(kj > qi + (nk - n), -np.inf, sb)
                    m_new = np.maximum(mrow, np.max(sb, axis=-1, keepdims=True))
                    # a row whose max is still -inf has seen no visible key yet
                    safe_m = np.where(np.isneginf(m_new), 0.0, m_new)
                    e = np.exp(sb - safe_m)
                    corr = np.exp(mrow - safe_m)
                    l_new = corr * lrow + np.sum(e, axis=-1, keepdims=True)
                    with np.errstate(invalid="ignore", divide="ignore"):
                        ob = np.where(
                            l_new > 0, (lrow * corr * ob + e @ v[b, h, j0:j1]) / l_new, 0.0
                        )
                    mrow, lrow = m_new, l_new
                o[b, h, i0:i1] = ob
                with np.errstate(divide="ignore"):
                    lse[b, h, i0:i1] = np.where(lrow > 0, mrow + np.log(np.where(lrow > 0, lrow, 1.0)), -np.inf)[:, 0]
    return o, lse


def _repeat_heads(x, group):
    """[B, Hkv, N, d] -> [B, Hkv*group, N, d]: key/value head j serves query heads
    j*group .. j*group + group - 1."""
    return np.repeat(_as64(x), group, axis=1)


def attention_fwd_gqa_ref(q, k, v, scale, causal):
    """Grouped-query (and multi-query) attention: Q has H heads, K and V have Hkv
    heads with Hkv dividing H, and query head h attends with key/value head
    h // (H / Hkv).  The attention variants named in "Atención Flash-2" (unite.ai
    page); the definition is the standard attention of each query head with its
    key/value head, so the oracle repeats K and V over the group.
    """
    group = q.shape[1] // k.shape[1]
    assert group * k.shape[1] == q.shape[1]
    return attention_fwd_ref(q, _repeat_heads(k, group), _repeat_heads(v, group), scale, causal)


def attention_bwd_gqa_ref(q, k, v, do, scale, causal):
    """Gradients of sum(O * dO) for grouped-query attention: dQ per query head;
    dK and dV of a key/value head are the sums over its query heads (chain rule
    through the repetition of K and V)."""
    b_, hkv, n, d = np.shape(k)
    group = q.shape[1] // hkv
    dq, dk_e, dv_e = attention_bwd_ref(q, _repeat_heads(k, group), _repeat_heads(v, group), do, scale,
                                       causal)
    dk = dk_e.reshape(b_, hkv, group, n, d).sum(axis=2)
    dv = dv_e.reshape(b_, hkv, group, n, d).sum(axis=2)
    return dq, dk, dv


# Facts of the OCP FP8 E4M3 format used by the FP8 forward ("Atención Flash-3",
# item "Soporte para FP8", of the unite.ai page names FP8 support; the format
# itself is not on the pages): 3 stored mantissa bits, so a value in the normal
# range (>= 2^-6) is rounded to nearest with relative error at most 2^-4, and
# below 2^-6 the spacing is 2^-9, so the absolute error is at most 2^-10.
E4M3_REL = 2.0**-4
E4M3_MIN_NORMAL = 2.0**-6
E4M3_SUB_ABS = 2.0**-10


def _e4m3_bound_from_scores(s, v):
    m = np.max(s, axis=-1, keepdims=True)
    m0 = np.where(np.isneginf(m), 0.0, m)
    p = np.exp(s - m0)
    l = np.sum(p, axis=-1, keepdims=True)
    av = np.abs(_as64(v))
    small = (p < E4M3_MIN_NORMAL) & ~np.isneginf(s)
    num = E4M3_REL * np.matmul(p, av) + E4M3_SUB_ABS * np.matmul(small.astype(np.float64), av)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(l > 0, num / np.where(l > 0, l, 1.0), 0.0)


def e4m3_p_rounding_bound(q, k, v, scale, causal, rows=None):
    """Worst-case |O_fp8 - O| per output element when the probabilities are
    rounded to e4m3 before P V (the FP8 forward), everything else exact.

    Reading (the pages give no error analysis): the kernel forms
    p'_j = g * p_j with p_j = exp(S_ij - m_i) <= 1 and a factor g >= 1 (its
    running maximum may trail the true one), rounds p'_j to e4m3 and divides the
    sum of p'_j v_j by the unrounded sum g * l.  The rounding error of each p'_j
    is at most 2^-4 p'_j, or 2^-10 when p'_j < 2^-6, so
        |dO_ic| <= (2^-4 sum_j p_j |V_jc| + 2^-10 sum_{j: p_j < 2^-6} |V_jc|) / l
    with l = sum_j p_j (g >= 1 only shrinks the second term).  Returns an array
    of O's shape, or with ``rows`` (query indices per head, as for
    ``attention_rows_ref``) the bound of those rows only, [B, H, R, d].
    """
    if rows is None:
        return _e4m3_bound_from_scores(scores(q, k, scale, causal), v)
    q, k, v = _as64(q), _as64(k), _as64(v)
    b_, h_, n, d = q.shape
    off = k.shape[2] - n
    out = np.zeros((b_, h_, len(rows[0]), d))
    for b in range(b_):
        for h in range(h_):
            for t, i in enumerate(rows[h]):
                last = int(i) + off + 1 if causal else k.shape[2]
                if last <= 0:
                    continue
                srow = scale * (k[b, h, :last] @ q[b, h, int(i)])
                out[b, h, t] = _e4m3_bound_from_scores(srow[None, :], v[b, h, :last])[0]
    return out
