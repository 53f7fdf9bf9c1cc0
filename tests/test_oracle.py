"""Pins for the fp64 oracle: closed forms, invariants, brute force, library
cross-checks and finite differences.  CPU only.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a missing mask) fails at least one of
them; ``test_planted_*`` checks that claim by planting such slips in copies of
the oracle and confirming a pin catches each one.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as orc

RNG = np.random.default_rng(1234)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# --- softmax pieces (unite.ai page, "La Matemática detrás de la Atención Flash")


def test_safe_softmax_rows_sum_to_one_and_match_textbook():
    x = rand(7, 33, scale=5.0)
    p = orc.safe_softmax(x)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-14, rtol=0)
    naive = np.exp(x) / np.exp(x).sum(-1, keepdims=True)  # no overflow at this range
    assert np.allclose(p, naive, atol=1e-15, rtol=1e-13)


def test_safe_softmax_survives_overflow_range():
    x = np.array([[1000.0, 1000.0 + math.log(3.0)]])
    p = orc.safe_softmax(x)
    assert np.allclose(p, [[0.25, 0.75]], atol=1e-15)


def test_softmax_merge_equals_full_softmax():
    for nx, ny in [(1, 1), (5, 9), (64, 64), (3, 200)]:
        x = rand(nx, scale=4.0)
        y = rand(ny, scale=4.0) + 3.0
        mx, my = x.max(), y.max()
        fx, fy = np.exp(x - mx), np.exp(y - my)
        merged, m, l = orc.softmax_merge(fx, mx, fx.sum(), fy, my, fy.sum())
        full = orc.safe_softmax(np.concatenate([x, y]))
        assert np.allclose(merged, full, atol=1e-15, rtol=1e-12)
        assert m == max(mx, my)
        assert math.isclose(m + math.log(l), np.log(np.exp(np.concatenate([x, y])).sum()), rel_tol=1e-13)


# --- forward: definition, closed forms, invariants


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k = rand(2, 3, 40, 8), rand(2, 3, 40, 8)
    s = orc.scores(q, k, 1 / math.sqrt(8), causal)
    _, lse = orc.attention_fwd_ref(q, k, rand(2, 3, 40, 8), 1 / math.sqrt(8), causal)
    p = np.exp(s - lse[..., None])
    assert np.allclose(p.sum(-1), 1.0, atol=1e-13, rtol=0)


def test_closed_form_two_keys():
    # scores [0, ln 3] -> weights [1/4, 3/4]; V = [4, 8] -> O = 7; LSE = ln 4.
    q = np.array([[[[1.0], [1.0]]]])
    k = np.array([[[[0.0], [math.log(3.0)]]]])
    v = np.array([[[[4.0], [8.0]]]])
    o, lse = orc.attention_fwd_ref(q, k, v, 1.0, False)
    assert np.allclose(o[0, 0, :, 0], [7.0, 7.0], atol=1e-13)
    assert np.allclose(lse[0, 0], [math.log(4.0)] * 2, atol=1e-14)
    o, lse = orc.attention_fwd_ref(q, k, v, 1.0, True)
    assert np.allclose(o[0, 0, :, 0], [4.0, 7.0], atol=1e-13)
    assert np.allclose(lse[0, 0], [0.0, math.log(4.0)], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_values(causal):
    n, d = 37, 16
    q = rand(1, 2, n, d)
    k = np.broadcast_to(rand(1, 2, 1, d), (1, 2, n, d)).copy()
    v = rand(1, 2, n, d)
    o, lse = orc.attention_fwd_ref(q, k, v, 0.3, causal)
    if causal:
        want = np.cumsum(v, axis=2) / np.arange(1, n + 1)[None, None, :, None]
        cnt = np.arange(1, n + 1)
    else:
        want = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        cnt = np.full(n, n)
    assert np.allclose(o, want, atol=1e-13)
    # LSE = scale * q.k + ln(count)
    sk = 0.3 * np.einsum("bhid,bhd->bhi", q, k[:, :, 0])
    assert np.allclose(lse, sk + np.log(cnt)[None, None], atol=1e-12)


def test_dominant_key_selects_its_value():
    n, d = 20, 8
    q = rand(1, 1, n, d)
    k = rand(1, 1, n, d, scale=0.1)
    target = (np.arange(n) * 7 + 3) % n
    for i in range(n):
        k[0, 0, target[i]] = 0.0
    # make key target[i] dominate row i by 2000 in score: exp(-2000) == 0 in fp64
    q = np.zeros((1, 1, n, d))
    for i in range(n):
        q[0, 0, i, i % d] = 1.0
    k = np.zeros((1, 1, n, d))
    v = rand(1, 1, n, d)
    for j in range(n):
        k[0, 0, j, j % d] = 2000.0 * (1 + j // d)
    o, _ = orc.attention_fwd_ref(q, k, v, 1.0, False)
    for i in range(n):
        # keys sharing coordinate i % d: the one with the largest multiple wins
        cands = [j for j in range(n) if j % d == i % d]
        win = max(cands, key=lambda j: 1 + j // d)
        assert np.allclose(o[0, 0, i], v[0, 0, win], atol=1e-12)


def test_causal_first_row_is_first_value():
    q, k, v = rand(2, 2, 9, 4), rand(2, 2, 9, 4), rand(2, 2, 9, 4)
    o, lse = orc.attention_fwd_ref(q, k, v, 0.7, True)
    assert np.array_equal(o[:, :, 0], v[:, :, 0])
    assert np.allclose(lse[:, :, 0], 0.7 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    q, k, v = rand(1, 2, 30, 8), rand(1, 2, 30, 8), rand(1, 2, 30, 8)
    u = rand(8)
    o1, l1 = orc.attention_fwd_ref(q, k, v, 0.5, causal)
    o2, l2 = orc.attention_fwd_ref(q, k + u, v, 0.5, causal)
    assert np.allclose(o1, o2, atol=1e-12)
    assert np.allclose(l2 - l1, 0.5 * np.einsum("bhid,d->bhi", q, u), atol=1e-12)


def test_permutation_equivariance_non_causal():
    q, k, v = rand(1, 1, 25, 8), rand(1, 1, 25, 8), rand(1, 1, 25, 8)
    pq, pk = RNG.permutation(25), RNG.permutation(25)
    o1, l1 = orc.attention_fwd_ref(q, k, v, 0.4, False)
    o2, l2 = orc.attention_fwd_ref(q[:, :, pq], k[:, :, pk], v[:, :, pk], 0.4, False)
    assert np.allclose(o2, o1[:, :, pq], atol=1e-13)
    assert np.allclose(l2, l1[:, :, pq], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_pure_python_brute_force(causal):
    n, d = 6, 3
    q, k, v = rand(1, 1, n, d), rand(1, 1, n, d), rand(1, 1, n, d)
    sc = 0.8
    o, lse = orc.attention_fwd_ref(q, k, v, sc, causal)
    for i in range(n):
        keys = range(i + 1) if causal else range(n)
        w = {j: math.exp(sc * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d))) for j in keys}
        z = sum(w.values())
        assert math.isclose(lse[0, 0, i], math.log(z), rel_tol=1e-13, abs_tol=1e-13)
        for c in range(d):
            ref = sum(w[j] * v[0, 0, j, c] for j in keys) / z
            assert math.isclose(o[0, 0, i, c], ref, rel_tol=1e-12, abs_tol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_library_sdpa_cross_check(causal):
    q, k, v = rand(2, 3, 50, 16), rand(2, 3, 50, 16), rand(2, 3, 50, 16)
    o, lse = orc.attention_fwd_ref(q, k, v, 0.25, causal)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ot = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.25)
    assert np.allclose(o, ot.numpy(), atol=1e-13)
    s = 0.25 * torch.einsum("bhid,bhjd->bhij", tq, tk)
    if causal:
        s = s.masked_fill(torch.ones(50, 50, dtype=torch.bool).triu(1), float("-inf"))
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,bq,bk", [(300, 128, 128), (300, 256, 256), (300, 100, 64), (64, 128, 128)])
def test_online_tiled_loop_equals_full(causal, n, bq, bk):
    q, k, v = rand(1, 2, n, 16, scale=2.0), rand(1, 2, n, 16, scale=2.0), rand(1, 2, n, 16)
    o1, l1 = orc.attention_fwd_ref(q, k, v, 0.25, causal)
    o2, l2 = orc.online_softmax_attention(q, k, v, 0.25, causal, bq, bk)
    assert np.allclose(o1, o2, atol=1e-12)
    assert np.allclose(l1, l2, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_equal_full_rows(causal):
    q, k, v = rand(1, 3, 70, 8), rand(1, 3, 70, 8), rand(1, 3, 70, 8)
    o, lse = orc.attention_fwd_ref(q, k, v, 0.35, causal)
    rows = [np.array([0, 5, 33, 69]), np.array([1, 2, 3, 4]), np.array([0, 17, 18, 69])]
    orow, lrow = orc.attention_rows_ref(q, k, v, rows, 0.35, causal)
    for h in range(3):
        assert np.allclose(orow[0, h], o[0, h, rows[h]], atol=1e-13)
        assert np.allclose(lrow[0, h], lse[0, h, rows[h]], atol=1e-13)


# --- backward: finite differences and autograd of the definition


def _loss(q, k, v, do, sc, causal):
    o, _ = orc.attention_fwd_ref(q, k, v, sc, causal)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_central_finite_differences(causal):
    n, d, sc, h = 6, 3, 0.9, 1e-6
    q, k, v, do = rand(1, 1, n, d), rand(1, 1, n, d), rand(1, 1, n, d), rand(1, 1, n, d)
    dq, dk, dv = orc.attention_bwd_ref(q, k, v, do, sc, causal)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, sc, causal)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, sc, causal)
            num[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd(causal):
    q, k, v, do = rand(2, 2, 40, 8), rand(2, 2, 40, 8), rand(2, 2, 40, 8), rand(2, 2, 40, 8)
    dq, dk, dv = orc.attention_bwd_ref(q, k, v, do, 0.3, causal)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    ot = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.3)
    ot.backward(torch.from_numpy(do))
    assert np.allclose(dq, tq.grad.numpy(), atol=1e-12)
    assert np.allclose(dk, tk.grad.numpy(), atol=1e-12)
    assert np.allclose(dv, tv.grad.numpy(), atol=1e-12)


def test_backward_row_term_equals_rowsum_do_o():
    # rowsum(P * dP) == rowsum(dO * O): the identity the GPU preprocess relies on.
    q, k, v, do = rand(1, 2, 30, 8), rand(1, 2, 30, 8), rand(1, 2, 30, 8), rand(1, 2, 30, 8)
    o, lse = orc.attention_fwd_ref(q, k, v, 0.5, True)
    p = np.exp(orc.scores(q, k, 0.5, True) - lse[..., None])
    dp = np.einsum("bhid,bhjd->bhij", do, v)
    assert np.allclose((p * dp).sum(-1), (do * o).sum(-1), atol=1e-12)


# --- grouped-query attention


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_central_finite_differences(causal):
    # H = 4 query heads sharing Hkv = 2 key/value heads: dK, dV must sum the group
    n, d, sc, h = 5, 3, 0.8, 1e-6
    q, k, v, do = rand(1, 4, n, d), rand(1, 2, n, d), rand(1, 2, n, d), rand(1, 4, n, d)
    dq, dk, dv = orc.attention_bwd_gqa_ref(q, k, v, do, sc, causal)

    def loss(q_, k_, v_):
        o, _ = orc.attention_fwd_gqa_ref(q_, k_, v_, sc, causal)
        return float(np.sum(o * do))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args = {"q": q, "k": k, "v": v}
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args[name] = xp
            lp = loss(args["q"], args["k"], args["v"])
            args[name] = xm
            lm = loss(args["q"], args["k"], args["v"])
            num[idx] = (lp - lm) / (2 * h)
        assert np.linalg.norm(num - g) / np.linalg.norm(g) < 1e-6, name


def test_gqa_single_group_is_plain_attention_per_head():
    q, k, v = rand(2, 6, 20, 8), rand(2, 3, 20, 8), rand(2, 3, 20, 8)
    o, lse = orc.attention_fwd_gqa_ref(q, k, v, 0.4, True)
    for h in range(6):
        o1, l1 = orc.attention_fwd_ref(q[:, h : h + 1], k[:, h // 2 : h // 2 + 1], v[:, h // 2 : h // 2 + 1], 0.4, True)
        assert np.allclose(o[:, h : h + 1], o1, atol=1e-14) and np.allclose(lse[:, h : h + 1], l1, atol=1e-14)


# --- stored regression fixture (written by tests/golden/make_golden.py, oracle only)


def test_golden_fixture_reproduces():
    with open(os.path.join(GOLDEN, "oracle_small.json")) as f:
        cases = json.load(f)["cases"]
    assert cases
    for c in cases:
        q, k, v, do = (np.array(c[x]) for x in ("q", "k", "v", "do"))
        o, lse = orc.attention_fwd_ref(q, k, v, c["scale"], c["causal"])
        dq, dk, dv = orc.attention_bwd_ref(q, k, v, do, c["scale"], c["causal"])
        for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            assert np.allclose(got, np.array(c[name]), atol=1e-12), (c["name"], name)


# --- planted mistakes: each plausible slip must trip a pin above


def _printed_toy_loop(q, k, v, scale, causal, block):
    """The page's loop with its printed output update (old-sum factor L missing)."""
    b_, h_, n, d = q.shape
    o = np.zeros_like(q)
    for b in range(b_):
        for h in range(h_):
            for i0 in range(0, n, block):
                qb = q[b, h, i0 : i0 + block]
                ob = np.zeros_like(qb)
                m = np.full((len(qb), 1), -np.inf)
                l = np.zeros((len(qb), 1))
                for j0 in range(0, n, block):
                    sb = scale * qb @ k[b, h, j0 : j0 + block].T
                    mn = np.maximum(m, sb.max(-1, keepdims=True))
                    e = np.exp(sb - mn)
                    c = np.exp(m - mn)
                    ln = c * l + e.sum(-1, keepdims=True)
                    ob = (c * ob + e @ v[b, h, j0 : j0 + block]) / ln
                    m, l = mn, ln
                o[b, h, i0 : i0 + block] = ob
    return o


def test_planted_printed_toy_update_is_caught():
    q, k, v = rand(1, 1, 300, 8), rand(1, 1, 300, 8), rand(1, 1, 300, 8)
    o_ref, _ = orc.attention_fwd_ref(q, k, v, 0.3, False)
    # one block: printed form coincides with the definition
    assert np.allclose(_printed_toy_loop(q, k, v, 0.3, False, 512), o_ref, atol=1e-12)
    # several blocks: it does not, so the blockwise pin would catch it
    assert not np.allclose(_printed_toy_loop(q, k, v, 0.3, False, 128), o_ref, atol=1e-3)


def test_planted_forward_slips_are_caught(monkeypatch):
    q, k, v = rand(1, 2, 12, 4), rand(1, 2, 12, 4), rand(1, 2, 12, 4)
    good_o, good_l = orc.attention_fwd_ref(q, k, v, 0.6, True)

    def caught():
        o, l = orc.attention_fwd_ref(q, k, v, 0.6, True)
        return not (np.allclose(o, good_o, atol=1e-12) and np.allclose(l, good_l, atol=1e-12))

    real_scores = orc.scores
    slips = {
        "mask_off_by_one": lambda q_, k_, s, c: np.where(
            np.triu(np.ones((12, 12), bool), k=2), -np.inf, s * np.einsum("bhid,bhjd->bhij", q_, k_)
        ),
        "wrong_sign": lambda q_, k_, s, c: -real_scores(q_, k_, s, c),
        "transposed": lambda q_, k_, s, c: np.swapaxes(real_scores(q_, k_, s, c), -1, -2),
        "no_scale": lambda q_, k_, s, c: real_scores(q_, k_, 1.0, c),
    }
    for name, fn in slips.items():
        monkeypatch.setattr(orc, "scores", fn)
        assert caught(), name
    monkeypatch.setattr(orc, "scores", real_scores)
    assert not caught()


def test_planted_backward_slip_is_caught():
    # dropping the row term of the softmax Jacobian fails finite differences
    n, d, sc, h = 5, 2, 0.7, 1e-6
    q, k, v, do = rand(1, 1, n, d), rand(1, 1, n, d), rand(1, 1, n, d), rand(1, 1, n, d)
    s = orc.scores(q, k, sc, False)
    p = orc.safe_softmax(s)
    dp = np.einsum("bhid,bhjd->bhij", do, v)
    dq_bad = sc * np.einsum("bhij,bhjd->bhid", p * dp, k)
    num = np.zeros_like(q)
    for idx in np.ndindex(q.shape):
        qp, qm = q.copy(), q.copy()
        qp[idx] += h
        qm[idx] -= h
        num[idx] = (_loss(qp, k, v, do, sc, False) - _loss(qm, k, v, do, sc, False)) / (2 * h)
    assert np.linalg.norm(num - dq_bad) / np.linalg.norm(num) > 1e-3


# --- unequal query and key lengths (Nq != Nk); causal mask aligned bottom right


@pytest.mark.parametrize("nq,nk", [(3, 5), (5, 3), (1, 4), (4, 1), (6, 6)])
def test_unequal_lengths_pure_python_brute_force(nq, nk):
    d, sc = 3, 0.7
    q, k, v = rand(1, 1, nq, d), rand(1, 1, nk, d), rand(1, 1, nk, d)
    o, lse = orc.attention_fwd_ref(q, k, v, sc, True)
    for i in range(nq):
        keys = [j for j in range(nk) if j <= i + nk - nq]
        if not keys:  # no visible key: O = 0, LSE = -inf
            assert lse[0, 0, i] == -np.inf and np.all(o[0, 0, i] == 0.0)
            continue
        w = {j: math.exp(sc * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d))) for j in keys}
        z = sum(w.values())
        assert math.isclose(lse[0, 0, i], math.log(z), rel_tol=1e-13, abs_tol=1e-13)
        for c in range(d):
            ref = sum(w[j] * v[0, 0, j, c] for j in keys) / z
            assert math.isclose(o[0, 0, i, c], ref, rel_tol=1e-12, abs_tol=1e-13)


def test_fewer_queries_are_the_last_rows_of_the_square_case():
    # bottom-right alignment: Nq queries against Nk keys are the last Nq rows of
    # the square causal problem whose queries end with them
    nk, nq = 40, 13
    q, k, v = rand(2, 2, nk, 8), rand(2, 2, nk, 8), rand(2, 2, nk, 8)
    o_sq, l_sq = orc.attention_fwd_ref(q, k, v, 0.3, True)
    o, lse = orc.attention_fwd_ref(q[:, :, nk - nq :], k, v, 0.3, True)
    assert np.allclose(o, o_sq[:, :, nk - nq :], atol=1e-14)
    assert np.allclose(lse, l_sq[:, :, nk - nq :], atol=1e-14)


def test_more_queries_than_keys_mask_the_first_rows():
    nq, nk = 30, 11
    q, k, v = rand(1, 2, nq, 8), rand(1, 2, nk, 8), rand(1, 2, nk, 8)
    o, lse = orc.attention_fwd_ref(q, k, v, 0.4, True)
    assert np.all(o[:, :, : nq - nk] == 0.0) and np.all(np.isneginf(lse[:, :, : nq - nk]))
    o_sq, l_sq = orc.attention_fwd_ref(q[:, :, nq - nk :], k, v, 0.4, True)
    assert np.allclose(o[:, :, nq - nk :], o_sq, atol=1e-14)
    assert np.allclose(lse[:, :, nq - nk :], l_sq, atol=1e-14)


def test_single_query_sees_every_key():
    q, k, v = rand(1, 3, 1, 16), rand(1, 3, 77, 16), rand(1, 3, 77, 16)
    o_c, l_c = orc.attention_fwd_ref(q, k, v, 0.25, True)
    o_n, l_n = orc.attention_fwd_ref(q, k, v, 0.25, False)
    assert np.allclose(o_c, o_n, atol=1e-15) and np.allclose(l_c, l_n, atol=1e-15)


def test_unequal_lengths_library_sdpa_cross_check():
    # torch's SDPA with an explicit boolean mask of the same convention
    for nq, nk in [(20, 50), (50, 20)]:
        q, k, v = rand(1, 2, nq, 16), rand(1, 2, nk, 16), rand(1, 2, nk, 16)
        o, _ = orc.attention_fwd_ref(q, k, v, 0.25, True)
        keep = torch.ones(nq, nk, dtype=torch.bool).tril(nk - nq)
        ot = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(x) for x in (q, k, v)), attn_mask=keep, scale=0.25)
        rows = slice(max(0, nq - nk), nq)  # torch gives NaN on rows with no visible key
        assert np.allclose(o[:, :, rows], ot.numpy()[:, :, rows], atol=1e-13)


@pytest.mark.parametrize("nq,nk", [(200, 300), (300, 200), (130, 500)])
def test_unequal_lengths_online_loop_and_sampled_rows(nq, nk):
    q, k, v = rand(1, 2, nq, 8, scale=2.0), rand(1, 2, nk, 8, scale=2.0), rand(1, 2, nk, 8)
    o1, l1 = orc.attention_fwd_ref(q, k, v, 0.3, True)
    o2, l2 = orc.online_softmax_attention(q, k, v, 0.3, True, 128, 64)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    rows = [np.array([0, 1, nq // 2, nq - 1])] * 2
    orow, lrow = orc.attention_rows_ref(q, k, v, rows, 0.3, True)
    for h in range(2):
        assert np.allclose(orow[0, h], o1[0, h, rows[h]], atol=1e-13)
        assert np.array_equal(np.isneginf(lrow[0, h]), np.isneginf(l1[0, h, rows[h]]))
        fin = np.isfinite(l1[0, h, rows[h]])
        assert np.allclose(lrow[0, h][fin], l1[0, h, rows[h]][fin], atol=1e-13)


@pytest.mark.parametrize("nq,nk", [(3, 6), (6, 3)])
def test_unequal_lengths_backward_finite_differences(nq, nk):
    d, sc, hh = 3, 0.8, 1e-6
    q, k, v, do = rand(1, 1, nq, d), rand(1, 1, nk, d), rand(1, 1, nk, d), rand(1, 1, nq, d)
    dq, dk, dv = orc.attention_bwd_ref(q, k, v, do, sc, True)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += hh
            xm[idx] -= hh
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, sc, True)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, sc, True)
            num[idx] = (lp - lm) / (2 * hh)
        assert np.linalg.norm(num - g) <= 1e-6 * max(1.0, np.linalg.norm(g)), name
    if nq > nk:  # queries with no visible key have no gradient
        assert np.all(dq[:, :, : nq - nk] == 0.0)


def test_planted_top_left_alignment_is_caught():
    # a mask aligned at the top left (j <= i) instead of the bottom right fails the
    # suffix pin above whenever Nq != Nk
    nk, nq = 40, 13
    q, k, v = rand(1, 1, nk, 8), rand(1, 1, nk, 8), rand(1, 1, nk, 8)
    o_sq, _ = orc.attention_fwd_ref(q, k, v, 0.3, True)
    s = 0.3 * np.einsum("bhid,bhjd->bhij", q[:, :, nk - nq :], k)
    s = np.where(np.triu(np.ones((nq, nk), bool), k=1), -np.inf, s)
    p = orc.safe_softmax(s)
    o_bad = np.einsum("bhij,bhjd->bhid", p, v)
    assert not np.allclose(o_bad, o_sq[:, :, nk - nq :], atol=1e-3)


# ---------------------------------------------------------------- FP8 reading


def _simulate_fp8_p(q, k, v, scale, causal, stale_log2=0.0):
    """O with every probability rounded to e4m3 before P V, the way the FP8
    forward does it: p' = g * exp(S - m) in float32 with g = 2^stale_log2 (a
    running maximum that trails the true one), rounded to e4m3 by torch, summed
    against V and divided by the unrounded g * l."""
    s = orc.scores(q, k, scale, causal)
    m = np.max(s, axis=-1, keepdims=True)
    g = 2.0**stale_log2
    p = (g * np.exp(s - m)).astype(np.float32)
    p8 = torch.from_numpy(p).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    l = np.sum(p.astype(np.float64), axis=-1, keepdims=True)
    return np.matmul(p8, v) / l


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("gain,stale", [(1.0, 0.0), (1.0, 5.3), (1.0, 8.0), (4.0, 0.0), (4.0, 7.5)])
def test_e4m3_rounding_bound_holds_for_simulated_fp8(causal, gain, stale):
    rng = np.random.default_rng(int(10 * gain + stale))
    q, k, v = (rng.normal(size=(1, 2, 300, 64)) for _ in range(3))
    q, k = q * gain, k * gain
    o_ref, _ = orc.attention_fwd_ref(q, k, v, 0.125, causal)
    o8 = _simulate_fp8_p(q, k, v, 0.125, causal, stale)
    bound = orc.e4m3_p_rounding_bound(q, k, v, 0.125, causal)
    err = np.abs(o8 - o_ref)
    assert np.all(err <= bound * (1 + 1e-6) + 1e-12)
    # the bound is a worst case, but not a vacuous one
    assert np.max(err / np.maximum(bound, 1e-300)) > 0.05


def test_e4m3_rounding_noise_is_what_the_tolerance_reading_says():
    # rounding P to 3 mantissa bits adds relative noise of about 2^-3 / sqrt(12)
    # times the mean of 2^e / p over a binade (0.72), i.e. ~2.6 % in O; the FP8
    # parity bound allows rel-L2 <= 5e-2
    rng = np.random.default_rng(3)
    q, k, v = (rng.normal(size=(1, 4, 1024, 128)) for _ in range(3))
    scale = 1 / math.sqrt(128)
    for causal in (False, True):
        o_ref, _ = orc.attention_fwd_ref(q, k, v, scale, causal)
        o8 = _simulate_fp8_p(q, k, v, scale, causal)
        rel = np.linalg.norm(o8 - o_ref) / np.linalg.norm(o_ref)
        assert 0.01 < rel < 0.04, rel


def test_e4m3_bound_rows_equal_full_bound():
    rng = np.random.default_rng(4)
    q, k, v = (rng.normal(size=(1, 2, 200, 32)) for _ in range(3))
    full = orc.e4m3_p_rounding_bound(q, k, v, 0.2, True)
    rows = [np.array([0, 17, 199]), np.array([3, 100, 150])]
    part = orc.e4m3_p_rounding_bound(q, k, v, 0.2, True, rows=rows)
    for h in range(2):
        assert np.allclose(part[0, h], full[0, h, rows[h]], rtol=1e-12, atol=1e-15)


def test_planted_fp8_slips_break_the_e4m3_bound():
    # the bound admits e4m3 rounding of P and nothing else: a 10 % error in the
    # score scale (a descale applied wrongly) or a running-maximum factor that is
    # not divided out again must leave it
    rng = np.random.default_rng(5)
    q, k, v = (rng.normal(size=(1, 2, 256, 64)) for _ in range(3))
    o_ref, _ = orc.attention_fwd_ref(q, k, v, 0.125, False)
    bound = orc.e4m3_p_rounding_bound(q, k, v, 0.125, False)
    wrong_scale = _simulate_fp8_p(q, k * 1.1, v, 0.125, False)
    assert np.any(np.abs(wrong_scale - o_ref) > bound)
    kept_factor = _simulate_fp8_p(q, k, v, 0.125, False, stale_log2=1.0) * 2.0
    assert np.any(np.abs(kept_factor - o_ref) > bound)


def test_fp8_inputs_recipe():
    from exact_tiled_attention_35_b200.inputs import fp8_values, make_fp8_inputs, make_inputs

    q8, k8, v8, qs, ks, vs = make_fp8_inputs(1, 2, 100, 64, seed=3)
    q32 = make_inputs(1, 2, 100, 64, dtype=torch.float32, seed=3)[0].double().numpy()
    for x8, s in ((q8, qs), (k8, ks), (v8, vs)):
        assert x8.dtype == torch.float8_e4m3fn
        assert float(x8.float().abs().max()) == 448.0  # amax lands on the top of the range
    # decoded values are within e4m3 rounding of the drawn ones
    err = np.abs(fp8_values(q8, qs) - q32)
    assert np.all(err <= 2.0**-4 * np.abs(q32) + 2.0**-10 * qs + 1e-12)
