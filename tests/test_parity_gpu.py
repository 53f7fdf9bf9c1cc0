"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the same
seeded inputs.  GPU only.  Bounds and error measures: tests/parity.py (bf16
forward O within 1e-2 of the oracle before the output's bf16 rounding, rel-L2
<= 5e-3, LSE max-abs <= 1e-2; dQ/dK/dV rel-L2 <= 2e-2).  Outputs are filled with
NaN before every call, so a row or gradient the kernels never write fails.

The five workloads at their full sizes are checked in test_parity_report_gpu.py.
"""

import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_35_b200 as fa
from exact_tiled_attention_35_b200.inputs import make_inputs, to_f64
from oracle import attention_bwd_ref, attention_fwd_ref
from parity import O_MAXABS, check_bwd, check_fwd, max_abs, rel_l2

pytestmark = pytest.mark.gpu


def run_fwd(B, H, N, d, causal, dtype=torch.bfloat16, seed=0, gain=1.0):
    q, k, v = make_inputs(B, H, N, d, dtype=dtype, seed=seed, qk_gain=gain)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.forward(qd, kd, vd, causal=causal, out=o, lse=lse)
    fa.check_device_status()
    return (q, k, v), to_f64(o), to_f64(lse)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load_library()


# ---------------------------------------------------------------- forward


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 77, 128, 200, 256, 384, 640, 1000])
def test_forward_sweep(N, causal, d):
    (q, k, v), o, lse = run_fwd(1, 3, N, d, causal, seed=N + d)
    o_ref, lse_ref = attention_fwd_ref(to_f64(q), to_f64(k), to_f64(v), 1 / math.sqrt(d), causal)
    check_fwd(o, lse, o_ref, lse_ref, (N, causal, d))


@pytest.mark.parametrize("seed", [1, 2])
def test_forward_several_heads_and_batches(seed):
    (q, k, v), o, lse = run_fwd(3, 5, 300, 128, True, seed=seed)
    o_ref, lse_ref = attention_fwd_ref(to_f64(q), to_f64(k), to_f64(v), 1 / math.sqrt(128), True)
    check_fwd(o, lse, o_ref, lse_ref, seed)


@pytest.mark.parametrize("N,causal", [(256, True), (333, False)])
def test_forward_fp32_sweep(N, causal):
    (q, k, v), o, lse = run_fwd(2, 2, N, 128, causal, dtype=torch.float32, seed=5)
    o_ref, lse_ref = attention_fwd_ref(to_f64(q), to_f64(k), to_f64(v), 1 / math.sqrt(128), causal)
    check_fwd(o, lse, o_ref, lse_ref, N, bf16_out=False)


def test_forward_is_deterministic():
    q, k, v = (t.cuda() for t in make_inputs(1, 4, 1000, 128, seed=9))
    o1, l1 = fa.forward(q, k, v, causal=True)
    o2, l2 = fa.forward(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 32, 4096, 128, True), (1, 12, 16384, 64, True),
                                             (1, 7, 32768, 64, True), (4, 16, 1024, 64, False)])
def test_forward_schedule_covers_every_item_once(B, H, N, d, causal):
    # The persistent forward hands (head, query-tile pair) items to CTAs through
    # a ticket counter, in L2-sized head chunks.  Each item's arithmetic does not
    # depend on which CTA runs it or when, so the whole launch must equal, bit
    # for bit, launches of one head each (a single chunk, a different order), and
    # a second whole launch (a different dynamic assignment).
    q, k, v = (t.cuda() for t in make_inputs(B, H, N, d, seed=21))
    o, lse = fa.forward(q, k, v, causal=causal)
    o2, lse2 = fa.forward(q, k, v, causal=causal)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    for b in range(B):
        for h in range(H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            oh, lh = fa.forward(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), causal=causal)
            assert torch.equal(oh, o[sl]) and torch.equal(lh, lse[sl]), (b, h)
    fa.check_device_status()


def test_forward_ticket_slots_reset_across_many_launches():
    # More launches than the scheduler has ticket slots: every slot is reused, so a
    # slot left dirty by a previous launch would make CTAs skip items.
    q, k, v = (t.cuda() for t in make_inputs(1, 6, 1000, 64, seed=22))
    o0, l0 = fa.forward(q, k, v, causal=True)
    o = torch.empty_like(o0)
    lse = torch.empty_like(l0)
    bad = torch.zeros((), dtype=torch.bool, device="cuda")
    for _ in range(600):
        o.fill_(float("nan"))
        fa.forward(q, k, v, causal=True, out=o, lse=lse)
        bad |= (o != o0).any() | (lse != l0).any()
    assert not bool(bad)
    fa.check_device_status()


def test_forward_key_shift_invariance_on_gpu():
    # adding one vector u to every key leaves O unchanged (the LSE shift is checked
    # against the oracle on the shifted keys)
    B, H, N, d = 1, 2, 512, 64
    q, k, v = make_inputs(B, H, N, d, seed=11)
    u = torch.zeros(d)
    u[::8] = 1.0
    k2 = (k.float() + u).to(torch.bfloat16)
    qd, kd, vd, k2d = (t.cuda() for t in (q, k, v, k2))
    o1, _ = fa.forward(qd, kd, vd)
    o2, l2 = fa.forward(qd, k2d, vd)
    assert max_abs(to_f64(o1), to_f64(o2)) <= O_MAXABS
    o_ref, l_ref = attention_fwd_ref(to_f64(q), to_f64(k2), to_f64(v), 1 / math.sqrt(d), False)
    check_fwd(to_f64(o2), to_f64(l2), o_ref, l_ref, "shifted")


# ---------------------------------------------------------------- backward


def run_bwd(B, H, N, d, causal, dtype=torch.bfloat16, seed=0):
    q, k, v, do = make_inputs(B, H, N, d, dtype=dtype, seed=seed, with_do=True)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, causal=causal)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    fa.backward(qd, kd, vd, o, dod, lse, causal=causal, dq=dq, dk=dk, dv=dv)
    fa.check_device_status()
    return (q, k, v, do), tuple(to_f64(x) for x in (dq, dk, dv))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 256, 384, 700])
def test_backward_sweep(N, causal, d):
    (q, k, v, do), got = run_bwd(1, 2, N, d, causal, seed=N)
    ref = attention_bwd_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), 1 / math.sqrt(d), causal)
    check_bwd(got, ref, (N, causal, d))


def test_backward_fp32_storage():
    (q, k, v, do), got = run_bwd(1, 2, 300, 64, True, dtype=torch.float32, seed=4)
    ref = attention_bwd_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), 1 / 8.0, True)
    for g, r in zip(got, ref):
        assert rel_l2(g, r) < 1e-5


@pytest.mark.parametrize("B,H,Hkv,N,d,causal", [(2, 16, 16, 2048, 128, True), (2, 32, 32, 4096, 128, True),
                                                 (1, 24, 6, 4096, 64, True), (1, 8, 8, 8192, 128, False)])
def test_backward_schedule_covers_every_tile_once(B, H, Hkv, N, d, causal):
    # The persistent backward hands out its (key/value head, key tile) work
    # items from a ticket counter, in L2-sized head chunks.  dK and dV of a key
    # tile come from one item whatever the order or the CTA that takes it, so a
    # multi-chunk launch must give them bit for bit as launches of one key/value
    # head each do (an item skipped or taken twice would show); dQ is summed by
    # reduce-adds in an order that varies, so it is held to fp32 rounding.
    q, k, v, do = (t.cuda() for t in make_inputs(B, H, N, d, seed=23, with_do=True))
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    o, lse = fa.forward_gqa(q, k, v, causal=causal)
    dq, dk, dv = fa.backward_gqa(q, k, v, o, do, lse, causal=causal)
    G = H // Hkv
    for b in range(B):
        for hk in range(Hkv):
            qs = (slice(b, b + 1), slice(hk * G, (hk + 1) * G))
            ks = (slice(b, b + 1), slice(hk, hk + 1))
            dq1, dk1, dv1 = fa.backward_gqa(q[qs].contiguous(), k[ks].contiguous(), v[ks].contiguous(),
                                            o[qs].contiguous(), do[qs].contiguous(), lse[qs].contiguous(),
                                            causal=causal)
            assert torch.equal(dk1, dk[ks]) and torch.equal(dv1, dv[ks]), (b, hk)
            rel = float((dq1.float() - dq[qs].float()).norm() / dq1.float().norm())
            assert rel < 1e-3, (b, hk, rel)
    fa.check_device_status()


def test_backward_ignores_workspace_contents_and_resets_its_counters():
    # The workspace's contents are ignored on entry: one filled with 0xFF bytes
    # (the main kernel's two work-item counters included) gives the dK, dV of a
    # zeroed one bit for bit, and the main kernel leaves both counters at zero
    # (its last CTA resets them).  The counters are the last 256-byte segment.
    B, H, N, d = 1, 8, 1000, 128
    q, k, v, do = (t.cuda() for t in make_inputs(B, H, N, d, seed=31, with_do=True))
    o, lse = fa.forward(q, k, v, causal=True)
    size = fa.workspace_size(B, H, N, d)
    ref = fa.backward(q, k, v, o, do, lse, causal=True,
                      workspace=torch.zeros(size, dtype=torch.uint8, device="cuda"))
    ws = torch.full((size,), 255, dtype=torch.uint8, device="cuda")
    for _ in range(3):  # the same workspace again and again
        got = fa.backward(q, k, v, o, do, lse, causal=True, workspace=ws)
        fa.check_device_status()
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
        rel = float((got[0].float() - ref[0].float()).norm() / ref[0].float().norm())
        assert rel < 1e-3, rel
        assert ws[size - 256:size - 240].view(torch.int64).tolist() == [0, 0]


# ---------------------------------------------------------------- grouped-query


@pytest.mark.parametrize("H,Hkv", [(8, 2), (8, 1), (4, 4)])
@pytest.mark.parametrize("N,causal,d", [(300, True, 128), (256, False, 64), (640, True, 64)])
def test_gqa_forward_and_backward(H, Hkv, N, causal, d):
    from exact_tiled_attention_35_b200.inputs import make_inputs
    from oracle import attention_bwd_gqa_ref, attention_fwd_gqa_ref

    q, _, _, do = make_inputs(1, H, N, d, seed=H * 10 + Hkv, with_do=True)
    _, k, v = make_inputs(1, Hkv, N, d, seed=7 + Hkv)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward_gqa(qd, kd, vd, causal=causal)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    fa.backward_gqa(qd, kd, vd, o, dod, lse, causal=causal, dq=dq, dk=dk, dv=dv)
    fa.check_device_status()
    scale = 1 / math.sqrt(d)
    o_ref, lse_ref = attention_fwd_gqa_ref(to_f64(q), to_f64(k), to_f64(v), scale, causal)
    check_fwd(to_f64(o), to_f64(lse), o_ref, lse_ref, (H, Hkv, N))
    ref = attention_bwd_gqa_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), scale, causal)
    check_bwd(tuple(to_f64(x) for x in (dq, dk, dv)), ref, (H, Hkv, N))


def test_gqa_with_full_heads_matches_multi_head_bitwise():
    q, k, v = (t.cuda() for t in make_inputs(2, 4, 384, 128, seed=3))
    o1, l1 = fa.forward(q, k, v, causal=True)
    o2, l2 = fa.forward_gqa(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ---------------------------------------------------------------- unequal query / key lengths


def _check_fwd_with_empty_rows(o, lse, o_ref, lse_ref, what):
    # rows that see no key: O = 0 and LSE = -inf exactly; the rest as check_fwd
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), what
    assert np.all(o[empty] == 0.0), what
    full = ~empty
    if np.any(full):
        check_fwd(o[full], lse[full], o_ref[full], lse_ref[full], what)


def _qk_inputs(B, H, Hkv, Nq, Nk, d, seed):
    q, do = make_inputs(B, H, Nq, d, seed=seed, with_do=True)[0::3]
    k, v = make_inputs(B, Hkv, Nk, d, seed=seed + 100)[1:3]
    return q, k, v, do


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (77, 300), (128, 1024), (300, 77), (1000, 1), (384, 130),
                                   (200, 201), (640, 256)])
def test_forward_unequal_lengths(Nq, Nk, causal, d):
    from oracle import attention_fwd_gqa_ref

    q, k, v, _ = _qk_inputs(1, 4, 2, Nq, Nk, d, seed=Nq + Nk)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:3], float("nan"), device="cuda")
    fa.forward_qk(qd, kd, vd, causal=causal, out=o, lse=lse)
    fa.check_device_status()
    o_ref, lse_ref = attention_fwd_gqa_ref(to_f64(q), to_f64(k), to_f64(v), 1 / math.sqrt(d), causal)
    _check_fwd_with_empty_rows(to_f64(o), to_f64(lse), o_ref, lse_ref, (Nq, Nk, causal, d))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(77, 300), (300, 77), (128, 640), (1, 200), (200, 1), (250, 384)])
def test_backward_unequal_lengths(Nq, Nk, causal, d):
    from oracle import attention_bwd_gqa_ref

    q, k, v, do = _qk_inputs(1, 4, 2, Nq, Nk, d, seed=7 * Nq + Nk)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward_qk(qd, kd, vd, causal=causal)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    fa.backward_qk(qd, kd, vd, o, dod, lse, causal=causal, dq=dq, dk=dk, dv=dv)
    fa.check_device_status()
    ref = attention_bwd_gqa_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), 1 / math.sqrt(d), causal)
    check_bwd(tuple(to_f64(x) for x in (dq, dk, dv)), ref, (Nq, Nk, causal, d))


def test_unequal_lengths_equal_to_square_entry_points():
    q, k, v, do = _qk_inputs(2, 4, 4, 384, 384, 128, seed=5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o1, l1 = fa.forward_qk(qd, kd, vd, causal=True)
    o2, l2 = fa.forward(qd, kd, vd, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = fa.backward_qk(qd, kd, vd, o1, dod, l1, causal=True)
    g2 = fa.backward(qd, kd, vd, o2, dod, l2, causal=True)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])  # dK, dV: one CTA each
    assert float((g1[0].float() - g2[0].float()).norm() / g2[0].float().norm()) < 1e-3


def test_fewer_queries_are_the_last_rows_of_the_square_case_on_gpu():
    # bottom-right alignment on the device: new queries against a longer key/value
    # sequence reproduce the last rows of the square causal problem
    q, k, v, _ = _qk_inputs(1, 4, 4, 1000, 1000, 128, seed=6)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o_sq, l_sq = fa.forward(qd, kd, vd, causal=True)
    o, lse = fa.forward_qk(qd[:, :, 1000 - 300 :].contiguous(), kd, vd, causal=True)
    assert max_abs(to_f64(o), to_f64(o_sq[:, :, 700:])) <= 1e-2
    assert max_abs(to_f64(lse), to_f64(l_sq[:, :, 700:])) <= 1e-4


def test_forward_permutation_equivariance_on_gpu():
    # non-causal attention commutes with permutations: permuting the queries
    # permutes the output rows (bit for bit: every row is computed on its own),
    # and permuting keys together with values leaves O and LSE unchanged up to
    # the summation order
    B, H, N, d = 1, 3, 700, 128
    q, k, v = (t.cuda() for t in make_inputs(B, H, N, d, seed=31))
    g = torch.Generator().manual_seed(5)
    perm_q = torch.randperm(N, generator=g).cuda()
    perm_k = torch.randperm(N, generator=g).cuda()
    o, lse = fa.forward(q, k, v)
    oq, lq = fa.forward(q[:, :, perm_q].contiguous(), k, v)
    assert torch.equal(oq, o[:, :, perm_q]) and torch.equal(lq, lse[:, :, perm_q])
    ok_, lk = fa.forward(q, k[:, :, perm_k].contiguous(), v[:, :, perm_k].contiguous())
    fa.check_device_status()
    assert max_abs(to_f64(ok_), to_f64(o)) <= O_MAXABS
    assert max_abs(to_f64(lk), to_f64(lse)) <= 1e-4


# ---------------------------------------------------------------- sizes at the edges


def test_many_heads_small_tiles():
    # 8192 heads of one 128-row tile: thousands of work items through the
    # forward's scheduler and 8192 backward CTAs, checked on a spread of heads
    B, H, N, d = 2, 4096, 128, 64
    q, k, v, do = (t.cuda() for t in make_inputs(B, H, N, d, seed=41, with_do=True))
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.forward(q, k, v, causal=True, out=o, lse=lse)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
    fa.backward(q, k, v, o, do, lse, causal=True, dq=dq, dk=dk, dv=dv)
    fa.check_device_status()
    for t in (o, lse, dq, dk, dv):
        assert not bool(torch.isnan(t).any())
    for b, h in [(0, 0), (0, 4095), (1, 1234), (1, 4095)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [to_f64(x[sl].cpu()) for x in (q, k, v)]
        o_ref, lse_ref = attention_fwd_ref(*args, 1 / math.sqrt(d), True)
        check_fwd(to_f64(o[sl]), to_f64(lse[sl]), o_ref, lse_ref, (b, h))
        ref = attention_bwd_ref(*args, to_f64(do[sl].cpu()), 1 / math.sqrt(d), True)
        check_bwd([to_f64(g[sl]) for g in (dq, dk, dv)], ref, (b, h))


def test_long_single_head_forward_sampled_rows():
    # one head of 131072 keys (causal): 512 query-tile pairs in one head
    from exact_tiled_attention_35_b200.inputs import sample_rows
    from oracle import attention_rows_ref

    B, H, N, d = 1, 1, 131072, 128
    q, k, v = make_inputs(B, H, N, d, seed=43)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.forward(qd, kd, vd, causal=True, out=o, lse=lse)
    fa.check_device_status()
    assert not bool(torch.isnan(o).any()) and not bool(torch.isnan(lse).any())
    rows = [sample_rows(N, 48, 43, 0)]
    o_ref, lse_ref = attention_rows_ref(to_f64(q), to_f64(k), to_f64(v), rows, 1 / math.sqrt(d), True)
    check_fwd(to_f64(o)[:, :, rows[0]], to_f64(lse)[:, :, rows[0]], o_ref, lse_ref, "N=131072")


@pytest.mark.parametrize("N", [129, 255, 257, 383])
def test_one_row_past_a_tile_boundary(N):
    # ragged tails one row either side of a tile edge, grouped heads, both passes
    from oracle import attention_bwd_gqa_ref, attention_fwd_gqa_ref

    q, do = make_inputs(1, 4, N, 128, seed=N, with_do=True)[0::3]
    k, v = make_inputs(1, 2, N, 128, seed=N + 1)[1:3]
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward_gqa(qd, kd, vd, causal=True)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    fa.backward_gqa(qd, kd, vd, o, dod, lse, causal=True, dq=dq, dk=dk, dv=dv)
    fa.check_device_status()
    args = (to_f64(q), to_f64(k), to_f64(v))
    o_ref, lse_ref = attention_fwd_gqa_ref(*args, 1 / math.sqrt(128), True)
    check_fwd(to_f64(o), to_f64(lse), o_ref, lse_ref, N)
    ref = attention_bwd_gqa_ref(*args, to_f64(do), 1 / math.sqrt(128), True)
    check_bwd([to_f64(x) for x in (dq, dk, dv)], ref, N)
