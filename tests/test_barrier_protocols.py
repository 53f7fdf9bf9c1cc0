"""Deadlock and phase-aliasing checks of the kernels' barrier protocols, on the CPU.

The sm_100a kernels hand work between warp roles through mbarriers that are
waited on by phase parity.  Two failure modes cannot be seen by a parity test
on a lucky schedule: a cycle of waits (a hang, which the bounded waits turn
into a timeout) and a barrier that completes twice before its waiter looks,
so that the waiter's parity matches again and it misses the phase.  A device
sanitizer is not available here, so these tests model each kernel's roles as
sequential programs of barrier operations -- in the order the kernel issues
them, with the counts it initialises them with -- and run them under many
random interleavings:

* every wait names the phase index it means, and the model asserts, when the
  wait is satisfied, that exactly that phase is the latest completed one;
* a state in which no role can move while some have not finished is a
  deadlock.

The models mirror csrc/fa_fwd_sm100.cu (producer warp, MMA-issuing thread,
two softmax groups; item ring, K/V ring, Q buffers) and the persistent
backward main kernel of csrc/fa_bwd_sm100.cu (producer warp, MMA-issuing
thread, compute warps, dQ reduce warps; item ring, K/V buffers, Q stages,
single dO buffer, dQ sharing dP's tensor-memory columns or not).  A change to
either kernel's barrier protocol must be made here too.  One of these models
found the phase-aliasing bug described in the design notes (an early-issue
variant of the forward that re-waited a Q buffer whose next load had already
landed).
"""

from __future__ import annotations

import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0  # done = completed phases


class Model:
    """Roles are generators yielding ("wait", bar, phase_index) or ("arrive", bar, n)."""

    def __init__(self):
        self.bars, self.shared = {}, {}

    def bar(self, name, count=1):
        if name not in self.bars:
            self.bars[name] = _Bar(count)
        return self.bars[name]

    @staticmethod
    def wait(name, index):
        return ("wait", name, index)

    @staticmethod
    def arrive(name, n=1):
        return ("arrive", name, n)

    def run(self, roles, rng):
        cur = {k: None for k in roles}
        done, blocked = set(), set()
        while len(done) < len(roles):
            live = [k for k in roles if k not in done]
            ready = [k for k in live if k not in blocked]
            if not ready:
                return {k: cur[k] for k in live}  # deadlock
            k = rng.choice(ready)
            op = cur[k]
            if op is None:
                try:
                    op = next(roles[k])
                except StopIteration:
                    done.add(k)
                    continue
                cur[k] = op
            b = self.bar(op[1])
            if op[0] == "arrive":
                b.pending += op[2]
                while b.pending >= b.count:
                    b.pending -= b.count
                    b.done += 1
                cur[k] = None
                blocked.clear()
                continue
            # try_wait.parity(P) passes while the current phase's parity differs from P
            if (b.done & 1) != (op[2] & 1):
                assert b.done == op[2] + 1, (k, op, b.done, "phase overtaken")
                cur[k] = None
            else:
                blocked.add(k)
        return None


# ---------------------------------------------------------------- forward


def forward_roles(m, items, nslot):
    """items: per work item (n_0, n_1), the key tiles each of its two query tiles sees."""
    W, A = m.wait, m.arrive
    for t in range(2):
        for b in ("q_full", "q_empty", "s_full", "o_full"):
            m.bar(f"{b}{t}")
        m.bar(f"p_lo{t}", 128)
        m.bar(f"p_hi{t}", 128)
    for s in range(2):
        m.bar(f"it_empty{s}", 9)  # the MMA issuer and the 8 softmax warps

    def producer():
        qcnt, gseq = [0, 0], 0
        for r in range(len(items) + 1):
            s = r % 2
            if r >= 2:
                yield W(f"it_empty{s}", r // 2 - 1)
            m.shared[f"item{s}"] = items[r] if r < len(items) else None
            yield A(f"it_full{s}")
            if r == len(items):
                return
            n = items[r]
            for t in range(2):
                if n[t] == 0:
                    continue
                if qcnt[t] > 0:
                    yield W(f"q_empty{t}", qcnt[t] - 1)
                yield A(f"q_full{t}")
                qcnt[t] += 1
            for s2 in range(2 * max(n)):
                seq = gseq + s2
                slot, rnd = seq % nslot, seq // nslot
                if rnd > 0:
                    yield W(f"kv_empty{slot}", rnd - 1)
                yield A(f"kv_full{slot}")
            gseq += 2 * max(n)

    def mma():
        kslot = 0
        fills = [0] * nslot  # per ring slot: how many times it has been filled and consumed
        gt, qcnt = [0, 0], [0, 0]
        for r in range(len(items) + 1):
            s = r % 2
            yield W(f"it_full{s}", r // 2)
            w = m.shared[f"item{s}"]
            yield A(f"it_empty{s}")
            if w is None:
                return
            nmax = max(w)
            if nmax == 0:
                continue
            for t in range(2):
                if w[t] > 0:
                    yield W(f"q_full{t}", qcnt[t])
            yield W(f"kv_full{kslot}", fills[kslot])
            for t in range(2):
                if w[t] > 0:
                    yield A(f"s_full{t}")
                    if w[t] == 1:
                        yield A(f"q_empty{t}")
            yield A(f"kv_empty{kslot}")
            for j in range(nmax):
                vslot = (kslot + 1) % nslot
                nslot_ = (vslot + 1) % nslot
                yield W(f"kv_full{vslot}", fills[vslot])
                k_next = False
                for t in range(2):
                    if j >= w[t]:
                        continue
                    yield W(f"p_lo{t}", gt[t] + j)
                    yield W(f"p_hi{t}", gt[t] + j)
                    if j + 1 < w[t]:
                        if not k_next:
                            yield W(f"kv_full{nslot_}", fills[nslot_])
                            k_next = True
                        yield A(f"s_full{t}")
                        if j + 2 == w[t]:
                            yield A(f"q_empty{t}")
                    else:
                        yield A(f"o_full{t}")
                yield A(f"kv_empty{vslot}")
                fills[kslot] += 1
                fills[vslot] += 1
                if k_next:
                    yield A(f"kv_empty{nslot_}")
                kslot = nslot_
            for t in range(2):
                gt[t] += w[t]
                qcnt[t] += w[t] > 0

    def softmax(t):
        gtile, icnt = 0, 0
        for r in range(len(items) + 1):
            s = r % 2
            yield W(f"it_full{s}", r // 2)
            w = m.shared[f"item{s}"]
            yield A(f"it_empty{s}", 4)
            if w is None:
                return
            n = w[t]
            if n == 0:
                continue
            for j in range(n):
                yield W(f"s_full{t}", gtile + j)
                yield A(f"p_lo{t}", 64)   # stands for the group's 128 arrivals in two halves
                yield A(f"p_lo{t}", 64)
                yield A(f"p_hi{t}", 128)
            yield W(f"o_full{t}", icnt)
            gtile += n
            icnt += 1

    return {"producer": producer(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1)}


def _forward_items(rng):
    out = []
    for _ in range(rng.randint(1, 7)):
        u, p = rng.random(), rng.randint(0, 6)
        if u < 0.45:
            out.append((2 * p + 1, 2 * p + 2))  # a causal query-tile pair
        elif u < 0.7:
            out.append((p + 1, p + 1))          # non-causal
        elif u < 0.8:
            out.append((0, p + 1))              # first tile fully masked (more queries than keys)
        elif u < 0.9:
            out.append((1, 1))
        else:
            out.append((0, 0))                  # nothing visible
    return out


@pytest.mark.parametrize("nslot", [4, 5, 10, 12, 16])
def test_forward_protocol_has_no_deadlock_or_overtaken_phase(nslot):
    rng = random.Random(nslot)
    for _ in range(600):
        items = _forward_items(rng)
        m = Model()
        stuck = m.run(forward_roles(m, items, nslot), rng)
        assert stuck is None, (items, stuck)


# ---------------------------------------------------------------- backward


def backward_roles(m, items, nst, dq_shared, with_dq=True):
    """items: per work item the number of query tiles it loops over."""
    W, A = m.wait, m.arrive
    readers = 1 + 8 + (4 if with_dq else 0)
    for s in range(2):
        m.bar(f"it_empty{s}", readers)
    m.bar("p_full", 256)
    m.bar("ds_full", 256)
    m.bar("dq_empty", 128)

    def producer():
        g = dog = nkv = 0
        for r in range(len(items) + 1):
            s = r % 2
            if r >= 2:
                yield W(f"it_empty{s}", r // 2 - 1)
            m.shared[f"item{s}"] = items[r] if r < len(items) else None
            yield A(f"it_full{s}")
            if r == len(items):
                return

            def load_tile():
                nonlocal g, dog
                st, rnd = g % nst, g // nst
                if rnd > 0:
                    yield W(f"q_empty{st}", rnd - 1)
                yield A(f"q_full{st}")
                g += 1
                if dog > 0:
                    yield W("do_empty", dog - 1)
                yield A("do_full")
                dog += 1

            yield from load_tile()
            if r > 0:
                yield W("kv_empty", r - 1)
            yield A("kv_full")
            nkv += 1
            for _ in range(1, items[r]):
                yield from load_tile()

    def mma():
        g = 0
        for r in range(len(items) + 1):
            s = r % 2
            yield W(f"it_full{s}", r // 2)
            niter = m.shared[f"item{s}"]
            yield A(f"it_empty{s}")
            if niter is None:
                return
            yield W("kv_full", r)
            yield W(f"q_full{g % nst}", g // nst)
            yield A("s_full")
            if with_dq and dq_shared and g > 0:
                yield W("dq_empty", g - 1)
            yield W("do_full", g)
            yield A("dp_full")
            for it in range(niter):
                st, more = g % nst, it + 1 < niter
                yield W("p_full", g)
                yield A("do_empty")                       # dV(g) read dO(g)
                if not with_dq and not more:
                    yield A("kv_empty")
                if more:
                    yield W(f"q_full{(g + 1) % nst}", (g + 1) // nst)
                    yield A("s_full")                     # S(g+1)
                yield W("ds_full", g)
                yield A(f"q_empty{st}")                   # dK(g) read Q(g)
                if with_dq:
                    if not dq_shared and g > 0:
                        yield W("dq_empty", g - 1)
                    yield A("dq_full")
                    if not more:
                        yield A("kv_empty")
                yield A("ds_free")
                if not more:
                    yield A("acc_full")
                if more:
                    if with_dq and dq_shared:
                        yield W("dq_empty", g)
                    yield W("do_full", g + 1)
                    yield A("dp_full")                    # dP(g+1)
                g += 1

    def compute():
        g = 0
        for r in range(len(items) + 1):
            s = r % 2
            yield W(f"it_full{s}", r // 2)
            niter = m.shared[f"item{s}"]
            yield A(f"it_empty{s}", 8)
            if niter is None:
                return
            for it in range(niter):
                yield W(f"q_full{g % nst}", g // nst)
                yield W("s_full", g)
                yield A("p_full", 256)
                yield W("dp_full", g)
                if g > 0:
                    yield W("ds_free", g - 1)
                yield A("ds_full", 256)
                g += 1
            yield W("acc_full", r)

    def reduce():
        g = 0
        for r in range(len(items) + 1):
            s = r % 2
            yield W(f"it_full{s}", r // 2)
            niter = m.shared[f"item{s}"]
            yield A(f"it_empty{s}", 4)
            if niter is None:
                return
            for it in range(niter):
                yield W("dq_full", g)
                yield A("dq_empty", 128)
                g += 1

    roles = {"producer": producer(), "mma": mma(), "compute": compute()}
    if with_dq:
        roles["reduce"] = reduce()
    return roles


@pytest.mark.parametrize("nst,dq_shared,with_dq", [(2, True, True), (3, False, True), (2, True, False),
                                                   (3, False, False)])
def test_backward_protocol_has_no_deadlock_or_overtaken_phase(nst, dq_shared, with_dq):
    rng = random.Random(10 * nst + dq_shared + 2 * with_dq)
    for _ in range(600):
        items = [rng.randint(1, 6) for _ in range(rng.randint(1, 6))]
        m = Model()
        stuck = m.run(backward_roles(m, items, nst, dq_shared, with_dq), rng)
        assert stuck is None, (items, stuck)


def test_model_catches_a_re_wait_on_a_phase_that_moved_on():
    # The checker itself, on the shape of the bug it found: a consumer that
    # waits twice for phase 0 of a barrier whose producer may complete it again
    # in between is reported, either as a deadlock (the parity matches again
    # and the wait never returns) or as an overtaken phase.
    found = 0
    rng = random.Random(3)
    for _ in range(200):
        m = Model()

        def producer():
            for _ in range(3):
                yield Model.arrive("b")

        def consumer():
            yield Model.wait("b", 0)
            yield Model.wait("b", 0)  # the re-wait

        try:
            found += m.run({"p": producer(), "c": consumer()}, rng) is not None
        except AssertionError as e:
            assert "phase overtaken" in str(e)
            found += 1
    assert found > 0
