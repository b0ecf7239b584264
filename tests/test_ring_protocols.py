"""The mbarrier protocols of the 2:4 decode kernel and the grouped-scale
kernel, run on the CPU under random schedules (no GPU).

An mbarrier completes a phase when its expected arrivals have come; a wait
on parity P passes while the barrier's current phase parity differs from P.
That wait is exact only if the phase the waiter wants is the one in progress
or the one just completed: a waiter two phases behind would block on a phase
that already passed, one two phases ahead would pass early.  Each kernel
role below is the sequence of waits and arrivals its code makes (with the
same stage counts), the waits written as the phase they want; completions
of TMA copies and tensor-core commits arrive at random later steps.  The
simulation asserts the exactness condition at every step a waiter is
blocked, that no barrier gets more arrivals than a phase takes, and that no
schedule deadlocks.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0  # done = completed phases

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than a phase takes"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def run(roles, seed, max_steps=200000):
    """roles: generators of ('wait', bar, phase), ('arrive', bar), ('async', bar)."""
    rng = random.Random(seed)
    live = [[r, next(r, None)] for r in roles]
    asyncs = []  # arrivals still in flight (copies, commits)
    for _ in range(max_steps):
        live = [x for x in live if x[1] is not None]
        for _, act in live:  # every blocked waiter: the exactness condition
            if act[0] == "wait":
                bar, phase = act[1], act[2]
                assert phase <= bar.done <= phase + 1, (
                    f"a wait for phase {phase} sees {bar.done} completed phases")
        ready = [x for x in live if x[1][0] != "wait" or x[1][1].done >= x[1][2] + 1]
        if not ready and not asyncs:
            assert not live, "deadlock"
            return
        if asyncs and (not ready or rng.random() < 0.3):
            asyncs.pop(rng.randrange(len(asyncs))).arrive()
            continue
        x = rng.choice(ready)
        act = x[1]
        if act[0] == "arrive":
            act[1].arrive()
        elif act[0] == "async":
            asyncs.append(act[1])
        x[1] = next(x[0], None)
    raise AssertionError("schedule did not finish")


# ----------------------------------------------------------------- 2:4 decode kernel
def gemv24_roles(nkb, nko, S=4, SPW=4, NG=4, NI=2):
    w_full = [Bar(1) for _ in range(SPW)]
    w_empty = [Bar(4) for _ in range(SPW)]  # the four warps of a group
    op_full = [Bar(4) for _ in range(S)]
    op_empty = [Bar(1) for _ in range(S)]
    o_full, acc_full = Bar(1), Bar(NI)
    early = min(nkb, SPW)

    def producer():
        for u in range(early):          # the first units, expected before the CTA barrier
            yield ("async", w_full[u])
        if nko:
            yield ("async", o_full)
        for u in range(early, nkb):
            st = u % SPW
            yield ("wait", w_empty[st], u // SPW - 1)
            yield ("async", w_full[st])

    def group_warp(g):
        for kb in range(g, nkb, NG):
            st, ps = kb % S, kb % SPW
            if kb >= S:                 # a fresh barrier passes the first wait
                yield ("wait", op_empty[st], kb // S - 1)
            yield ("wait", w_full[ps], kb // SPW)
            yield ("arrive", w_empty[ps])
            yield ("arrive", op_full[st])
        if g == 0:                      # the epilogue
            yield ("wait", acc_full, 0)

    def issuer(i):
        if i == 0 and nko:
            yield ("wait", o_full, 0)
        for kb in range(i, nkb, NI):
            st = kb % S
            yield ("wait", op_full[st], kb // S)
            yield ("async", op_empty[st])   # tcgen05.commit
        yield ("async", acc_full)

    return ([producer()] + [group_warp(g) for g in range(NG) for _ in range(4)] +
            [issuer(i) for i in range(NI)])


@pytest.mark.parametrize("nkb", [0, 1, 2, 3, 4, 5, 7, 8, 16, 31, 33])
@pytest.mark.parametrize("nko", [0, 1])
def test_gemv24_protocol(nkb, nko):
    for seed in range(40):
        run(gemv24_roles(nkb, nko), seed)


# ----------------------------------------------------------------- grouped-scale kernel
def grouped_roles(nkb_i, nkb_o, SP=4, SU=4, NT=4, NE=8, NACC=4):
    pk_full = [Bar(1) for _ in range(SP)]
    pk_empty = [Bar(NT) for _ in range(SP)]
    op_full = [Bar(NT) for _ in range(SU)]
    op_empty = [Bar(1) for _ in range(SU)]
    acc_full = [Bar(1) for _ in range(NACC)]
    acc_empty = [Bar(NE) for _ in range(NACC)]

    def producer():
        for kb in range(nkb_i):
            s = kb % SP
            if kb >= SP:
                yield ("wait", pk_empty[s], kb // SP - 1)
            yield ("async", pk_full[s])

    def unpack_warp(t):
        for kb in range(nkb_i + nkb_o):
            sp, su = kb % SP, kb % SU
            if kb >= nkb_i:             # outlier k-block: by TMA, one warp's copy
                if kb >= SU:
                    yield ("wait", op_empty[su], kb // SU - 1)
                yield ("async" if t == 0 else "arrive", op_full[su])
                continue
            yield ("wait", pk_full[sp], kb // SP)
            if kb >= SU:
                yield ("wait", op_empty[su], kb // SU - 1)
            yield ("arrive", pk_empty[sp])
            yield ("arrive", op_full[su])

    def issuer():
        for kb in range(nkb_i):
            s, b = kb % SU, kb % NACC
            if kb >= NACC:
                yield ("wait", acc_empty[b], kb // NACC - 1)
            yield ("wait", op_full[s], kb // SU)
            yield ("async", op_empty[s])
            yield ("async", acc_full[b])
        if nkb_o:
            b = nkb_i % NACC
            if nkb_i >= NACC:
                yield ("wait", acc_empty[b], nkb_i // NACC - 1)
            for ko in range(nkb_o):
                kb = nkb_i + ko
                s = kb % SU
                yield ("wait", op_full[s], kb // SU)
                yield ("async", op_empty[s])
            yield ("async", acc_full[b])

    def drain_warp():
        for g in range(nkb_i):
            b = g % NACC
            yield ("wait", acc_full[b], g // NACC)
            yield ("arrive", acc_empty[b])
        if nkb_o:
            yield ("wait", acc_full[nkb_i % NACC], nkb_i // NACC)

    return ([producer()] + [unpack_warp(t) for t in range(NT)] + [issuer()] +
            [drain_warp() for _ in range(NE)])


@pytest.mark.parametrize("nkb_i", [1, 2, 3, 4, 5, 8, 9, 63, 64])
@pytest.mark.parametrize("nkb_o", [0, 1, 2])
def test_grouped_protocol(nkb_i, nkb_o):
    for seed in range(25):
        run(grouped_roles(nkb_i, nkb_o), seed)


def test_checker_catches_a_ring_filled_out_of_order():
    """The checker itself: a producer that runs two phases ahead (no wait on
    the empty barrier) trips the exactness assertion."""
    full, empty = Bar(1), Bar(1)

    def producer():
        for u in range(6):
            yield ("arrive", full)

    def consumer():
        for u in range(6):
            yield ("wait", full, u)
            yield ("arrive", empty)

    with pytest.raises(AssertionError):
        for seed in range(20):
            run([producer(), consumer()], seed)
