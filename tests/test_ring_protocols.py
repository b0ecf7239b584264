"""The mbarrier and named-barrier protocols of the kernels (the CTA-pair
kernel, the persistent warp-specialised CTA-pair kernel, the dense and 2:4
decode kernels, the grouped-scale kernel, the quantiser's team ring), run on
the CPU under random schedules (no GPU).

An mbarrier completes a phase when its expected arrivals have come; a wait
on parity P passes while the barrier's current phase parity differs from P.
That wait is exact only if the phase the waiter wants is the one in progress
or the one just completed: a waiter two phases behind would block on a phase
that already passed, one two phases ahead would pass early.

Each kernel role below is the sequence of waits, arrivals and buffer
accesses its code makes (with the kernel's stage counts), the waits written
as the phase they want.  Completions of TMA copies and tensor-core commits
arrive at random later steps.  Buffers are owned while in use: an operand
stage by the MMA from its full-wait until its commit lands, a staging slot
by its readers from their full-wait until their empty-arrival, an
accumulator by the drain while it reads it.  The simulation asserts:

* the exactness condition, at every step a waiter is blocked;
* that no barrier gets more arrivals than a phase takes;
* that nothing writes a buffer while another role still owns it (a TMA copy
  into a staging slot, unpacked operands into a stage, an MMA into an
  accumulator);
* that no schedule deadlocks.
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


class Sync:
    """A named barrier (bar.sync) over n roles: each waits until all n have
    arrived at the same generation."""

    def __init__(self, n):
        self.n, self.arrived, self.gen = n, 0, 0

    def arrive(self):
        self.arrived += 1
        my = self.gen
        if self.arrived == self.n:
            self.arrived, self.gen = 0, self.gen + 1
        return my


class Buf:
    """A buffer and how many roles own it right now."""

    def __init__(self, name):
        self.name, self.owners = name, 0


def run(roles, seed, max_steps=400000):
    """roles: generators of ('wait', bar, phase), ('arrive', bar),
    ('async', bar[, buf released when it lands]), ('own', buf),
    ('free', buf), ('write', buf), ('sync', named barrier)."""
    rng = random.Random(seed)
    live = [[r, next(r, None)] for r in roles]
    for x in live:  # a role at a named barrier has arrived there
        if x[1] is not None and x[1][0] == "sync":
            x[1] = ("synced", x[1][1], x[1][1].arrive())
    asyncs = []  # (barrier, buffer released when the arrival lands) still in flight
    for _ in range(max_steps):
        live = [x for x in live if x[1] is not None]
        for _, act in live:  # every blocked waiter: the exactness condition
            if act[0] == "wait":
                bar, phase = act[1], act[2]
                assert phase <= bar.done <= phase + 1, (
                    f"a wait for phase {phase} sees {bar.done} completed phases")
        ready = [x for x in live
                 if (x[1][0] != "wait" or x[1][1].done >= x[1][2] + 1) and
                 (x[1][0] != "synced" or x[1][1].gen > x[1][2])]
        if not ready and not asyncs:
            assert not live, "deadlock"
            return
        if asyncs and (not ready or rng.random() < 0.3):
            bar, buf = asyncs.pop(rng.randrange(len(asyncs)))
            if buf is not None:
                buf.owners -= 1
            bar.arrive()
            continue
        x = rng.choice(ready)
        act = x[1]
        if act[0] == "arrive":
            act[1].arrive()
        elif act[0] == "async":
            asyncs.append((act[1], act[2] if len(act) > 2 else None))
        elif act[0] == "own":
            act[1].owners += 1
        elif act[0] == "free":
            act[1].owners -= 1
        elif act[0] == "write":
            assert act[1].owners == 0, f"{act[1].name} written while in use"
        x[1] = next(x[0], None)
        if x[1] is not None and x[1][0] == "sync":
            x[1] = ("synced", x[1][1], x[1][1].arrive())
    raise AssertionError("schedule did not finish")


# ----------------------------------------------------------------- decode kernels (dense and 2:4)
def decode_roles(nkb, nko, S=4, SPW=4, NG=4, NI=2):
    """Producer, NG groups of four unpack warps (group g: k-blocks g, g + NG,
    ...), NI MMA issuers (issuer i: k-blocks i, i + NI, ...)."""
    w_full = [Bar(1) for _ in range(SPW)]
    w_empty = [Bar(4) for _ in range(SPW)]  # the four warps of a group
    op_full = [Bar(4) for _ in range(S)]
    op_empty = [Bar(1) for _ in range(S)]
    o_full, acc_full = Bar(1), Bar(NI)
    slot = [Buf(f"staging slot {i}") for i in range(SPW)]
    stage = [Buf(f"operand stage {i}") for i in range(S)]
    early = min(nkb, SPW)

    def producer():
        for u in range(early):          # the first units, expected before the CTA barrier
            yield ("write", slot[u])
            yield ("async", w_full[u])
        if nko:
            yield ("async", o_full)
        for u in range(early, nkb):
            st = u % SPW
            yield ("wait", w_empty[st], u // SPW - 1)
            yield ("write", slot[st])
            yield ("async", w_full[st])

    def group_warp(g):
        for kb in range(g, nkb, NG):
            st, ps = kb % S, kb % SPW
            if kb >= S:                 # a fresh barrier passes the first wait
                yield ("wait", op_empty[st], kb // S - 1)
            yield ("wait", w_full[ps], kb // SPW)
            yield ("own", slot[ps])     # the packed bytes into registers
            yield ("free", slot[ps])
            yield ("arrive", w_empty[ps])
            yield ("write", stage[st])  # unpacked operands (and pairs) into the stage
            yield ("arrive", op_full[st])
        if g == 0:                      # the epilogue
            yield ("wait", acc_full, 0)

    def issuer(i):
        if i == 0 and nko:
            yield ("wait", o_full, 0)
        for kb in range(i, nkb, NI):
            st = kb % S
            yield ("wait", op_full[st], kb // S)
            yield ("own", stage[st])
            yield ("async", op_empty[st], stage[st])   # tcgen05.commit
        yield ("async", acc_full)

    return ([producer()] + [group_warp(g) for g in range(NG) for _ in range(4)] +
            [issuer(i) for i in range(NI)])


@pytest.mark.parametrize("nkb", [0, 1, 2, 3, 4, 5, 7, 8, 16, 31, 33])
@pytest.mark.parametrize("nko", [0, 1])
def test_sparse_decode_protocol(nkb, nko):
    """The 2:4 decode kernel: 4 operand stages, 4 staging units."""
    for seed in range(40):
        run(decode_roles(nkb, nko), seed)


@pytest.mark.parametrize("nkb", [1, 4, 8, 9, 10, 11, 31, 64])
@pytest.mark.parametrize("nko", [0, 1])
def test_dense_decode_protocol(nkb, nko):
    """The dense decode kernel: 8 operand stages, 10 staging units."""
    for seed in range(30):
        run(decode_roles(nkb, nko, S=8, SPW=10), seed)


# ----------------------------------------------------------------- CTA-pair kernel
def pair_roles(nkb_i, nkb_o, S=4, SP=4, NA=4, NB=8, b_waits_outliers=True):
    """Two CTAs; the leader's operand-full barriers take the arrivals of
    every A and B warp of both CTAs (remote arrivals); each commit arrives on
    both CTAs' operand-empty barriers; each CTA has its own staging ring.
    Outlier k-blocks take two staging units (Wo rows, then Xo rows)."""
    nkb = nkb_i + nkb_o
    nunits = nkb_i + 2 * nkb_o
    op_full = [Bar(2 * (NA + NB)) for _ in range(S)]            # the leader's
    op_empty = [[Bar(1) for _ in range(S)] for _ in range(2)]   # per CTA
    pk_full = [[Bar(1) for _ in range(SP)] for _ in range(2)]
    pk_empty = [[Bar(NB) for _ in range(SP)] for _ in range(2)]
    acc_full = [Bar(1), Bar(1)]
    drain = Bar(1)
    slot = [[Buf(f"CTA {c} staging slot {i}") for i in range(SP)] for c in range(2)]
    stage = [[Buf(f"CTA {c} operand stage {i}") for i in range(S)] for c in range(2)]

    def issuer():
        for kb in range(nkb):
            if kb == nkb_i and nkb_i:   # the outlier sums reuse the A-stage columns
                yield ("async", drain)
                yield ("wait", drain, 0)
            st = kb % S
            yield ("wait", op_full[st], kb // S)
            for c in range(2):
                yield ("own", stage[c][st])
            for c in range(2):          # commit, multicast to both CTAs
                yield ("async", op_empty[c][st], stage[c][st])
        yield ("async", acc_full[0])
        yield ("async", acc_full[1])

    def producer(c):
        for u in range(nunits):
            st = u % SP
            if u >= SP:
                yield ("wait", pk_empty[c][st], u // SP - 1)
            yield ("write", slot[c][st])
            yield ("async", pk_full[c][st])

    def a_warp(c):
        for kb in range(nkb):
            st = kb % S
            if kb >= S:
                yield ("wait", op_empty[c][st], kb // S - 1)
            if kb < nkb_i:
                yield ("write", stage[c][st])   # its rows into the tensor-memory stage
            yield ("arrive", op_full[st])
        yield ("wait", acc_full[c], 0)

    def b_warp(c):
        u = 0
        for kb in range(nkb):
            st = kb % S
            if kb >= S and (b_waits_outliers or kb < nkb_i):
                yield ("wait", op_empty[c][st], kb // S - 1)
            for _ in range(1 if kb < nkb_i else 2):
                ps = u % SP
                yield ("wait", pk_full[c][ps], u // SP)
                yield ("own", slot[c][ps])
                yield ("write", stage[c][st])
                yield ("free", slot[c][ps])
                yield ("arrive", pk_empty[c][ps])
                u += 1
            yield ("arrive", op_full[st])
        yield ("wait", acc_full[c], 0)

    roles = [issuer()]
    for c in range(2):
        roles += [producer(c)] + [a_warp(c) for _ in range(NA)] + [b_warp(c) for _ in range(NB)]
    return roles


@pytest.mark.parametrize("nkb_i", [0, 1, 3, 4, 5, 8, 31, 64])
@pytest.mark.parametrize("nkb_o", [0, 1, 2])
def test_pair_protocol(nkb_i, nkb_o):
    if nkb_i + nkb_o == 0:
        pytest.skip("no k-blocks")
    for seed in range(15):
        run(pair_roles(nkb_i, nkb_o), seed)


# ----------------------------------------------------------------- grouped-scale kernel
def grouped_roles(nkb_i, nkb_o, SP=4, SU=4, NT=4, NE=8, NACC=4, drain_phase_div=None):
    pk_full = [Bar(1) for _ in range(SP)]
    pk_empty = [Bar(NT) for _ in range(SP)]
    op_full = [Bar(NT) for _ in range(SU)]
    op_empty = [Bar(1) for _ in range(SU)]
    acc_full = [Bar(1) for _ in range(NACC)]
    acc_empty = [Bar(NE) for _ in range(NACC)]
    slot = [Buf(f"staging slot {i}") for i in range(SP)]
    stage = [Buf(f"operand stage {i}") for i in range(SU)]
    acc = [Buf(f"accumulator {i}") for i in range(NACC)]
    div = drain_phase_div or NACC

    def producer():
        for kb in range(nkb_i):
            s = kb % SP
            if kb >= SP:
                yield ("wait", pk_empty[s], kb // SP - 1)
            yield ("write", slot[s])
            yield ("async", pk_full[s])

    def unpack_warp(t):
        for kb in range(nkb_i + nkb_o):
            sp, su = kb % SP, kb % SU
            if kb >= nkb_i:             # outlier k-block: by TMA, one warp's copy
                if kb >= SU:
                    yield ("wait", op_empty[su], kb // SU - 1)
                if t == 0:
                    yield ("write", stage[su])
                yield ("async" if t == 0 else "arrive", op_full[su])
                continue
            yield ("wait", pk_full[sp], kb // SP)
            if kb >= SU:
                yield ("wait", op_empty[su], kb // SU - 1)
            yield ("own", slot[sp])
            yield ("write", stage[su])
            yield ("free", slot[sp])
            yield ("arrive", pk_empty[sp])
            yield ("arrive", op_full[su])

    def issuer():
        for kb in range(nkb_i):
            s, b = kb % SU, kb % NACC
            if kb >= NACC:
                yield ("wait", acc_empty[b], kb // NACC - 1)
            yield ("wait", op_full[s], kb // SU)
            yield ("write", acc[b])     # this group's sums overwrite the buffer
            yield ("own", stage[s])
            yield ("async", op_empty[s], stage[s])
            yield ("async", acc_full[b])
        if nkb_o:
            b = nkb_i % NACC
            if nkb_i >= NACC:
                yield ("wait", acc_empty[b], nkb_i // NACC - 1)
            yield ("write", acc[b])
            for ko in range(nkb_o):
                kb = nkb_i + ko
                s = kb % SU
                yield ("wait", op_full[s], kb // SU)
                yield ("own", stage[s])
                yield ("async", op_empty[s], stage[s])
            yield ("async", acc_full[b])

    def drain_warp():
        for g in range(nkb_i):
            b = g % NACC
            yield ("wait", acc_full[b], g // div)
            yield ("own", acc[b])
            yield ("free", acc[b])
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


# ----------------------------------------------------------------- quantiser team
def quantizer_roles(rows, NR, W=4, per_token=True, int8_out=False, norm=False):
    """One team of W warps (warp 0's lane 0 leads) over `rows` rows, with NR
    row slots: the leader waits for a row's copy, a named barrier hands the
    row to the team (and ends every warp's use of the previous row's slot,
    which the leader then refills with the row a ring ahead); the reductions
    go through shared slots written by each warp's lane 0 before a named
    barrier and read by all after it: per token, the absmax (and, with the
    norm, the sum of squares) in slot j & 1, the INT8 outliers' absmax in
    slot (j & 1) ^ 1; per group with the norm, the sum of squares in slot
    j & 1 behind its own barrier."""
    row_full = [Bar(1) for _ in range(NR)]
    slot = [Buf(f"row slot {i}") for i in range(NR)]
    red = [Buf(f"reduction slot {i}") for i in range(2)]
    red_ss = [Buf(f"sum-of-squares slot {i}") for i in range(2)]
    team = Sync(W)

    def warp(w):
        if w == 0:
            for j in range(min(NR, rows)):   # the first rows, one per slot
                yield ("write", slot[j])
                yield ("async", row_full[j])
        for j in range(rows):
            if w == 0:
                yield ("wait", row_full[j % NR], j // NR)
            yield ("sync", team)             # the row is the team's; row j-1's slot is free
            if w == 0 and j > 0 and j - 1 + NR < rows:
                yield ("write", slot[(j - 1) % NR])
                yield ("async", row_full[(j - 1) % NR])
            yield ("own", slot[j % NR])      # gather (and sum of squares)
            if norm and not per_token:       # grouped: the sum of squares' own barrier
                yield ("write", red_ss[j & 1])
                yield ("sync", team)
                yield ("own", red_ss[j & 1])
                yield ("free", red_ss[j & 1])
            if per_token:
                yield ("write", red[j & 1])
                if norm:
                    yield ("write", red_ss[j & 1])
                yield ("sync", team)
                yield ("own", red[j & 1])
                yield ("free", red[j & 1])
                if norm:
                    yield ("own", red_ss[j & 1])
                    yield ("free", red_ss[j & 1])
            if int8_out:                     # the outlier block's absmax, the other slot
                yield ("write", red[(j & 1) ^ 1])
                yield ("sync", team)
                yield ("own", red[(j & 1) ^ 1])
                yield ("free", red[(j & 1) ^ 1])
            yield ("free", slot[j % NR])     # codes and outliers written from registers

    return [warp(w) for w in range(W)]


@pytest.mark.parametrize("NR", [2, 3, 4])
@pytest.mark.parametrize("mode", ["token", "token-int8", "group", "token-norm",
                                  "token-norm-int8", "group-norm", "group-norm-int8"])
def test_quantizer_team_protocol(NR, mode):
    for rows in (1, 2, 3, 5, 9):
        for seed in range(20):
            run(quantizer_roles(rows, NR, per_token=mode.startswith("token"),
                                int8_out=mode.endswith("int8"), norm="norm" in mode), seed)


# ----------------------------------------------------------------- the checker itself
# ----------------------------------------------------------------- persistent CTA-pair kernel
def unit_order(ntp, nkb_i, nkb_o, out_delay):
    """The persistent kernel's work units in issue order: (tile, outlier, k).
    Tile j's INT4 k-blocks, tile j-1's outlier units after the first
    out_delay of them, the last tile's outlier units at the end."""
    units = []
    for j in range(ntp):
        for k in range(nkb_i):
            if j > 0 and k == out_delay:
                units += [(j - 1, True, o) for o in range(nkb_o)]
            units.append((j, False, k))
        if j > 0 and nkb_i <= out_delay:
            units += [(j - 1, True, o) for o in range(nkb_o)]
    if ntp > 0:
        units += [(ntp - 1, True, o) for o in range(nkb_o)]
    return units


def persistent_roles(ntp, nkb_i, nkb_o, x4=False, S=5, SP=6, NG=3, GW=3, NE=4, out_delay=6,
                     last_rescale_count=None):
    """Two CTAs of 16 warps: the leader's MMA issuer, per CTA one operand
    TMA producer, one packed-staging producer, NG unpack groups of GW warps
    (group g takes units g, g + NG, ...) and NE epilogue warps.  The leader's
    operand-full barriers take the arrivals of the unit's group in both CTAs;
    commits reach both CTAs.  Tiles alternate between two accumulators; the
    epilogue rescales tile j-1 (FP16 outliers) while tile j's k-blocks run;
    the last tile's two epilogue passes are shared by every warp after a
    CTA-wide barrier, with its own arrival count on the rescale barrier."""
    units = unit_order(ntp, nkb_i, nkb_o, out_delay)
    op_full = [Bar(2 * GW) for _ in range(S)]
    op_empty = [[Bar(1) for _ in range(S)] for _ in range(2)]
    x_full = [[Bar(1) for _ in range(S)] for _ in range(2)]
    pk_full = [[Bar(1) for _ in range(SP)] for _ in range(2)]
    pk_empty = [[Bar(GW) for _ in range(SP)] for _ in range(2)]
    acc_empty = [Bar(2 * NE) for _ in range(2)]
    rescaled = [Bar(2 * NE) for _ in range(2)]
    int_done = [[Bar(1) for _ in range(2)] for _ in range(2)]
    acc_full = [[Bar(1) for _ in range(2)] for _ in range(2)]
    rescaled_last = Bar(last_rescale_count or 2 * 16)
    mma_done = Bar(1)
    epi = [Sync(NE) for _ in range(2)]
    everyone = [Sync(16) for _ in range(2)]
    stage = [[Buf(f"CTA {c} operand stage {i}") for i in range(S)] for c in range(2)]
    slot = [[Buf(f"CTA {c} staging slot {i}") for i in range(SP)] for c in range(2)]
    acc = [[Buf(f"CTA {c} accumulator {b}") for b in range(2)] for c in range(2)]
    last, bl = ntp - 1, (ntp - 1) & 1
    ring = {"u": 0}

    def issue(u, b):
        st = u % S
        yield ("wait", op_full[st], u // S)
        for c in range(2):
            yield ("own", stage[c][st])
        for c in range(2):
            yield ("write", acc[c][b])
        for c in range(2):
            yield ("async", op_empty[c][st], stage[c][st])

    def issuer():
        u = 0
        for j in range(ntp):
            b = j & 1
            if j >= 2:
                yield ("wait", acc_empty[b], (j >> 1) - 1)
            k1 = min(out_delay, nkb_i) if j > 0 else nkb_i
            for _ in range(k1):
                yield from issue(u, b)
                u += 1
            if j > 0 and nkb_o > 0:
                bo = (j - 1) & 1
                yield ("wait", rescaled[bo], (j - 1) >> 1)
                for _ in range(nkb_o):
                    yield from issue(u, bo)
                    u += 1
                for c in range(2):
                    yield ("async", acc_full[c][bo])
            for _ in range(nkb_i - k1):
                yield from issue(u, b)
                u += 1
            for c in range(2):
                yield ("async", (int_done if nkb_o > 0 else acc_full)[c][b])
        ring["u"] = u

    def last_tile(c, w):
        """Every warp's share of the last tile (warp w of CTA c)."""
        yield ("sync", everyone[c])
        if nkb_o > 0:
            yield ("wait", int_done[c][bl], last >> 1)
            yield ("own", acc[c][bl])
            yield ("free", acc[c][bl])
            yield ("arrive", rescaled_last)
            if c == 0 and w == 0:
                yield ("wait", rescaled_last, 0)
                u = ring["u"]
                for _ in range(nkb_o):
                    yield from issue(u, bl)
                    u += 1
                for cc in range(2):
                    yield ("async", acc_full[cc][bl])
        yield ("wait", acc_full[c][bl], last >> 1)
        yield ("own", acc[c][bl])
        yield ("free", acc[c][bl])
        if c == 0 and w == 0:
            yield ("async", mma_done)
            yield ("wait", mma_done, 0)

    def mma_warp(c):
        if c == 0:
            yield from issuer()
        yield from last_tile(c, 0)

    def xprod(c):
        for u, (j, outl, k) in enumerate(units):
            st = u % S
            if u >= S:
                yield ("wait", op_empty[c][st], u // S - 1)
            if outl or not x4:
                yield ("write", stage[c][st])
                yield ("async", x_full[c][st])
            else:
                yield ("arrive", x_full[c][st])
        yield from last_tile(c, 4)

    def pprod(c):
        q = 0
        for (j, outl, k) in units:
            if outl:
                continue
            ps = q % SP
            if q >= SP:
                yield ("wait", pk_empty[c][ps], q // SP - 1)
            yield ("write", slot[c][ps])
            yield ("async", pk_full[c][ps])
            q += 1
        yield from last_tile(c, 8)

    def unpack(c, g, w):
        q = 0
        for u, (j, outl, k) in enumerate(units):
            if u % NG != g:
                q += 0 if outl else 1
                continue
            st = u % S
            if u >= S:
                yield ("wait", op_empty[c][st], u // S - 1)
            if not outl:
                ps = q % SP
                yield ("wait", pk_full[c][ps], q // SP)
                yield ("own", slot[c][ps])
                yield ("write", stage[c][st])
                yield ("free", slot[c][ps])
                yield ("arrive", pk_empty[c][ps])
                q += 1
            if outl or not x4:
                yield ("wait", x_full[c][st], u // S)
            yield ("arrive", op_full[st])
        yield from last_tile(c, 1 + 4 * g + w)

    def epilogue(c, e):
        for j in range(ntp - 1):
            b, uj = j & 1, j >> 1
            yield ("sync", epi[c])
            if nkb_o > 0:
                yield ("wait", int_done[c][b], uj)
                yield ("own", acc[c][b])
                yield ("free", acc[c][b])
                yield ("arrive", rescaled[b])
            yield ("wait", acc_full[c][b], uj)
            yield ("own", acc[c][b])
            yield ("free", acc[c][b])
            yield ("arrive", acc_empty[b])
        yield from last_tile(c, 12 + e)

    roles = []
    for c in range(2):
        roles += [mma_warp(c), xprod(c), pprod(c)]
        roles += [unpack(c, g, w) for g in range(NG) for w in range(GW)]
        roles += [epilogue(c, e) for e in range(NE)]
    return roles


@pytest.mark.parametrize("ntp", [1, 2, 3, 5])
@pytest.mark.parametrize("nkb_i,nkb_o", [(1, 0), (4, 1), (7, 2), (31, 2), (31, 0), (6, 2)])
@pytest.mark.parametrize("x4", [False, True])
def test_persistent_protocol(ntp, nkb_i, nkb_o, x4):
    for seed in range(4):
        run(persistent_roles(ntp, nkb_i, nkb_o, x4=x4), seed)


def test_checker_catches_a_short_last_rescale_count():
    """The last tile's rescale barrier counting only the epilogue warps (the
    count of the other tiles' barrier): its phase completes before every
    warp has rescaled, and the later arrivals overflow it."""
    assert _caught(lambda: persistent_roles(2, 7, 2, last_rescale_count=2 * 4))


def persistent2_roles(ntp, nkb_i, nkb_o, S=4, SP=3, NG=3, GW=3, skip_epi_done=False, rescale_count=None):
    """The persistent kernel's 512-token form: tiles one after another, each
    tile's k-blocks feeding both accumulators, then every warp of both CTAs
    in the tile's epilogue between CTA-wide named barriers; the next tile's
    MMAs wait until every warp of both CTAs has read the accumulators.  (That
    wait is also implied: the next tile's first operand-full phase needs the
    peer CTA's unpack group, which passes its CTA's closing barrier only after
    all of that CTA's warps have read; skip_epi_done models the kernel
    without it and stays correct.)"""
    op_full = [Bar(2 * GW) for _ in range(S)]
    op_empty = [[Bar(1) for _ in range(S)] for _ in range(2)]
    x_full = [[Bar(1) for _ in range(S)] for _ in range(2)]
    pk_full = [[Bar(1) for _ in range(SP)] for _ in range(2)]
    pk_empty = [[Bar(GW) for _ in range(SP)] for _ in range(2)]
    int_done = [Bar(1) for _ in range(2)]
    acc_full = [Bar(1) for _ in range(2)]
    rescaled, epi_done, mma_done = Bar(rescale_count or 2 * 16), Bar(2 * 16), Bar(1)
    cta = [Sync(16) for _ in range(2)]
    stage = [[Buf(f"CTA {c} operand stage {i}") for i in range(S)] for c in range(2)]
    slot = [[Buf(f"CTA {c} staging slot {i}") for i in range(SP)] for c in range(2)]
    acc = [Buf(f"CTA {c} accumulators") for c in range(2)]
    early = min(SP, ntp * nkb_i)
    ring = {"u": 0}

    def issue(u):
        st = u % S
        yield ("wait", op_full[st], u // S)
        for c in range(2):
            yield ("own", stage[c][st])
        for c in range(2):
            yield ("write", acc[c])
        for c in range(2):
            yield ("async", op_empty[c][st], stage[c][st])

    def epilogue(c, w, j):
        yield ("sync", cta[c])  # every role done with tile j's k-blocks
        yield ("sync", cta[c])  # the token scales staged
        if nkb_o > 0:
            yield ("wait", int_done[c], j)
            yield ("own", acc[c])
            yield ("free", acc[c])
            yield ("arrive", rescaled)
            if c == 0 and w == 0:
                yield ("wait", rescaled, j)
                for _ in range(nkb_o):
                    yield from issue(ring["u"])
                    ring["u"] += 1
                for cc in range(2):
                    yield ("async", acc_full[cc])
        yield ("wait", acc_full[c], j)
        yield ("own", acc[c])
        yield ("free", acc[c])
        yield ("arrive", epi_done)
        yield ("sync", cta[c])  # the ring may take the next tile's operands

    def mma_warp(c):
        for j in range(ntp):
            if c == 0:
                if j > 0 and not skip_epi_done:
                    yield ("wait", epi_done, j - 1)
                for _ in range(nkb_i):
                    yield from issue(ring["u"])
                    ring["u"] += 1
                for cc in range(2):
                    yield ("async", (int_done if nkb_o > 0 else acc_full)[cc])
            yield from epilogue(c, 0, j)
        if c == 0:
            yield ("async", mma_done)
            yield ("wait", mma_done, 0)

    def xprod(c):
        u = 0
        for j in range(ntp):
            for v in range(nkb_i + nkb_o):
                st = u % S
                if u >= S:
                    yield ("wait", op_empty[c][st], u // S - 1)
                yield ("write", stage[c][st])
                yield ("async", x_full[c][st])
                u += 1
            yield from epilogue(c, 4, j)

    def pprod(c):
        q = 0
        for j in range(ntp):
            for k in range(nkb_i):
                if q >= early:
                    ps = q % SP
                    if q >= SP:
                        yield ("wait", pk_empty[c][ps], q // SP - 1)
                    yield ("write", slot[c][ps])
                    yield ("async", pk_full[c][ps])
                q += 1
            yield from epilogue(c, 8, j)

    def prologue(c):
        for q in range(early):  # requested before the set-up barrier
            yield ("write", slot[c][q])
            yield ("async", pk_full[c][q])

    def unpack(c, g, w):
        u = q = 0
        for j in range(ntp):
            for v in range(nkb_i + nkb_o):
                outl = v >= nkb_i
                if u % NG == g:
                    st = u % S
                    if u >= S:
                        yield ("wait", op_empty[c][st], u // S - 1)
                    if not outl:
                        ps = q % SP
                        yield ("wait", pk_full[c][ps], q // SP)
                        yield ("own", slot[c][ps])
                        yield ("write", stage[c][st])
                        yield ("free", slot[c][ps])
                        yield ("arrive", pk_empty[c][ps])
                    yield ("wait", x_full[c][st], u // S)
                    yield ("arrive", op_full[st])
                u += 1
                q += 0 if outl else 1
            yield from epilogue(c, 1 + 4 * g + w, j)

    def epi_warp(c, e):
        for j in range(ntp):
            yield from epilogue(c, 12 + e, j)

    roles = []
    for c in range(2):
        roles += [prologue(c), mma_warp(c), xprod(c), pprod(c)]
        roles += [unpack(c, g, w) for g in range(NG) for w in range(GW)]
        roles += [epi_warp(c, e) for e in range(4)]
    return roles


@pytest.mark.parametrize("ntp", [1, 2, 3])
@pytest.mark.parametrize("nkb_i,nkb_o", [(1, 0), (2, 1), (7, 3), (31, 2), (16, 0), (10, 4)])
@pytest.mark.parametrize("skip", [False, True])
def test_persistent2_protocol(ntp, nkb_i, nkb_o, skip):
    for seed in range(4):
        run(persistent2_roles(ntp, nkb_i, nkb_o, skip_epi_done=skip), seed)


def test_checker_catches_a_staging_ring_smaller_than_the_groups():
    """Six operand stages with two staging slots for three unpack groups: a
    group can reach a slot's phase before its previous phase has landed (a
    parity wait then passes early).  This configuration was built once and
    produced wrong outputs and timeouts on the GPU; the simulation flags it."""
    assert _caught(lambda: persistent_roles(2, 8, 1, S=6, SP=2))


def test_checker_catches_a_short_tile_rescale_count():
    """The 512-token form's rescale barrier counting only four warps per CTA:
    the later arrivals overflow its phase."""
    assert _caught(lambda: persistent2_roles(2, 7, 2, rescale_count=2 * 4))


def _caught(make, seeds=60):
    for seed in range(seeds):
        try:
            run(make(), seed)
        except AssertionError:
            return True
    return False


def test_checker_catches_a_ring_filled_out_of_order():
    """A producer that never waits on the empty barrier runs phases ahead."""
    full, empty = Bar(1), Bar(1)

    def producer():
        for _ in range(6):
            yield ("arrive", full)

    def consumer():
        for u in range(6):
            yield ("wait", full, u)
            yield ("arrive", empty)

    assert _caught(lambda: [producer(), consumer()])


def test_checker_catches_a_stage_overwritten_under_the_mma():
    """B warps that skip the empty wait on the outlier k-blocks (the phases
    still add up) overwrite a stage the MMA still reads."""
    assert _caught(lambda: pair_roles(9, 4, b_waits_outliers=False))


def test_checker_catches_a_single_reduction_slot():
    """The per-token reduction and the INT8 outliers' reduction in the same
    slot (the quantiser's team with the two slots aliased): a fast warp's
    next write races a slower warp's read."""
    def single_slot_roles(rows=6, NR=2, W=4):
        row_full = [Bar(1) for _ in range(NR)]
        red = Buf("reduction slot")
        team = Sync(W)

        def warp(w):
            if w == 0:
                for j in range(min(NR, rows)):
                    yield ("async", row_full[j])
            for j in range(rows):
                if w == 0:
                    yield ("wait", row_full[j % NR], j // NR)
                yield ("sync", team)
                if w == 0 and j > 0 and j - 1 + NR < rows:
                    yield ("async", row_full[(j - 1) % NR])
                yield ("write", red)
                yield ("sync", team)
                yield ("own", red)
                yield ("free", red)
                yield ("write", red)
                yield ("sync", team)
                yield ("own", red)
                yield ("free", red)
        return [warp(w) for w in range(W)]

    assert _caught(single_slot_roles)


def test_checker_catches_a_wrong_accumulator_phase():
    """A drain that waits with the two-buffer phase on four buffers."""
    assert _caught(lambda: grouped_roles(9, 0, drain_phase_div=2))
