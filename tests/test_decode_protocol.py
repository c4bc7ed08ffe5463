"""Deadlock-freedom of the decode kernel's barrier protocol, on the CPU.

An event-driven model of the roles of `decode_kernel` (csrc/w4_decode.cu) for
one CTA: the producer (stage ring: full / empty), the MMA issuer (slot ready ->
MMA-done and empty commits; it takes the next unit's wait before the current
unit's commit, as the kernel does), and the eight dequantizing warps (lane
quarter x unit parity: stage full, slot MMA-done, row-block hand-over between
the two warps of a quarter through xfull / xfree).  Each role is a generator
that yields while the mbarrier phase it waits for has not completed; the run
fails if no role can make progress before all have finished.  The model is
run over the CTA ranges of several layer shapes (stream-K split as the host
computes it), with three TMEM slots (N = 16) and two (N = 32).
"""
import random

import pytest


ARRIVALS = [0]  # every arrive counts: a round with none and no finished role is a deadlock


class Bar:
    """mbarrier: `count` arrivals complete a phase; a wait on parity p
    passes once the phase of that parity has completed."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0

    def arrive(self):
        ARRIVALS[0] += 1
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def run_cta(KS, u0, u1, R, S):
    nu = u1 - u0
    full = [Bar(33) for _ in range(S)]  # TMA arrive_tx + 32 cp.async arrivals
    empty = [Bar(1) for _ in range(S)]
    ready = [Bar(4) for _ in range(R)]  # the unit's four dequant warps
    mdone = [Bar(1) for _ in range(R)]
    xfull = [Bar(1) for _ in range(4)]
    xfree = [Bar(1) for _ in range(4)]

    def land(s):
        for _ in range(33):
            full[s].arrive()

    def producer():
        pre = min(S, nu)
        for it in range(pre):
            land(it)
        s, ph = 0, 1
        for it in range(pre, nu):
            while not empty[s].passed(ph ^ 1):
                yield "empty"
            land(s)
            s += 1
            if s == S:
                s, ph = 0, ph ^ 1

    def mma():
        if nu == 0:
            return
        while not ready[0].passed(0):
            yield "ready0"
        j, jn, pn, s = 0, 1, 0, 0
        for it in range(nu):
            if it + 1 < nu:
                while not ready[jn].passed(pn):
                    yield "ready"
            mdone[j].arrive()
            empty[s].arrive()
            s = (s + 1) % S
            j, jn = jn, jn + 1
            if jn == R:
                jn, pn = 0, pn ^ 1

    def dequant(q, p):
        cur, nflush = -1, 0
        s = j = ph = 0
        pj = 1
        frb = u0 // KS
        fks = u0 % KS
        for it in range(nu + R):
            mine, fold = (it & 1) == p, it >= R
            if fold and frb != cur:
                if cur >= 0:
                    par = nflush & 1
                    nflush += 1
                    if p == 1:
                        while not xfree[q].passed(par ^ 1):
                            yield "xfree"
                        xfull[q].arrive()
                    else:
                        while not xfull[q].passed(par):
                            yield "xfull"
                        xfree[q].arrive()
                cur = frb
            if mine:
                if it < nu:
                    while not full[s].passed(ph):
                        yield "full"
                while not mdone[j].passed(pj):
                    yield "mdone"
                if it < nu:
                    ready[j].arrive()
            s += 1
            if s == S:
                s, ph = 0, ph ^ 1
            j += 1
            if j == R:
                j, pj = 0, pj ^ 1
            if fold:
                fks += 1
                if fks == KS:
                    fks, frb = 0, frb + 1
        if cur >= 0:
            par = nflush & 1
            if p == 1:
                while not xfree[q].passed(par ^ 1):
                    yield "xfree"
                xfull[q].arrive()
            else:
                while not xfull[q].passed(par):
                    yield "xfull"
                xfree[q].arrive()

    roles = {"producer": producer(), "mma": mma()}
    for q in range(4):
        for p in range(2):
            roles[f"dequant q{q} p{p}"] = dequant(q, p)
    state = {k: None for k in roles}
    while roles:
        before = ARRIVALS[0]
        finished = False
        for k in list(roles):
            try:
                state[k] = next(roles[k])
            except StopIteration:
                del roles[k]
                finished = True
        if roles and not finished and ARRIVALS[0] == before:
            # a full round without an arrival: every remaining role waits on a
            # phase that nothing can complete any more
            return {k: state[k] for k in roles}
    return None


def ranges(K, N, sms=148):
    """The host's stream-K split (make_work in csrc/w4_decode.cu)."""
    KS = (K + 255) // 256
    RB = (N + 127) // 128
    U = KS * RB
    P = min(U, sms)
    aligned = RB >= 8 * P or RB > 2048
    if aligned and P > RB:
        P = RB

    def start(c):
        return (c * RB // P) * KS if aligned else c * U // P

    return KS, [(start(c), start(c + 1)) for c in range(P)]


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 11008), (4096, 12288), (8192, 28672),
                                 (384, 1000), (640, 300), (128, 100), (11008, 4096),
                                 (256, 160000), (128, 270000), (384, 151553)])
@pytest.mark.parametrize("R,S", [(3, 7), (2, 5)])
def test_no_deadlock(K, N, R, S):
    KS, rs = ranges(K, N)
    rng = random.Random(K * 31 + N)
    picks = rs if len(rs) <= 24 else [rs[0], rs[-1]] + rng.sample(rs, 22)
    for u0, u1 in picks:
        stuck = run_cta(KS, u0, u1, R, S)
        assert stuck is None, f"units {u0}..{u1}: {stuck}"


def test_model_detects_a_deadlock():
    """The model is not vacuous: an issuer whose commit waited on a later
    unit's barrier would be caught (here: ready counted for 5 warps)."""
    global Bar
    orig = Bar

    class Strict(orig):
        def __init__(self, count):
            super().__init__(5 if count == 4 else count)

    Bar = Strict
    try:
        KS, rs = ranges(4096, 4096)
        assert run_cta(KS, *rs[0], 3, 7) is not None
    finally:
        Bar = orig


def counter_protocol(contrib, counters, stored, abort_after=None):
    """The split row block hand-over of `decode_kernel`, one (row block, warp)
    counter: each contributing CTA stores its partial, then arrives with an
    atomic add; the arrival that reads count - 1 adds the partials (those
    stored so far) and re-arms the counter to 0.  `abort_after` = number of
    contributors that arrive before the rest stop (a bounded wait ran out).
    Returns the partial sum written to Y, or None if nobody wrote it."""
    written = None
    c = len(contrib)
    for i, part in enumerate(contrib):
        if abort_after is not None and i >= abort_after:
            break
        stored.append(part)
        prev = counters[0]
        counters[0] += 1
        if prev == c - 1:
            written = sum(stored)
            counters[0] = 0
    return written


def test_counters_after_a_timeout_need_a_cleared_workspace():
    """A call that stops partway (a bounded wait ran out, W4_ERR_TIMEOUT)
    leaves the counter nonzero; the next call on the same workspace then
    writes no row or a wrong one.  Zero-filling the workspace again, as the
    header asks after W4_ERR_TIMEOUT, restores correct results."""
    parts = [1.0, 2.0, 4.0]
    ws = [0]
    assert counter_protocol(parts, ws, []) == 7.0 and ws[0] == 0  # normal calls re-arm
    assert counter_protocol(parts, ws, [], abort_after=2) is None
    assert ws[0] == 2  # left armed by the aborted call
    assert counter_protocol(parts, ws, []) != 7.0  # stale counter: wrong or missing
    ws[0] = 0  # the workspace zero-filled again
    assert counter_protocol(parts, ws, []) == 7.0
