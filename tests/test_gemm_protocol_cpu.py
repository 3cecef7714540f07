"""The tcgen05 GEMM's mbarrier protocol, modelled on the CPU.

The kernel (weight_shared_looped_b200/csrc/gemm_tc.cu) hands work between its
warp roles through four barrier rings: an activation ring of XS k blocks
(xfull: the TMA copy landed; xempty: the MMAs of that k block completed), and
a TMEM A ring of AB batches of BATCH k blocks (afull: every dequantisation
warp stored its tile and the watcher saw the batch's activations land; done:
the MMAs of that batch completed).  The model below runs the same roles -- the
TMA warp, the watcher, the MMA warp and DQ dequantisation warps, with the
copies and MMA completions as asynchronous events -- in seeded random orders
and speeds, with the ring depths read from the kernel source, and checks every
hand-off: the MMAs of a batch start only on A tiles that all dequantisation
warps wrote and on activation tiles that landed; no tile is overwritten before
the MMAs that read it completed; nothing stalls for good.

The negative control removes the watcher's wait for its A slot's previous
phase: with the 64-token tile's ring depths (activation ring deeper than the A
ring) the model then sees a barrier phase complete early, or a stall."""
import os
import random
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "weight_shared_looped_b200", "csrc", "gemm_tc.cu")


def _source():
    with open(SRC) as f:
        return f.read()


def _ring_depths():
    """{BN: (XS, AB, BATCH, DQ)} for the token tiles the launcher uses."""
    src = _source()

    def num(pat):
        m = re.search(pat, src)
        assert m, pat
        return int(m.group(1))

    bk = num(r"constexpr int BK = (\d+);")
    groups = num(r"constexpr int DQ_GROUPS = (\d+);")
    tmem = num(r"constexpr int TMEM_COLS = (\d+);")
    assert re.search(r"constexpr int A_COLS = BK / 2;", src)
    assert re.search(r"constexpr int BATCH = DQ_GROUPS;", src)
    assert re.search(r"constexpr int DQ_WARPS = 4 \* DQ_GROUPS;", src)
    assert "A_BATCHES = (TMEM_COLS - BN) / (A_COLS * BATCH)" in src
    m = re.search(r"X_STAGES = BN >= 128 \? (\d+) : (\d+);", src)
    assert m
    tiles = sorted(set(int(x) for x in re.findall(r"launch_tc_bn<(\d+), [34], (?:true|false)>", src)))
    assert tiles == [64, 128], tiles
    out = {}
    for bn in tiles:
        xs = int(m.group(1)) if bn >= 128 else int(m.group(2))
        out[bn] = (xs, (tmem - bn) // ((bk // 2) * groups), groups, 4 * groups)
    return out


class Barrier:
    """An mbarrier: a phase completes when its pending arrivals reach zero and
    its transaction count is zero; a wait names the parity of the phase."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def _advance(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._advance()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._advance()

    def passed(self, parity):
        # try_wait.parity(p) succeeds once the phase with parity p has completed
        return (self.phase & 1) != parity


class Violation(AssertionError):
    pass


def simulate(nkb, XS, AB, BATCH, DQ, *, watcher_waits=True, seed=0, dq_stall=0.3):
    """Runs the protocol for nkb k blocks; raises Violation on a broken
    hand-off or a stall."""
    rnd = random.Random(seed)
    nbatch = -(-nkb // BATCH)
    X_BYTES = 1
    xfull = [Barrier(1) for _ in range(XS)]
    xempty = [Barrier(1) for _ in range(XS)]
    afull = [Barrier(DQ + 1) for _ in range(AB)]
    done = [Barrier(1) for _ in range(AB)]
    accb = Barrier(1)
    landed = set()          # k blocks whose activation tile is in its slot
    mma_done_kb = set()     # k blocks whose MMAs completed
    mma_done_b = set()      # batches whose MMAs completed
    written = {}            # batch -> dequantisation warps that stored its tiles
    events = []             # asynchronous completions (copies, MMA commits)

    def check(cond, what):
        if not cond:
            raise Violation(what)

    def tma():
        for i in range(nkb):
            if i >= XS:
                while not xempty[i % XS].passed((i // XS - 1) & 1):
                    yield False
                check(i - XS in mma_done_kb, f"activation slot of k block {i - XS} reused early")
                landed.discard(i - XS)
            xfull[i % XS].arrive_expect_tx(X_BYTES)

            def land(i=i):
                landed.add(i)
                xfull[i % XS].complete_tx(X_BYTES)
            events.append(land)
            yield True

    def watcher():
        for b in range(nbatch):
            for i in range(b * BATCH, min(nkb, (b + 1) * BATCH)):
                while not xfull[i % XS].passed((i // XS) & 1):
                    yield False
            if watcher_waits and b >= AB:
                while not afull[b % AB].passed(((b - AB) // AB) & 1):
                    yield False
            afull[b % AB].arrive()
            yield True

    def mma():
        for b in range(nbatch):
            while not afull[b % AB].passed((b // AB) & 1):
                yield False
            check(written.get(b, 0) == DQ, f"batch {b} started with {written.get(b, 0)} of {DQ} A tiles")
            for i in range(b * BATCH, min(nkb, (b + 1) * BATCH)):
                check(i in landed, f"k block {i} read before its activations landed")

                def kb_done(i=i):
                    mma_done_kb.add(i)
                    xempty[i % XS].arrive()
                events.append(kb_done)

            def b_done(b=b):
                mma_done_b.add(b)
                done[b % AB].arrive()
            events.append(b_done)
            yield True
        events.append(accb.arrive)

    def dequant():
        for b in range(nbatch):
            if b >= AB:
                while not done[(b - AB) % AB].passed(((b - AB) // AB) & 1):
                    yield False
                check(b - AB in mma_done_b, f"A slot of batch {b - AB} overwritten early")
            while rnd.random() < dq_stall:         # weight loads and dequantisation
                yield True
            written[b] = written.get(b, 0) + 1
            afull[b % AB].arrive()
            yield True
        while not accb.passed(0):
            yield False

    actors = [tma(), watcher(), mma()] + [dequant() for _ in range(DQ)]
    blocked = set()
    while actors:
        if events and (rnd.random() < 0.5 or len(blocked) == len(actors)):
            events.pop(rnd.randrange(len(events)))()
            blocked.clear()
            continue
        if len(blocked) == len(actors):
            raise Violation("stall: every role waits and nothing is in flight")
        a = rnd.choice(actors)
        try:
            progressed = next(a)
        except StopIteration:
            actors.remove(a)
            blocked.discard(id(a))
            blocked.clear()
            continue
        if progressed:
            blocked.clear()
        else:
            blocked.add(id(a))
    while events:
        events.pop()()
    check(sorted(mma_done_b) == list(range(nbatch)), "not every batch completed")


KBLOCKS = [1, 3, 4, 5, 12, 13, 16, 17, 31, 64]


@pytest.mark.parametrize("bn", [64, 128])
def test_protocol_hand_offs_hold(bn):
    XS, AB, BATCH, DQ = _ring_depths()[bn]
    for nkb in KBLOCKS:
        for seed in range(6):
            for stall in (0.0, 0.5, 0.9):
                simulate(nkb, XS, AB, BATCH, DQ, seed=seed, dq_stall=stall)


def test_watcher_wait_is_in_the_kernel():
    src = _source()
    assert re.search(r"warp_wait\(&afull\[b % AB\], \(\(b - AB\) / AB\) & 1", src)


def test_without_watcher_wait_the_deep_ring_breaks():
    """Negative control: the model catches the early phase completion the
    watcher's wait prevents, for the 64-token ring depths."""
    XS, AB, BATCH, DQ = _ring_depths()[64]
    assert XS > AB * BATCH          # the activation ring can run a batch past the A ring
    failures = 0
    for seed in range(20):
        try:
            simulate(64, XS, AB, BATCH, DQ, watcher_waits=False, seed=seed, dq_stall=0.9)
        except Violation:
            failures += 1
    assert failures > 0
