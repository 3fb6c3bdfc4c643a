"""Host model of the fused kernel's mbarrier protocol (race detection without
a GPU).

The four roles of ``fused_nf4_gemm_kernel`` are modelled as generators that
use the kernel's own index arithmetic: ring slot s = i % S and parity
(i / S) & 1; producers wait on "empty" with the flipped parity, consumers on
"full" with the plain one; the MMA waits for accumulator h with parity
(item & 1) ^ 1 at the first K-step of an item, and the epilogue waits on
"tfull" with parity item & 1.  An mbarrier is modelled exactly (pending
count, phase bit, try_wait(parity) true once the phase with that parity has
completed).  Random interleavings check: no deadlock, no ring slot written
before its previous contents were consumed, no accumulator overwritten
before the epilogue drained it, and every item's sums complete when read.
"""
import random

import pytest


class MBar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0           # parity of the phase in progress

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase ^= 1
            self.pending = self.count

    def try_wait(self, parity):
        # true once the phase with this parity has completed, i.e. the phase
        # in progress has the other parity
        return self.phase != parity


def model(n_items, nk, A, B, n_dec, n_epi, n_acc, seed, producer_parity_bug=False):
    rng = random.Random(seed)
    full_a = [MBar(1) for _ in range(A)]
    empty_a = [MBar(1) for _ in range(A)]
    full_b = [MBar(n_dec) for _ in range(B)]
    empty_b = [MBar(1) for _ in range(B)]
    tfull = MBar(1)
    tempty = [MBar(n_epi) for _ in range(n_acc)]
    a_slot = [None] * A          # (step id) written into each activation slot
    b_slot = [[None] * n_dec for _ in range(B)]
    acc = [None] * n_acc          # item whose sums the accumulator holds
    acc_steps = [0] * n_acc
    steps = [(it, k) for it in range(n_items) for k in range(nk)]
    log = {"consumed_a": set(), "consumed_b": set(), "drained": set()}

    def producer():
        for i, st in enumerate(steps):
            s, ph = i % A, (i // A) & 1
            while not empty_a[s].try_wait(ph if producer_parity_bug else ph ^ 1):
                yield False
            prev = a_slot[s]
            assert prev is None or prev in log["consumed_a"], "activation slot overwritten"
            a_slot[s] = st
            full_a[s].arrive()          # TMA completion
            yield True

    def decoder(d):
        for i, st in enumerate(steps):
            s, ph = i % B, (i // B) & 1
            while not empty_b[s].try_wait(ph ^ 1):
                yield False
            prev = b_slot[s][d]
            assert prev is None or prev in log["consumed_b"], "decoded slot overwritten"
            b_slot[s][d] = st
            full_b[s].arrive()
            yield True

    def mma():
        for i, st in enumerate(steps):
            it, k = st
            sa, pa = i % A, (i // A) & 1
            sb, pb = i % B, (i // B) & 1
            while not full_a[sa].try_wait(pa):
                yield False
            while not full_b[sb].try_wait(pb):
                yield False
            assert a_slot[sa] == st and all(x == st for x in b_slot[sb])
            for h in range(n_acc):
                if k == 0:
                    while not tempty[h].try_wait((it & 1) ^ 1):
                        yield False
                    assert acc[h] is None or acc[h] in log["drained"], "accumulator reused early"
                    acc[h], acc_steps[h] = it, 0
                acc_steps[h] += 1
            log["consumed_a"].add(st)
            log["consumed_b"].add(st)
            empty_a[sa].arrive()        # commit after the MMAs
            empty_b[sb].arrive()
            if k == nk - 1:
                tfull.arrive()
            yield True

    def epilogue(e):
        for it in range(n_items):
            while not tfull.try_wait(it & 1):
                yield False
            for h in range(n_acc):
                assert acc[h] == it and acc_steps[h] == nk, "incomplete sums read"
                yield True
                if e == n_epi - 1:
                    log["drained"].add(it)
                tempty[h].arrive()
            yield True

    agents = [producer(), mma()] + [decoder(d) for d in range(n_dec)] + [epilogue(e) for e in range(n_epi)]
    live = list(agents)
    idle = 0                      # consecutive turns in which nobody progressed
    while live:
        g = rng.choice(live)
        try:
            progressed = next(g)
        except StopIteration:
            live.remove(g)
            progressed = True
        idle = 0 if progressed else idle + 1
        assert idle < 200 * len(agents), "deadlock"


# n_acc: four accumulators of 128 x 128 (forward), two of 128 x 256 (dX)
@pytest.mark.parametrize("n_acc", [4, 2])
@pytest.mark.parametrize("A,B", [(2, 4), (2, 2), (3, 2), (4, 3)])
def test_fused_protocol_random_interleavings(A, B, n_acc):
    for seed in range(20):
        model(n_items=3, nk=5, A=A, B=B, n_dec=4, n_epi=4, n_acc=n_acc, seed=seed)


def test_mbarrier_model():
    bar = MBar(1)
    assert bar.try_wait(1) and not bar.try_wait(0)   # fresh barrier: phase 0 in progress
    bar.arrive()
    assert bar.try_wait(0) and not bar.try_wait(1)


def test_model_catches_a_wrong_parity():
    """A producer that waits on "empty" with the consumers' parity either
    overwrites a live slot or never starts: the model must reject it."""
    failures = 0
    for seed in range(20):
        try:
            model(n_items=2, nk=5, A=2, B=2, n_dec=2, n_epi=2, n_acc=2, seed=seed,
                  producer_parity_bug=True)
        except AssertionError:
            failures += 1
    assert failures == 20
