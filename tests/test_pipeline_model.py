"""Host model of the fused kernel's mbarrier protocol (race detection without
a GPU).

``fused_nf4_gemm_kernel`` runs on a pair of CTAs.  Its roles are modelled as
generators that use the kernel's own index arithmetic: ring slot
s = i % S and parity (i / S) & 1; producers wait on their CTA's "empty" with
the flipped parity, consumers on "full" with the plain one; the MMA (CTA 0
only) waits for accumulator h with parity (item & 1) ^ 1 at the first K-step
of an item, and each CTA's epilogue waits on its "tfull" with parity
item & 1.  The pair protocol: CTA 0's producer arms CTA 0's activation
barrier with both CTAs' bytes and both producers' copies complete their
bytes there; decoder groups take K-steps in turn and every decoder warp of
both CTAs arrives on CTA 0's barrier of the stage; the MMA's commits arrive
on the stage and accumulator barriers of both CTAs (multicast); both CTAs'
epilogue warps release an accumulator on CTA 0's barrier.  An mbarrier is
modelled exactly (pending arrivals, transaction count, phase bit,
try_wait(parity) true once the phase with that parity has completed).
Random interleavings check: no deadlock, no ring slot of either CTA written
before its previous contents were consumed, no accumulator of either CTA
overwritten before its epilogue drained it, and every item's sums complete
when read.
"""
import random

import pytest


class MBar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0           # parity of the phase in progress

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase ^= 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        assert self.pending >= 0
        self._maybe_complete()

    def complete_tx(self, n):
        self.tx -= n               # may go below zero before the arming arrival
        self._maybe_complete()

    def try_wait(self, parity):
        # true once the phase with this parity has completed, i.e. the phase
        # in progress has the other parity
        return self.phase != parity


def model(n_items, nk, A, B, groups, n_dec, n_epi, n_acc, seed, producer_parity_bug=False,
          arm_one_cta_only=False):
    rng = random.Random(seed)
    ctas = (0, 1)
    full_a = [MBar(1) for _ in range(A)]                     # CTA 0's, armed by CTA 0
    empty_a = {q: [MBar(1) for _ in range(A)] for q in ctas}
    full_b = [MBar(2 * n_dec) for _ in range(B)]             # CTA 0's
    empty_b = {q: [MBar(1) for _ in range(B)] for q in ctas}
    tfull = {q: MBar(1) for q in ctas}
    tempty = [MBar(2 * n_epi) for _ in range(n_acc)]         # CTA 0's
    a_slot = {q: [None] * A for q in ctas}
    b_slot = {q: [[None] * n_dec for _ in range(B)] for q in ctas}
    acc = {q: [None] * n_acc for q in ctas}                   # item whose sums each holds
    acc_steps = {q: [0] * n_acc for q in ctas}
    steps = [(it, k) for it in range(n_items) for k in range(nk)]
    log = {"consumed_a": set(), "consumed_b": set(), "drained": {q: set() for q in ctas}}
    BYTES = 4

    def producer(q):
        for i, st in enumerate(steps):
            s, ph = i % A, (i // A) & 1
            while not empty_a[q][s].try_wait(ph if producer_parity_bug else ph ^ 1):
                yield False
            if q == 0:
                full_a[s].arrive(expect_tx=BYTES if arm_one_cta_only else 2 * BYTES)
            prev = a_slot[q][s]
            assert prev is None or prev in log["consumed_a"], "activation slot overwritten"
            yield True
            a_slot[q][s] = st
            full_a[s].complete_tx(BYTES)   # this CTA's copy lands
            yield True

    def decoder(q, g, d):
        for i in range(g, len(steps), groups):
            st = steps[i]
            s, ph = i % B, (i // B) & 1
            while not empty_b[q][s].try_wait(ph ^ 1):
                yield False
            prev = b_slot[q][s][d]
            assert prev is None or prev in log["consumed_b"], "decoded slot overwritten"
            b_slot[q][s][d] = st
            full_b[s].arrive()              # CTA 0's barrier, local or remote
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
            for q in ctas:
                assert a_slot[q][sa] == st, "activation half missing"
                assert all(x == st for x in b_slot[q][sb]), "decoded half missing"
            for h in range(n_acc):
                if k == 0:
                    while not tempty[h].try_wait((it & 1) ^ 1):
                        yield False
                    for q in ctas:
                        assert acc[q][h] is None or acc[q][h] in log["drained"][q], \
                            "accumulator reused early"
                        acc[q][h], acc_steps[q][h] = it, 0
                for q in ctas:
                    acc_steps[q][h] += 1
            log["consumed_a"].add(st)
            log["consumed_b"].add(st)
            for q in ctas:                  # multicast commits
                empty_a[q][sa].arrive()
                empty_b[q][sb].arrive()
            if k == nk - 1:
                for q in ctas:
                    tfull[q].arrive()
            yield True

    def epilogue(q, e):
        for it in range(n_items):
            while not tfull[q].try_wait(it & 1):
                yield False
            for h in range(n_acc):
                assert acc[q][h] == it and acc_steps[q][h] == nk, "incomplete sums read"
                yield True
                if e == n_epi - 1:
                    log["drained"][q].add(it)
                tempty[h].arrive()          # CTA 0's barrier
            yield True

    agents = [producer(0), producer(1), mma()]
    agents += [decoder(q, g, d) for q in ctas for g in range(groups) for d in range(n_dec)]
    agents += [epilogue(q, e) for q in ctas for e in range(n_epi)]
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


# two accumulators per CTA (128 lanes x 256 columns each), two decoder groups
@pytest.mark.parametrize("A,B", [(4, 4), (2, 2), (3, 2), (4, 3)])
@pytest.mark.parametrize("groups", [2, 1])
def test_fused_protocol_random_interleavings(A, B, groups):
    for seed in range(12):
        model(n_items=3, nk=5, A=A, B=B, groups=groups, n_dec=2, n_epi=2, n_acc=2, seed=seed)


def test_mbarrier_model():
    bar = MBar(1)
    assert bar.try_wait(1) and not bar.try_wait(0)   # fresh barrier: phase 0 in progress
    bar.arrive()
    assert bar.try_wait(0) and not bar.try_wait(1)
    # bytes that land before the arming arrival keep the phase open until it comes
    bar = MBar(1)
    bar.complete_tx(4)
    assert not bar.try_wait(0)
    bar.arrive(expect_tx=8)
    assert not bar.try_wait(0)
    bar.complete_tx(4)
    assert bar.try_wait(0)


def test_model_catches_a_wrong_parity():
    """A producer that waits on "empty" with the consumers' parity either
    overwrites a live slot or never starts: the model must reject it."""
    failures = 0
    for seed in range(20):
        try:
            model(n_items=2, nk=5, A=2, B=2, groups=2, n_dec=2, n_epi=2, n_acc=2, seed=seed,
                  producer_parity_bug=True)
        except AssertionError:
            failures += 1
    assert failures == 20


def test_model_catches_arming_for_one_cta():
    """CTA 0 arming its barrier with only its own bytes lets the MMA start
    before the peer's half has landed (or leaves the phase unbalanced)."""
    failures = 0
    for seed in range(20):
        try:
            model(n_items=2, nk=5, A=2, B=2, groups=2, n_dec=2, n_epi=2, n_acc=2, seed=seed,
                  arm_one_cta_only=True)
        except AssertionError:
            failures += 1
    assert failures == 20
