"""Host models of two more mbarrier protocols (race detection without a GPU).

``rank_rows_kernel``: one TMA producer, one MMA issuer and four epilogue
warps per CTA.  Ring slot s = g % S and parity (g / S) & 1 over the stage
uses g of all the CTA's tiles; the MMA waits on "tempty" with parity
(it - 1) & 1 before the first product of tile it (the epilogue has read tile
it - 1), commits "empty" per stage and "done" once per tile; each epilogue
warp waits on "done" with parity it & 1 and arrives on "tempty".

``nf4_encode_bf16_kernel``'s ring: the producer claims chunks (the first S
statically, then from a counter shared by the CTAs), passes each with its
stage and ends the compute warps' loop with chunk -1 and a plain arrival;
a stage that carried the stop has no copy left to land, so its last copy
parity is reset before the producer's final landing wait.

Both use the exact mbarrier model of ``test_pipeline_model``.  Random
interleavings check: no deadlock, no slot written before its previous
contents were consumed, no accumulator overwritten before it was read,
every tile's sums complete when read, and every chunk processed by exactly
one CTA.  Mutants of each protocol (a missing wait, a kept parity) must
fail.
"""
import random

import pytest

from tests.test_pipeline_model import MBar


def _run(agents, rng):
    live = list(agents)
    idle = 0
    while live:
        g = rng.choice(live)
        try:
            progressed = next(g)
        except StopIteration:
            live.remove(g)
            progressed = True
        idle = 0 if progressed else idle + 1
        assert idle < 200 * len(agents), "deadlock"


def rows_model(m_tiles, grid, nk, S, seed, skip_tempty=False, epi_parity_bug=False):
    rng = random.Random(seed)
    agents, logs = [], []
    for cta in range(grid):
        tiles = list(range(cta, m_tiles, grid))
        full = [MBar(1) for _ in range(S)]
        empty = [MBar(1) for _ in range(S)]
        done = MBar(1)
        tempty = MBar(4)
        slot = [None] * S
        acc = {"tile": None, "steps": 0}
        log = {"consumed": set(), "read": set()}
        logs.append(log)
        BYTES = 4

        def producer(tiles=tiles, full=full, empty=empty, slot=slot, log=log):
            g = 0
            for t in tiles:
                for i in range(nk):
                    s, ph = g % S, (g // S) & 1
                    if g >= S:
                        while not empty[s].try_wait(ph ^ 1):
                            yield False
                    full[s].arrive(expect_tx=BYTES)
                    prev = slot[s]
                    assert prev is None or prev in log["consumed"], "stage overwritten"
                    yield True
                    slot[s] = (t, i)
                    full[s].complete_tx(BYTES)
                    yield True
                    g += 1

        def mma(tiles=tiles, full=full, empty=empty, done=done, tempty=tempty, slot=slot,
                acc=acc, log=log):
            g = 0
            for it, t in enumerate(tiles):
                if it > 0 and not skip_tempty:
                    while not tempty.try_wait((it - 1) & 1):
                        yield False
                for i in range(nk):
                    s, ph = g % S, (g // S) & 1
                    while not full[s].try_wait(ph):
                        yield False
                    assert slot[s] == (t, i), "stage not landed"
                    if i == 0:
                        assert acc["tile"] is None or acc["tile"] in log["read"], \
                            "accumulator overwritten before it was read"
                        acc["tile"], acc["steps"] = t, 0
                    acc["steps"] += 1
                    log["consumed"].add((t, i))
                    empty[s].arrive()
                    g += 1
                    yield True
                done.arrive()
                yield True

        def epilogue(w, tiles=tiles, done=done, tempty=tempty, acc=acc, log=log):
            for it, t in enumerate(tiles):
                par = (it & 1) ^ 1 if epi_parity_bug else it & 1
                while not done.try_wait(par):
                    yield False
                assert acc["tile"] == t and acc["steps"] == nk, "incomplete sums read"
                yield True
                if w == 3:
                    log["read"].add(t)
                tempty.arrive()
                yield True

        agents += [producer(), mma()] + [epilogue(w) for w in range(4)]
    _run(agents, rng)
    read = set().union(*(log["read"] for log in logs))
    assert read == set(range(m_tiles)), "a tile was never written"


@pytest.mark.parametrize("m_tiles,grid", [(32, 20), (3, 2), (5, 5), (7, 2)])
@pytest.mark.parametrize("S", [4, 2, 3])
def test_rows_protocol_random_interleavings(m_tiles, grid, S):
    for seed in range(6):
        rows_model(m_tiles, grid, nk=5, S=S, seed=seed)


def test_rows_model_catches_missing_accumulator_wait():
    """An MMA that starts the next tile without waiting for the epilogue
    overwrites sums that have not been read."""
    failures = 0
    for seed in range(20):
        try:
            rows_model(m_tiles=4, grid=1, nk=3, S=4, seed=seed, skip_tempty=True)
        except AssertionError:
            failures += 1
    assert failures >= 18


def test_rows_model_catches_wrong_done_parity():
    failures = 0
    for seed in range(20):
        try:
            rows_model(m_tiles=3, grid=1, nk=3, S=2, seed=seed, epi_parity_bug=True)
        except AssertionError:
            failures += 1
    assert failures == 20


def encoder_model(nchunks, grid, S, C, seed, keep_stop_parity=False):
    rng = random.Random(seed)
    counter = [0]
    processed = {}            # chunk -> CTA
    agents = []
    for cta in range(grid):
        full = [MBar(1) for _ in range(S)]
        empty = [MBar(C) for _ in range(S)]
        chunk_of = [None] * S
        slot = [None] * S
        read = [set() for _ in range(S)]   # compute warps that have read the stage's chunk
        BYTES = 4

        def producer(cta=cta, full=full, empty=empty, chunk_of=chunk_of, slot=slot, read=read):
            last_parity = [2] * S
            j = 0
            while True:
                s, ph = j % S, (j // S) & 1
                if j >= S:
                    while not empty[s].try_wait(ph ^ 1):
                        yield False
                    assert len(read[s]) == C, "stage reused before every warp read it"
                if j < S:
                    c = cta + j * grid
                else:
                    c = S * grid + counter[0]
                    counter[0] += 1
                    yield True
                if c >= nchunks:
                    chunk_of[s] = -1
                    read[s] = set()
                    full[s].arrive()
                    if not keep_stop_parity:
                        last_parity[s] = 2
                    break
                chunk_of[s] = c
                read[s] = set()
                full[s].arrive(expect_tx=BYTES)
                yield True
                slot[s] = c
                full[s].complete_tx(BYTES)
                last_parity[s] = ph
                j += 1
                yield True
            for s in range(S):
                if last_parity[s] < 2:
                    while not full[s].try_wait(last_parity[s]):
                        yield False

        def compute(w, cta=cta, full=full, empty=empty, chunk_of=chunk_of, slot=slot, read=read):
            j = 0
            while True:
                s, ph = j % S, (j // S) & 1
                while not full[s].try_wait(ph):
                    yield False
                c = chunk_of[s]
                if c < 0:
                    break
                assert slot[s] == c, "chunk read before its copy landed"
                read[s].add(w)
                if w == 0:
                    assert c not in processed, "chunk processed twice"
                    processed[c] = cta
                yield True
                empty[s].arrive()
                j += 1
                yield True

        agents += [producer()] + [compute(w) for w in range(C)]
    _run(agents, rng)
    assert sorted(processed) == list(range(nchunks)), "a chunk was never processed"


@pytest.mark.parametrize("nchunks,grid", [(40, 3), (5, 3), (2, 3), (0, 2), (17, 4)])
@pytest.mark.parametrize("S", [3, 2])
def test_encoder_claims_random_interleavings(nchunks, grid, S):
    for seed in range(6):
        encoder_model(nchunks, grid, S, C=3, seed=seed)


def test_encoder_model_catches_kept_stop_parity():
    """Keeping the stop stage's last copy parity makes the producer's final
    landing wait look for a phase that has been overtaken: it never ends."""
    failures = 0
    for seed in range(10):
        try:
            encoder_model(nchunks=12, grid=1, S=3, C=2, seed=seed, keep_stop_parity=True)
        except AssertionError:
            failures += 1
    assert failures == 10
