"""Model check of the barrier protocols of the streaming small-M decode kernels (decode.cu,
gemv_tma.cu).

The kernel's roles are played by Python generators under random schedules, with
mbarrier semantics reduced to what the kernel relies on: a phase completes when its
arrival count and transaction bytes reach zero, and a parity wait passes once the phase
of that parity has completed (so a waiter two phases behind would be fooled). The model
asserts that every wait that passes sees exactly the fill it names (no stale or future
data), and that every schedule terminates (no deadlock):

  producer   per chunk i: wait empty[i % NS] (use i / NS - 1), expect_tx, copy -> full
  prep       keeps RS tiles of raw S'/Z in flight; per tile: wait rawfull, wait
             prepempty (tile - TS), transpose, arrive prepfull, refill the raw slot
  consumers  NW warps; each waits for every chunk of every tile in order, and for the
             tile's prepfull after its first chunk; arrives empty, then tdone per tile
  epilogue   per tile: wait tdone, arrive prepempty

A second check plants the mistake the protocol avoids (chunks dealt round-robin to warps
over a shared ring smaller than twice the warp count) and requires the model to catch it.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0
        self.fills = []  # payload of each completed phase
        self.cur = None

    def arrive(self, payload=None):
        if payload is not None:
            self.cur = payload
        self.pending -= 1
        self._complete()

    def expect(self, payload, tx):
        self.tx += tx
        self.cur = payload
        self.pending -= 1
        self._complete()

    def land(self, tx):
        self.tx -= tx
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.fills.append(self.cur)
            self.phase += 1
            self.pending = self.count

    def ready(self, parity):
        return (self.phase & 1) != parity


def run_protocol(tiles, NC, NW, NS, RS, TS, seed):
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(NS)]
    empty = [Bar(NW) for _ in range(NS)]
    rawfull = [Bar(1) for _ in range(RS)]
    prepfull = [Bar(1) for _ in range(TS)]
    prepempty = [Bar(1) for _ in range(TS)]
    tdone = [Bar(NW) for _ in range(TS)]
    inflight = []
    prep_done = []

    def producer():
        i = 0
        for tl in range(tiles):
            for ch in range(NC):
                st, use = i % NS, i // NS
                if use > 0:
                    while not empty[st].ready((use - 1) & 1):
                        yield
                full[st].expect(("chunk", i), 1)
                inflight.append((full[st], 1))
                i += 1
                yield

    def prep():
        def issue(t):
            rawfull[t % RS].expect(("raw", t), 1)
            inflight.append((rawfull[t % RS], 1))
        issued = min(RS, tiles)
        for t in range(issued):
            issue(t)
        for tl in range(tiles):
            rs, ps = tl % RS, tl % TS
            while not rawfull[rs].ready((tl // RS) & 1):
                yield
            assert rawfull[rs].fills[tl // RS] == ("raw", tl)
            assert len(rawfull[rs].fills) - 1 == tl // RS, "raw slot overrun"
            if tl >= TS:
                while not prepempty[ps].ready(((tl // TS) - 1) & 1):
                    yield
            yield  # transpose
            prep_done.append(tl)
            prepfull[ps].arrive(("prep", tl))
            if issued < tiles:
                issue(issued)
                issued += 1
            yield

    def consumer():
        i = 0
        for tl in range(tiles):
            ps = tl % TS
            for ch in range(NC):
                st = i % NS
                while not full[st].ready((i // NS) & 1):
                    yield
                assert len(full[st].fills) - 1 == i // NS, ("stale or future chunk", i)
                assert full[st].fills[i // NS] == ("chunk", i)
                if ch == 0:
                    while not prepfull[ps].ready((tl // TS) & 1):
                        yield
                    assert len(prepfull[ps].fills) - 1 == tl // TS, ("stale S'/Z", tl)
                    assert prepfull[ps].fills[tl // TS] == ("prep", tl)
                yield  # compute
                empty[st].arrive()
                i += 1
            tdone[ps].arrive()
            yield

    def epilogue():
        for tl in range(tiles):
            ps = tl % TS
            while not tdone[ps].ready((tl // TS) & 1):
                yield
            assert len(tdone[ps].fills) - 1 == tl // TS
            yield
            prepempty[ps].arrive()

    alive = [producer(), prep(), epilogue()] + [consumer() for _ in range(NW)]
    steps = 0
    while alive or inflight:
        steps += 1
        if steps > 400000:
            raise RuntimeError("deadlock")
        if inflight and (not alive or rnd.random() < 0.3):
            bar, tx = inflight.pop(rnd.randrange(len(inflight)))
            bar.land(tx)
            continue
        g = rnd.choice(alive)
        try:
            next(g)
        except StopIteration:
            alive.remove(g)
    assert prep_done == list(range(tiles))


@pytest.mark.parametrize("tiles", [1, 2, 5, 9])
@pytest.mark.parametrize("NC", [1, 2, 3])
@pytest.mark.parametrize("NS,RS", [(2, 2), (3, 4), (5, 4), (16, 2)])
def test_decode_protocol_random_schedules(tiles, NC, NS, RS):
    for seed in range(4):
        run_protocol(tiles, NC, NW=8, NS=NS, RS=RS, TS=4, seed=seed * 7919 + tiles)


def run_round_robin_shared_ring(total, NW, NS, seed):
    """The rejected design: chunk i to warp i % NW over a ring of NS shared stages."""
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(NS)]
    empty = [Bar(1) for _ in range(NS)]
    inflight = []

    def producer():
        for i in range(total):
            st, use = i % NS, i // NS
            if use > 0:
                while not empty[st].ready((use - 1) & 1):
                    yield
            full[st].expect(("chunk", i), 1)
            inflight.append((full[st], 1))
            yield

    def consumer(w):
        for i in range(w, total, NW):
            st = i % NS
            while not full[st].ready((i // NS) & 1):
                yield
            assert full[st].fills[-1] == ("chunk", i), ("read the wrong fill", i)
            yield
            empty[st].arrive()

    alive = [producer()] + [consumer(w) for w in range(NW)]
    steps = 0
    while alive or inflight:
        steps += 1
        if steps > 200000:
            raise RuntimeError("deadlock")
        if inflight and (not alive or rnd.random() < 0.3):
            bar, tx = inflight.pop(rnd.randrange(len(inflight)))
            bar.land(tx)
            continue
        g = rnd.choice(alive)
        try:
            next(g)
        except StopIteration:
            alive.remove(g)


def test_model_catches_round_robin_aliasing():
    caught = 0
    for seed in range(20):
        try:
            run_round_robin_shared_ring(total=44, NW=16, NS=10, seed=seed)
        except (AssertionError, IndexError):
            caught += 1
    assert caught > 0



def run_tma_protocol(tiles, NC, NW, NS, SS, KP, seed, producer_waits=True):
    """The TMA-fed 32-row-tile decode kernel (gemv_tma.cu):

    producer   per tile: wait szempty[tile % SS] (tile - SS consumed), S'/Z copy -> szfull;
               then its NC chunks: wait empty[i % NS], copy -> full
    consumers  NW warps; every chunk of every tile in order, the tile's szfull after its
               first chunk; arrive empty per chunk, szempty per tile; then wait
               pempty[tile % KP] (epilogue done with tile - KP), write partials, arrive tdone
    epilogue   per tile: wait tdone, sum, arrive pempty
    """
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(NS)]
    empty = [Bar(NW) for _ in range(NS)]
    szfull = [Bar(1) for _ in range(SS)]
    szempty = [Bar(NW) for _ in range(SS)]
    tdone = [Bar(NW) for _ in range(KP)]
    pempty = [Bar(1) for _ in range(KP)]
    inflight = []
    epi_done = []

    def producer():
        i = 0
        for tl in range(tiles):
            ss = tl % SS
            if tl >= SS and producer_waits:
                while not szempty[ss].ready((tl // SS - 1) & 1):
                    yield
            szfull[ss].expect(("sz", tl), 1)
            inflight.append((szfull[ss], 1))
            yield
            for ch in range(NC):
                st, use = i % NS, i // NS
                if use > 0:
                    while not empty[st].ready((use - 1) & 1):
                        yield
                full[st].expect(("chunk", i), 1)
                inflight.append((full[st], 1))
                i += 1
                yield

    def consumer():
        i = 0
        for tl in range(tiles):
            ss, kp = tl % SS, tl % KP
            for ch in range(NC):
                st = i % NS
                while not full[st].ready((i // NS) & 1):
                    yield
                assert len(full[st].fills) - 1 == i // NS, ("stale or future chunk", i)
                assert full[st].fills[i // NS] == ("chunk", i)
                if ch == 0:
                    while not szfull[ss].ready((tl // SS) & 1):
                        yield
                assert len(szfull[ss].fills) - 1 == tl // SS, ("stale or future S'/Z", tl)
                assert szfull[ss].fills[tl // SS] == ("sz", tl)
                yield  # compute
                empty[st].arrive()
                i += 1
            szempty[ss].arrive()
            if tl >= KP:
                while not pempty[kp].ready((tl // KP - 1) & 1):
                    yield
            yield  # partials
            tdone[kp].arrive(("tile", tl))
            yield

    def epilogue():
        for tl in range(tiles):
            kp = tl % KP
            while not tdone[kp].ready((tl // KP) & 1):
                yield
            assert len(tdone[kp].fills) - 1 == tl // KP
            yield
            epi_done.append(tl)
            pempty[kp].arrive()

    alive = [producer(), epilogue()] + [consumer() for _ in range(NW)]
    steps = 0
    while alive or inflight:
        steps += 1
        if steps > 600000:
            raise RuntimeError("deadlock")
        if inflight and (not alive or rnd.random() < 0.3):
            bar, tx = inflight.pop(rnd.randrange(len(inflight)))
            bar.land(tx)
            continue
        g = rnd.choice(alive)
        try:
            next(g)
        except StopIteration:
            alive.remove(g)
    assert epi_done == list(range(tiles))


@pytest.mark.parametrize("tiles", [1, 2, 3, 7])
@pytest.mark.parametrize("NC", [1, 3])
@pytest.mark.parametrize("NS", [2, 5])
def test_tma_protocol_random_schedules(tiles, NC, NS):
    for seed in range(4):
        run_tma_protocol(tiles, NC, NW=6, NS=NS, SS=2, KP=2, seed=seed * 104729 + tiles)


def test_tma_model_catches_missing_slot_wait():
    """Planted mistake: the producer refills an S'/Z slot without waiting for the consumers
    to release it; the model must see a consumer read the wrong tile's S'/Z, or a wait that
    can no longer complete."""
    caught = 0
    for seed in range(30):
        try:
            run_tma_protocol(6, 1, NW=6, NS=4, SS=2, KP=2, seed=seed, producer_waits=False)
        except (AssertionError, IndexError, RuntimeError):  # wrong tile read, or a lost phase
            caught += 1
    assert caught > 0
