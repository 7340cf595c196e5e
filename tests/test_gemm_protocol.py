"""Model check of the barrier protocol of the tensor-core prefill GEMM (tc_gemm.cu).

The dequantized weight tile of each stage lives in tensor memory, in columns tied to the
stage of the shared-memory ring, and one accumulator serves every tile. The kernel's roles
are played by Python generators under random schedules. The tensor core is a FIFO of
issued MMAs that completes them in order at random times. Each tcgen05.commit arrives on
its barrier once every MMA issued before it has completed.

  producer   per (tile, kb) iteration i: wait empty[i % NS] (use i / NS - 1), expect_tx,
             copy X and the raw codes -> raw_full
  dequant    NW warps; per iteration: wait raw_full, write the stage's A columns, arrive
             full
  MMA lane   per tile: wait acc_empty (the previous tile read out); per iteration: wait
             raw_full and full, issue the stage's MMAs, commit empty; after the tile's
             last stage, commit acc_full
  epilogue   NE warps; per tile: wait acc_full, read the accumulator, arrive acc_empty

The model asserts these properties:
- every wait that passes sees exactly the fill it names;
- no A columns are rewritten while an MMA that reads them is still in the tensor core's
  queue;
- no tile's first MMA overwrites the accumulator before the epilogue has read the
  previous tile;
- every schedule terminates.

Planted mistakes (a missing wait) must be caught.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0
        self.fills = []
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


def run_gemm_protocol(tiles, KB, NS, NW, NE, seed, mma_waits_acc_empty=True,
                      producer_waits_empty=True):
    rnd = random.Random(seed)
    raw_full = [Bar(1) for _ in range(NS)]
    full = [Bar(NW) for _ in range(NS)]
    empty = [Bar(1) for _ in range(NS)]
    acc_full = Bar(1)
    acc_empty = Bar(NE)
    inflight = []        # TMA copies not yet landed: (barrier, bytes)
    mma_fifo = []        # issued MMAs: (stage, iteration, commits to fire on completion)
    reading = [0] * NS   # MMAs in the queue that read a stage's A columns
    a_cols = [None] * NS  # iteration whose A tile the stage's columns hold (per warp count)
    a_writes = [0] * NS
    epi_read = []        # tiles the epilogue has finished reading
    acc_tile = [None]    # tile whose partial sums the accumulator holds

    def producer():
        i = 0
        for t in range(tiles):
            for kb in range(KB):
                s, use = i % NS, i // NS
                if use > 0 and producer_waits_empty:
                    while not empty[s].ready((use - 1) & 1):
                        yield
                raw_full[s].expect(("stage", i), 1)
                inflight.append((raw_full[s], 1))
                i += 1
                yield

    def dequant():
        i = 0
        for t in range(tiles):
            for kb in range(KB):
                s, use = i % NS, i // NS
                while not raw_full[s].ready(use & 1):
                    yield
                assert len(raw_full[s].fills) - 1 == use, ("stale or future stage", i)
                assert raw_full[s].fills[use] == ("stage", i)
                assert reading[s] == 0, ("A columns rewritten under a queued MMA", i)
                if a_cols[s] != i:
                    a_cols[s], a_writes[s] = i, 0
                a_writes[s] += 1
                yield  # dequantize, tcgen05.st, wait::st
                full[s].arrive()
                i += 1

    def mma():
        i = 0
        for t in range(tiles):
            if t >= 1 and mma_waits_acc_empty:
                while not acc_empty.ready((t - 1) & 1):
                    yield
            for kb in range(KB):
                s, use = i % NS, i // NS
                while not (raw_full[s].ready(use & 1) and full[s].ready(use & 1)):
                    yield
                assert a_cols[s] == i and a_writes[s] == NW, ("MMA on an unfinished A", i)
                if kb == 0:
                    assert t == 0 or (t - 1) in epi_read, ("accumulator overwritten", t)
                    acc_tile[0] = t
                reading[s] += 1
                commits = [empty[s]] + ([acc_full] if kb == KB - 1 else [])
                mma_fifo.append((s, i, t, commits))
                i += 1
                yield

    def epilogue():
        for t in range(tiles):
            while not acc_full.ready(t & 1):
                yield
            assert len(acc_full.fills) - 1 == t
            assert acc_full.fills[t] == ("acc", t)
            assert acc_tile[0] == t, ("accumulator holds another tile", t)
            yield  # tcgen05.ld, store
            if t not in epi_read:
                epi_read.append(t)
            acc_empty.arrive()

    def complete_mma():
        s, i, t, commits = mma_fifo.pop(0)
        reading[s] -= 1
        for bar in commits:
            bar.arrive(("acc", t) if bar is acc_full else None)

    alive = ([producer(), mma()] + [dequant() for _ in range(NW)] +
             [epilogue() for _ in range(NE)])
    steps = 0
    while alive or inflight or mma_fifo:
        steps += 1
        if steps > 500000:
            raise RuntimeError("deadlock")
        r = rnd.random()
        if inflight and (not alive or r < 0.25):
            bar, tx = inflight.pop(rnd.randrange(len(inflight)))
            bar.land(tx)
            continue
        if mma_fifo and (not alive or r < 0.45):
            complete_mma()
            continue
        if not alive:
            continue
        g = rnd.choice(alive)
        try:
            next(g)
        except StopIteration:
            alive.remove(g)
    assert epi_read == list(range(tiles))


@pytest.mark.parametrize("tiles", [1, 2, 4])
@pytest.mark.parametrize("KB", [1, 3, 7])
@pytest.mark.parametrize("NS", [2, 5, 6])
def test_gemm_protocol_random_schedules(tiles, KB, NS):
    for seed in range(4):
        run_gemm_protocol(tiles, KB, NS, NW=3, NE=2, seed=seed * 7907 + tiles * 31 + KB)


def test_gemm_model_catches_missing_acc_empty_wait():
    """Planted mistake: the MMA lane starts a tile without waiting for the epilogue to have
    read the previous one; the model must see the accumulator overwritten."""
    caught = 0
    for seed in range(30):
        try:
            run_gemm_protocol(4, 2, 4, NW=2, NE=2, seed=seed, mma_waits_acc_empty=False)
        except AssertionError:
            caught += 1
    assert caught > 0


def test_gemm_model_catches_missing_empty_wait():
    """Planted mistake: the producer refills a stage without waiting for its MMAs; the model
    must see a stale stage, A columns rewritten under a queued MMA, or a lost phase."""
    caught = 0
    for seed in range(30):
        try:
            run_gemm_protocol(3, 4, 2, NW=2, NE=1, seed=seed, producer_waits_empty=False)
        except (AssertionError, IndexError, RuntimeError):
            caught += 1
    assert caught > 0
