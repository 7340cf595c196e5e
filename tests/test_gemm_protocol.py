"""Model checks of the barrier protocols of the tensor-core kernels: the prefill GEMM
(tc_gemm.cu) and, at the end, the skinny kernel's INT4 form (tc_skinny.cu).

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


def run_skinny_protocol(groups, LS, OS, NB, NW, NE, seed, expansion_waits_op_empty=True):
    """The skinny tensor-core kernel's INT4 form (tc_skinny.cu), one CTA:

    producer   per group i: wait ld_empty[i % LS], copy the packed codes -> ld_full; wait
               op_empty[i % OS], copy the activations into the operand stage -> b_full
    expansion  NW warps; per group: wait ld_full and op_empty, write A into the operand
               stage, arrive ld_empty and a_full
    MMA lane   per group: wait a_full, b_full and acc_empty[i % NB], issue, commit op_empty
               and acc_full[i % NB]
    epilogue   NE warps; per group: wait acc_full, read the accumulator, arrive acc_empty
    """
    rnd = random.Random(seed)
    ld_full = [Bar(1) for _ in range(LS)]
    ld_empty = [Bar(NW) for _ in range(LS)]
    a_full = [Bar(NW) for _ in range(OS)]
    b_full = [Bar(1) for _ in range(OS)]
    op_empty = [Bar(1) for _ in range(OS)]
    acc_full = [Bar(1) for _ in range(NB)]
    acc_empty = [Bar(NE) for _ in range(NB)]
    inflight, mma_fifo = [], []
    reading = [0] * OS
    a_of = [None] * OS
    a_writes = [0] * OS
    acc_of = [None] * NB
    epi_reads = [0] * groups

    def producer():
        for i in range(groups):
            s, u = i % LS, i // LS
            if u > 0:
                while not ld_empty[s].ready((u - 1) & 1):
                    yield
            ld_full[s].expect(("codes", i), 1)
            inflight.append((ld_full[s], 1))
            yield
            o, ou = i % OS, i // OS
            if ou > 0:
                while not op_empty[o].ready((ou - 1) & 1):
                    yield
            b_full[o].expect(("x", i), 1)
            inflight.append((b_full[o], 1))
            yield

    def expansion():
        for i in range(groups):
            s, u, o, ou = i % LS, i // LS, i % OS, i // OS
            while not ld_full[s].ready(u & 1):
                yield
            if ou > 0 and expansion_waits_op_empty:
                while not op_empty[o].ready((ou - 1) & 1):
                    yield
            assert len(ld_full[s].fills) - 1 == u and ld_full[s].fills[u] == ("codes", i)
            assert reading[o] == 0, ("A rewritten under a queued MMA", i)
            if a_of[o] != i:
                a_of[o], a_writes[o] = i, 0
            a_writes[o] += 1
            yield
            ld_empty[s].arrive()
            a_full[o].arrive()

    def mma():
        for i in range(groups):
            o, ou, b, v = i % OS, i // OS, i % NB, i // NB
            while not (a_full[o].ready(ou & 1) and b_full[o].ready(ou & 1)):
                yield
            if v > 0:
                while not acc_empty[b].ready((v - 1) & 1):
                    yield
            assert a_of[o] == i and a_writes[o] == NW, ("MMA on an unfinished A", i)
            assert len(b_full[o].fills) - 1 == ou and b_full[o].fills[ou] == ("x", i)
            assert v == 0 or epi_reads[i - NB] == NE, ("accumulator overwritten", i)
            acc_of[b] = i
            reading[o] += 1
            mma_fifo.append((o, i, b))
            yield

    def epilogue():
        for i in range(groups):
            b, v = i % NB, i // NB
            while not acc_full[b].ready(v & 1):
                yield
            assert acc_full[b].fills[v] == ("acc", i) and acc_of[b] == i
            yield
            epi_reads[i] += 1
            acc_empty[b].arrive()

    def complete_mma():
        o, i, b = mma_fifo.pop(0)
        reading[o] -= 1
        op_empty[o].arrive()
        acc_full[b].arrive(("acc", i))

    alive = ([producer(), mma()] + [expansion() for _ in range(NW)] +
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
    assert epi_reads == [NE] * groups


@pytest.mark.parametrize("groups", [1, 3, 8, 17])
@pytest.mark.parametrize("LS,OS,NB", [(6, 4, 4), (2, 2, 1), (3, 5, 2)])
def test_skinny_protocol_random_schedules(groups, LS, OS, NB):
    for seed in range(4):
        run_skinny_protocol(groups, LS, OS, NB, NW=3, NE=2, seed=seed * 6007 + groups)


def test_skinny_model_catches_missing_op_empty_wait():
    """Planted mistake: the expansion warps write a stage's A without waiting for the MMAs
    that read its previous contents; the model must see A rewritten under a queued MMA."""
    caught = 0
    for seed in range(30):
        try:
            run_skinny_protocol(9, 4, 2, 2, NW=2, NE=1, seed=seed, expansion_waits_op_empty=False)
        except (AssertionError, IndexError, RuntimeError):
            caught += 1
    assert caught > 0
