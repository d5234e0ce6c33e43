"""A model of the tensor-core codec kernels' barrier protocols, run on the CPU
over random panel schedules and random completion orders of the asynchronous
work (TMA loads and stores, MMA commits).

Each role of the kernels (TMA producer, converter warps, MMA issuer,
epilogue, store warp) is a coroutine that takes the same waits and arrivals,
in the same order, as its loop in codec_tc.cu.  Barriers model the hardware's
parity waits exactly: a wait on parity P passes whenever the count of
completed phases differs from P in parity.  The checks:

  * every wait passes on the very phase it means (a pass two phases early or
    late is a silent error on the GPU);
  * every reader of a stage or scratch tile sees the step's own data, and no
    TMA load or writer overwrites data that is still being read;
  * the run ends (no deadlock).

The decoder's scratch tiles are shared by first-pass steps (widened codes,
written by the converters) and second-pass steps (output, written by the
epilogue).  Releasing a second-pass stage as soon as its output tile is ready
let the converters, which wait for a tile only in first-pass steps, pass a
tile's wait two phases early; the model finds such a schedule, and the
kernel releases the stage after the tile's stores have read it instead.
"""
import random

import pytest

pytestmark = pytest.mark.filterwarnings("ignore")


class Fail(Exception):
    pass


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


LEAD = 3  # first-pass steps that open a block (kLead in codec_tc.cu)


def steps_of(ncs, lead=LEAD):
    """(pass, block k, block start, index within the pass, steps of the pass)
    of every step of a CTA that owns panels with ncs chunks, in the kernels'
    interleaved order: block k runs the first pass of panel k and the second
    pass of panel k-1, opening with `lead` first-pass steps."""
    out, k = [], 0
    while True:
        n1 = ncs[k] if k < len(ncs) else 0
        n2 = ncs[k - 1] if 1 <= k <= len(ncs) else 0
        if n1 + n2 == 0:
            return out
        i1 = i2 = 0
        while i1 + i2 < n1 + n2:
            second = i2 < n2 and (i1 >= n1 or i1 >= i2 + lead)
            out.append((1 if second else 0, k, i1 + i2 == 0, i2 if second else i1, n2 if second else n1))
            if second:
                i2 += 1
            else:
                i1 += 1
        k += 1


class Sim:
    def __init__(self, rng):
        self.rng, self.B, self.events = rng, {}, []

    def bar(self, name, count=1):
        self.B[name] = Bar(count)

    def wait(self, name, intended):
        b = self.B[name]
        while (b.done & 1) == (intended & 1):
            yield
        if b.done != intended + 1:
            raise Fail(f"{name}: the wait for phase {intended} passed with {b.done} phases complete")

    def later(self, fn):
        self.events.append([self.rng.randint(1, 40), fn])

    def run(self, agents):
        alive, n = dict(agents), 0
        while alive or self.events:
            pick = self.rng.choice(list(alive) + (["ev"] if self.events else []))
            n += 1
            if n > 3_000_000:
                raise Fail(f"no progress: {sorted(alive)} still running")
            if pick == "ev":
                e = self.rng.choice(self.events)
                e[0] -= 1
                if e[0] <= 0:
                    self.events.remove(e)
                    e[1]()
                continue
            try:
                next(alive[pick])
            except StopIteration:
                del alive[pick]


def decoder(ncs, rng, release_at_readiness=False, presplit=False, n_stages=4):
    """The decoder: D2 (first pass) and D3 (second pass), four stages, two
    scratch tiles taken as j = step & 1, two TMEM buffers per kind."""
    seq, sim = steps_of(ncs), Sim(rng)
    N = len(seq)
    for s in range(n_stages):
        for b in ("full", "cfull", "empty"):
            sim.bar(f"{b}{s}")
    for j in range(2):
        for b in ("sfree", "oready", "tfull", "tempty", "wfull", "wempty"):
            sim.bar(f"{b}{j}")
    sim.bar("pcfull")
    B = sim.B
    stage, stage_rd = [None] * n_stages, [0] * n_stages
    tile, tile_rd = [None] * 2, [0] * 2

    def producer():
        for x in range(N):
            s = x % n_stages
            if x >= n_stages:
                yield from sim.wait(f"empty{s}", x // n_stages - 1)

            def land(x=x, s=s):
                if stage_rd[s]:
                    raise Fail(f"a TMA load overwrote stage {s} while it was read")
                stage[s] = x
                B[f"cfull{s}"].arrive()
            sim.later(land)
            yield

    def converters():
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s, j = x % n_stages, x & 1
            yield from sim.wait(f"cfull{s}", x // n_stages)
            if ps == 0 and x >= 2:
                yield from sim.wait(f"sfree{j}", (x >> 1) - 1)
            if stage[s] != x:
                raise Fail(f"converters read stage {s} holding step {stage[s]} at step {x}")
            if ps == 0:
                if tile_rd[j]:
                    raise Fail(f"converters overwrote tile {j} while it was read")
                tile[j] = ("wide", x)
            yield
            B[f"full{s}"].arrive()

    def mma():
        e2 = d2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s, j = x % n_stages, x & 1
            if ps == 1 and i == 0:
                yield from sim.wait("pcfull", k - 1)
            yield from sim.wait(f"full{s}", x // n_stages)
            if ps == 0:
                b = d2 & 1
                if d2 >= 2:
                    yield from sim.wait(f"tempty{b}", (d2 >> 1) - 1)
                if tile[j] != ("wide", x):
                    raise Fail(f"D2 read tile {j} holding {tile[j]} at step {x}")
                stage_rd[s] += 1
                tile_rd[j] += 1

                def done(x=x, s=s, j=j, b=b):
                    if stage[s] != x or tile[j] != ("wide", x):
                        raise Fail("a D2 operand changed under the MMA")
                    stage_rd[s] -= 1
                    tile_rd[j] -= 1
                    for name in (f"empty{s}", f"sfree{j}", f"tfull{b}"):
                        B[name].arrive()
                sim.later(done)
                d2 += 1
            else:
                b = e2 & 1
                if e2 >= 2:
                    yield from sim.wait(f"wempty{b}", (e2 >> 1) - 1)
                stage_rd[s] += 1

                def done(x=x, s=s, b=b):
                    if stage[s] != x:
                        raise Fail("a D3 operand changed under the MMA")
                    stage_rd[s] -= 1
                    B[f"wfull{b}"].arrive()
                sim.later(done)
                e2 += 1
            yield

    def epilogue():
        e2 = d2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s, j = x % n_stages, x & 1
            if bs and k >= 1:
                B["pcfull"].arrive()
            if ps == 0:
                b = d2 & 1
                yield from sim.wait(f"tfull{b}", d2 >> 1)
                yield
                B[f"tempty{b}"].arrive()
                d2 += 1
                continue
            b = e2 & 1
            yield from sim.wait(f"wfull{b}", e2 >> 1)
            yield from sim.wait(f"cfull{s}", x // n_stages)
            if x >= 2:
                yield from sim.wait(f"sfree{j}", (x >> 1) - 1)
            if stage[s] != x:
                raise Fail(f"the epilogue read codes of step {stage[s]} at step {x}")
            stage_rd[s] += 1
            yield
            stage_rd[s] -= 1
            if tile_rd[j]:
                raise Fail(f"the epilogue overwrote tile {j} while it was read")
            tile[j] = ("out", x)
            B[f"wempty{b}"].arrive()
            B[f"oready{j}"].arrive()
            e2 += 1

    def store():
        par = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            if ps == 0:
                continue
            s, j = x % n_stages, x & 1
            b = B[f"oready{j}"]
            while (b.done & 1) == ((par >> j) & 1):
                yield
            if release_at_readiness:
                B[f"empty{s}"].arrive()
            if tile[j] != ("out", x):
                raise Fail(f"the store read tile {j} holding {tile[j]} at step {x}")
            tile_rd[j] += 1
            read = []

            def rd(x=x, j=j):
                if tile[j] != ("out", x):
                    raise Fail("a tile changed under its store")
                tile_rd[j] -= 1
                read.append(1)
            sim.later(rd)
            while not read:
                yield
            par ^= 1 << j
            if not release_at_readiness:
                B[f"empty{s}"].arrive()
            B[f"sfree{j}"].arrive()

    sim.run({"producer": producer(), "converters": converters(), "mma": mma(), "epilogue": epilogue(),
             "store": store()})


def encoder(ncs, rng, presplit=False, n_stages=3):
    """The encoder: E1 (first pass) accumulates P over a panel, E2 (second
    pass) forms W' per chunk; three stages, two TMEM W buffers, two codes tiles."""
    seq, sim = steps_of(ncs), Sim(rng)
    N = len(seq)
    for s in range(n_stages):
        for b in ("full", "tfull", "empty"):
            sim.bar(f"{b}{s}")
    for j in range(2):
        for b in ("wfull", "wempty", "cready", "cfree"):
            sim.bar(f"{b}{j}")
    sim.bar("pfull0")
    sim.bar("pfull1")
    sim.bar("pcfull")
    B = sim.B
    stage, stage_rd = [None] * n_stages, [0] * n_stages
    ctile = [None] * 2
    P = [None, None]  # the panel whose P each TMEM slot holds (or is being written)

    def producer():
        for x in range(N):
            s = x % n_stages
            if x >= n_stages:
                yield from sim.wait(f"empty{s}", x // n_stages - 1)

            def land(x=x, s=s):
                if stage_rd[s]:
                    raise Fail(f"a TMA load overwrote stage {s} while it was read")
                stage[s] = x
                B[f"tfull{s}"].arrive()
            sim.later(land)
            yield

    def converters():
        if presplit:
            return
        for x in range(N):
            s = x % n_stages
            yield from sim.wait(f"tfull{s}", x // n_stages)
            if stage[s] != x:
                raise Fail(f"converters read stage {s} holding step {stage[s]} at step {x}")
            yield
            B[f"full{s}"].arrive()

    def mma():
        e2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s = x % n_stages
            if ps == 1 and i == 0:
                yield from sim.wait("pcfull", k - 1)
            yield from sim.wait(f"{'tfull' if presplit else 'full'}{s}", x // n_stages)
            stage_rd[s] += 1
            if ps == 0:
                last = i == n - 1
                if i == 0:
                    P[k & 1] = k  # E1 of panel k starts overwriting its slot

                def done(x=x, s=s, last=last, k=k):
                    if stage[s] != x:
                        raise Fail("an E1 operand changed under the MMA")
                    stage_rd[s] -= 1
                    B[f"empty{s}"].arrive()
                    if last:
                        B[f"pfull{k & 1}"].arrive()
                sim.later(done)
            else:
                b = e2 & 1
                if e2 >= 2:
                    yield from sim.wait(f"wempty{b}", (e2 >> 1) - 1)

                def done(x=x, s=s, b=b):
                    if stage[s] != x:
                        raise Fail("an E2 operand changed under the MMA")
                    stage_rd[s] -= 1
                    B[f"empty{s}"].arrive()
                    B[f"wfull{b}"].arrive()
                sim.later(done)
                e2 += 1
            yield

    def epilogue():
        e2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            if ps == 0:
                continue
            if i == 0:
                yield from sim.wait(f"pfull{(k - 1) & 1}", (k - 1) >> 1)
                if P[(k - 1) & 1] != k - 1:
                    raise Fail(f"the epilogue read P of panel {P[(k - 1) & 1]} for panel {k - 1}")
                yield
                B["pcfull"].arrive()
            b, cb = e2 & 1, e2 & 1
            yield from sim.wait(f"wfull{b}", e2 >> 1)
            yield
            B[f"wempty{b}"].arrive()
            if e2 >= 2:
                yield from sim.wait(f"cfree{cb}", (e2 >> 1) - 1)
            ctile[cb] = x
            B[f"cready{cb}"].arrive()
            e2 += 1

    def store():
        e2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            if ps == 0:
                continue
            cb = e2 & 1
            yield from sim.wait(f"cready{cb}", e2 >> 1)
            if ctile[cb] != x:
                raise Fail(f"the store read codes tile {cb} holding {ctile[cb]} at step {x}")
            read = []
            sim.later(lambda: read.append(1))
            while not read:
                yield
            B[f"cfree{cb}"].arrive()
            e2 += 1

    sim.run({"producer": producer(), "converters": converters(), "mma": mma(), "epilogue": epilogue(),
             "store": store()})


def _schedules(seed, n):
    rng = random.Random(seed)
    for _ in range(n):
        # panels of mixed lengths, as the longest-first schedule of a grouped
        # launch over 32-chunk (d_in 4096) and 12-chunk (d_in 1536) layers gives
        yield [rng.choice([1, 2, 3, 5, 12, 32]) for _ in range(rng.randint(1, 5))], rng


@pytest.mark.parametrize("presplit", [False, True])
def test_decoder_protocol_holds_on_random_schedules(presplit):
    for ncs, rng in _schedules(11 + presplit, 150):
        decoder(ncs, rng, presplit=presplit)


@pytest.mark.parametrize("presplit", [False, True])
def test_encoder_protocol_holds_on_random_schedules(presplit):
    for ncs, rng in _schedules(21 + presplit, 150):
        encoder(ncs, rng, presplit=presplit)


def test_releasing_a_second_pass_stage_at_tile_readiness_is_caught():
    """The earlier decoder released a second-pass stage as soon as its output
    tile was ready; the model finds a schedule where that breaks."""
    with pytest.raises(Fail):
        for ncs, rng in _schedules(3, 400):
            decoder(ncs, rng, release_at_readiness=True)
