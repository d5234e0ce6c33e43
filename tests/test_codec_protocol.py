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
  * every reader of a stage or tile sees the step's own data, and no TMA load
    or writer overwrites data that is still being read;
  * the run ends (no deadlock).

In the decoder, the converters write a first-pass step's widened codes into
one of two TMEM A tiles, and the epilogue writes a second-pass step's output
into shared-memory output tiles; each tile has one writer role and one
reader role.  A second-pass stage is released by the epilogue once it has
read the codes; the model catches a release at D3's completion instead,
where the stage's next TMA load can overwrite codes not yet read.  (An
earlier layout shared two scratch tiles between the converters and the
epilogue; there the model found that releasing a second-pass stage as soon
as its output tile was ready let the converters pass a tile's parity wait
two phases early.)
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


def decoder(ncs, rng, n_stages=4, n_out=2, release_at_mma=False):
    """The decoder: D2 (first pass) and D3 (second pass).  The converters widen
    a first-pass step's codes into one of two TMEM A tiles (their own, freed by
    the MMA commit); the epilogue writes a second-pass step's output into one of
    `n_out` shared-memory tiles (freed once the TMA stores have read them) and
    releases the step's stage as soon as it has read the codes."""
    seq, sim = steps_of(ncs), Sim(rng)
    N = len(seq)
    for s in range(n_stages):
        for b in ("full", "cfull", "empty"):
            sim.bar(f"{b}{s}")
    for j in range(2):
        for b in ("afree", "tfull", "tempty", "wfull", "wempty"):
            sim.bar(f"{b}{j}")
    for o in range(n_out):
        sim.bar(f"ofree{o}")
        sim.bar(f"oready{o}")
    sim.bar("pcfull")
    B = sim.B
    stage, stage_rd = [None] * n_stages, [0] * n_stages
    atile, atile_rd = [None] * 2, [0] * 2
    otile, otile_rd = [None] * n_out, [0] * n_out
    pc, pc_rd = [None], [0]

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
        d2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s = x % n_stages
            yield from sim.wait(f"cfull{s}", x // n_stages)
            if stage[s] != x:
                raise Fail(f"converters took stage {s} holding step {stage[s]} at step {x}")
            if ps == 0:
                a = d2 & 1
                if d2 >= 2:
                    yield from sim.wait(f"afree{a}", (d2 >> 1) - 1)
                stage_rd[s] += 1
                yield
                stage_rd[s] -= 1
                if atile_rd[a]:
                    raise Fail(f"converters overwrote A tile {a} while the MMA read it")
                atile[a] = x
                d2 += 1
            yield
            B[f"full{s}"].arrive()

    def mma():
        e2 = d2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s = x % n_stages
            if ps == 1 and i == 0:
                yield from sim.wait("pcfull", k - 1)
            yield from sim.wait(f"full{s}", x // n_stages)
            if ps == 0:
                b = a = d2 & 1
                if d2 >= 2:
                    yield from sim.wait(f"tempty{b}", (d2 >> 1) - 1)
                if atile[a] != x:
                    raise Fail(f"D2 read A tile {a} holding {atile[a]} at step {x}")
                stage_rd[s] += 1
                atile_rd[a] += 1

                def done(x=x, s=s, a=a, b=b):
                    if stage[s] != x or atile[a] != x:
                        raise Fail("a D2 operand changed under the MMA")
                    stage_rd[s] -= 1
                    atile_rd[a] -= 1
                    for name in (f"empty{s}", f"afree{a}", f"tfull{b}"):
                        B[name].arrive()
                sim.later(done)
                d2 += 1
            else:
                b = e2 & 1
                if e2 >= 2:
                    yield from sim.wait(f"wempty{b}", (e2 >> 1) - 1)
                if pc[0] != k - 1:
                    raise Fail(f"D3 of panel {k - 1} read P o c of panel {pc[0]}")
                stage_rd[s] += 1
                pc_rd[0] += 1

                def done(x=x, s=s, b=b, k=k):
                    if stage[s] != x or pc[0] != k - 1:
                        raise Fail("a D3 operand changed under the MMA")
                    stage_rd[s] -= 1
                    pc_rd[0] -= 1
                    B[f"wfull{b}"].arrive()
                    if release_at_mma:
                        B[f"empty{s}"].arrive()
                sim.later(done)
                e2 += 1
            yield

    def epilogue():
        e2 = d2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            s = x % n_stages
            if bs and k >= 1:
                if pc_rd[0]:
                    raise Fail("the epilogue overwrote P o c while D3 read it")
                pc[0] = k - 1
                B["pcfull"].arrive()
            if ps == 0:
                b = d2 & 1
                yield from sim.wait(f"tfull{b}", d2 >> 1)
                yield
                B[f"tempty{b}"].arrive()
                d2 += 1
                continue
            b, o = e2 & 1, e2 % n_out
            yield from sim.wait(f"wfull{b}", e2 >> 1)
            yield from sim.wait(f"cfull{s}", x // n_stages)
            if e2 >= n_out:
                yield from sim.wait(f"ofree{o}", e2 // n_out - 1)
            if stage[s] != x:
                raise Fail(f"the epilogue read codes of step {stage[s]} at step {x}")
            stage_rd[s] += 1
            yield
            if stage[s] != x:
                raise Fail(f"the codes of step {x} changed while the epilogue read them")
            stage_rd[s] -= 1
            if not release_at_mma:
                B[f"empty{s}"].arrive()
            yield
            if otile_rd[o]:
                raise Fail(f"the epilogue overwrote output tile {o} while it was stored")
            otile[o] = x
            B[f"wempty{b}"].arrive()
            B[f"oready{o}"].arrive()
            e2 += 1

    def store():
        e2 = 0
        for x, (ps, k, bs, i, n) in enumerate(seq):
            if ps == 0:
                continue
            o = e2 % n_out
            yield from sim.wait(f"oready{o}", e2 // n_out)
            if otile[o] != x:
                raise Fail(f"the store read output tile {o} holding {otile[o]} at step {x}")
            otile_rd[o] += 1
            read = []

            def rd(x=x, o=o):
                if otile[o] != x:
                    raise Fail("a tile changed under its store")
                otile_rd[o] -= 1
                read.append(1)
            sim.later(rd)
            while not read:
                yield
            B[f"ofree{o}"].arrive()
            e2 += 1

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


@pytest.mark.parametrize("n_stages,n_out", [(4, 2), (5, 1)])
def test_decoder_protocol_holds_on_random_schedules(n_stages, n_out):
    for ncs, rng in _schedules(11 + n_stages, 150):
        decoder(ncs, rng, n_stages=n_stages, n_out=n_out)


@pytest.mark.parametrize("presplit", [False, True])
def test_encoder_protocol_holds_on_random_schedules(presplit):
    for ncs, rng in _schedules(21 + presplit, 150):
        encoder(ncs, rng, presplit=presplit)


def test_releasing_a_second_pass_stage_at_mma_completion_is_caught():
    """A second-pass stage still holds the codes that the epilogue adds to the
    product: released when the MMA completes, its next TMA load can overwrite
    them before they are read.  The model finds such a schedule."""
    with pytest.raises(Fail):
        for ncs, rng in _schedules(3, 400):
            decoder(ncs, rng, release_at_mma=True)
