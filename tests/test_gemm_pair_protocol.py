"""CPU model of the barrier protocol of the paired-SM GEMM (gemm2_bf16_kernel): a TMA producer in each
CTA of the pair, the MMA issuer of the even CTA, and four epilogue warps in each CTA.  Random tile and
K-step counts and random delays of every asynchronous completion (each CTA's copies land in any order;
MMAs complete in issue order; commits arrive on both CTAs' barriers) are run against invariants:

- no deadlock;
- an MMA reads a stage only when both CTAs' halves of it hold the K step the protocol says, and no copy
  overwrites a stage before the MMAs reading it have completed;
- the epilogue of a CTA reads an accumulator only after its tile's last MMA has completed, and the MMA
  issuer starts a tile in an accumulator only after all eight epilogue warps have read the tile before.

Barrier semantics as in the kernel: a phase completes when its arrival count and its transaction bytes
are both reached (bytes may land before the expected count is posted); a parity test is true iff the
barrier's current phase parity differs from the tested one.  The model exercises no GPU."""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def _maybe_flip(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the phase expects"
        self.tx += expect_tx
        self._maybe_flip()

    def complete_tx(self, n):
        self.tx -= n
        self._maybe_flip()

    def done(self, parity):
        return (self.phase & 1) != parity


class Violation(AssertionError):
    pass


def check(cond, what):
    if not cond:
        raise Violation(what)


def run(n_tiles, k_iters, stages=6, seed=0, even_skips_expect=False, odd_skips_empty_wait=False):
    rng = random.Random(seed)
    cta = [dict(full=[Bar(1) for _ in range(stages)], empty=[Bar(1) for _ in range(stages)],
                acc_full=[Bar(1), Bar(1)], acc_empty=[Bar(8), Bar(8)], stage=[None] * stages,
                acc=[None, None]) for _ in range(2)]
    even = cta[0]
    copies, mma_fifo = [], []
    read = {}                                          # (tile, buf) -> set of (cta, warp) that read it

    def producer(r):
        c = cta[r]
        s = ph = 0
        for t in range(n_tiles):
            for kb in range(k_iters):
                while not (odd_skips_empty_wait and r == 1) and not c["empty"][s].done(ph ^ 1):
                    yield False
                if r == 0 and not even_skips_expect:
                    even["full"][s].arrive(expect_tx=2)    # both CTAs' bytes (one unit each here)
                copies.append((r, s, (t, kb)))
                s += 1
                if s == stages:
                    s, ph = 0, ph ^ 1
                yield True

    def land(ev):
        r, s, what = ev
        c = cta[r]
        check(c["stage"][s] is None or c["stage"][s][1] == "read", f"copy into CTA {r} stage {s} overwrote {c['stage'][s]}")
        c["stage"][s] = (what, "landed")
        even["full"][s].complete_tx(1)

    def mma():
        s = ph = 0
        for t in range(n_tiles):
            buf = t & 1
            while not even["acc_empty"][buf].done(((t >> 1) & 1) ^ 1):
                yield False
            if t >= 2:
                check(len(read.get((t - 2, buf), ())) == 8, f"tile {t} reuses accumulator {buf} before tile {t - 2} was read")
            for kb in range(k_iters):
                while not even["full"][s].done(ph):
                    yield False
                for r in (0, 1):
                    check(cta[r]["stage"][s] == ((t, kb), "landed"), f"MMA {t},{kb} on CTA {r} stage {cta[r]['stage'][s]}")
                mma_fifo.append(("mma", s, (t, kb)))
                mma_fifo.append(("commit_empty", s, None))
                s += 1
                if s == stages:
                    s, ph = 0, ph ^ 1
                yield True
            mma_fifo.append(("commit_acc", buf, t))
        yield True

    def complete(op):
        kind, a, b = op
        if kind == "mma":
            for r in (0, 1):
                check(cta[r]["stage"][a] == (b, "landed"), f"MMA {b} completed on CTA {r} stage {cta[r]['stage'][a]}")
                cta[r]["stage"][a] = (b, "consumed")
        elif kind == "commit_empty":
            for r in (0, 1):                             # multicast to both CTAs
                what = cta[r]["stage"][a][0]
                cta[r]["stage"][a] = (what, "read")
                cta[r]["empty"][a].arrive()
        else:
            for r in (0, 1):
                cta[r]["acc"][a] = b
                cta[r]["acc_full"][a].arrive()

    def epilogue(r, w):
        c = cta[r]
        for t in range(n_tiles):
            buf = t & 1
            while not c["acc_full"][buf].done((t >> 1) & 1):
                yield False
            check(c["acc"][buf] == t, f"CTA {r} epilogue of tile {t} read accumulator holding {c['acc'][buf]}")
            read.setdefault((t, buf), set()).add((r, w))
            even["acc_empty"][buf].arrive()              # remote arrive for the odd CTA
            yield True

    roles = [producer(0), producer(1), mma()] + [epilogue(r, w) for r in (0, 1) for w in range(4)]
    idle = 0
    while roles:
        while copies and rng.random() < 0.5:
            land(copies.pop(rng.randrange(len(copies))))
        while mma_fifo and rng.random() < 0.5:
            complete(mma_fifo.pop(0))
        prog = False
        for role in rng.sample(roles, len(roles)):
            try:
                prog |= next(role)
            except StopIteration:
                roles.remove(role)
                prog = True
        idle = 0 if (prog or copies or mma_fifo) else idle + 1
        if idle > 50:
            return False
    while mma_fifo:
        complete(mma_fifo.pop(0))
    check(all(len(read.get((t, t & 1), ())) == 8 for t in range(n_tiles)), "a tile was not read by every epilogue warp")
    return True


@pytest.mark.parametrize("stages", [6, 2])
def test_pair_protocol_finishes_and_keeps_every_invariant(stages):
    rng = random.Random(3)
    for trial in range(40):
        n_tiles, k_iters = rng.randint(0, 7), rng.randint(1, 9)
        assert run(n_tiles, k_iters, stages=stages, seed=trial), (n_tiles, k_iters)


def test_missing_expected_bytes_are_caught():
    # without the even CTA's expect_tx arrival the stage never completes: the model must stall
    assert not run(3, 4, seed=1, even_skips_expect=True)


def test_odd_producer_skipping_its_empty_wait_is_caught():
    # the odd CTA reusing a stage before the even CTA's MMAs released it must be noticed
    caught = 0
    for seed in range(10):
        try:
            ok = run(4, 6, stages=2, seed=seed, odd_skips_empty_wait=True)
        except AssertionError:
            ok = False
        caught += not ok
    assert caught > 0
