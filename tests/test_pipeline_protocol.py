"""CPU model of the attention kernel's per-CTA barrier protocol (loader, MMA issuer, two softmax
warpgroups) run over dense and sparse tile-use patterns.  It checks that the protocol cannot deadlock
and that every MMA reads the tile the loader last put in its slot, under random orders of
asynchronous completion.  The model mirrors the kernel's waits one for one (slot/ring indices, use
counts and parities); it exercises no GPU.

Barrier semantics modelled: a phase completes when its arrival count is reached; a parity test is
true iff the barrier's current phase parity differs from the tested parity (so a barrier that ran two
phases ahead is indistinguishable from one that did not -- the reason the MMA issuer guards each slot
test with its own count of released uses)."""
import random

import pytest

USE0, USE1 = 4, 8


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


def run(flags, ns=4, nci=4, seed=0, guard=True):
    """Returns (finished, stale_reads)."""
    n = len(flags)
    uses = lambda j, q: bool(flags[j] & (USE1 if q else USE0))
    kv_full = [Bar(1) for _ in range(ns)]
    kv_empty = [Bar(1) for _ in range(ns)]
    ci_full = [Bar(1) for _ in range(nci)]
    ci_empty = [Bar(8) for _ in range(nci)]
    s_full, p_full = [Bar(1), Bar(1)], [Bar(4), Bar(4)]
    commits, slot, stale = [], [None] * ns, []
    rng = random.Random(seed)

    def loader():
        for j in range(n):
            ci, sk, sv = j % nci, (2 * j) % ns, (2 * j + 1) % ns
            while not ci_empty[ci].done(((j // nci) & 1) ^ 1):
                yield False
            while not kv_empty[sk].done((((2 * j) // ns) & 1) ^ 1):
                yield False
            slot[sk] = ("K", j)
            ci_full[ci].arrive()
            kv_full[sk].arrive()
            yield True
            while not kv_empty[sv].done((((2 * j + 1) // ns) & 1) ^ 1):
                yield False
            slot[sv] = ("V", j)
            kv_full[sv].arrive()
            yield True

    def adv(j, q):
        while j < n and not uses(j, q):
            j += 1
        return j

    def mma():
        nxt, pend, last_s, last_pv, pc, rel = [adv(0, 0), adv(0, 1)], [-1, -1], [-1, -1], [-1, -1], [0, 0], [0] * ns
        while nxt[0] < n or nxt[1] < n or pend[0] >= 0 or pend[1] >= 0:
            prog = False
            for q in (0, 1):
                o = 1 - q
                if pend[q] >= 0:
                    j = pend[q]
                    sv, u = (2 * j + 1) % ns, (2 * j + 1) // ns
                    if (not guard or rel[sv] == u) and p_full[q].done(pc[q] & 1) and kv_full[sv].done(u & 1):
                        if slot[sv] != ("V", j):
                            stale.append(("V", j))
                        pc[q] += 1
                        last_pv[q] = j
                        if not uses(j, o) or last_pv[o] >= j:
                            commits.append(kv_empty[sv])
                            rel[sv] = u + 1
                        pend[q] = -1
                        prog = True
                if pend[q] < 0 and nxt[q] < n:
                    j = nxt[q]
                    sk, u = (2 * j) % ns, (2 * j) // ns
                    if (not guard or rel[sk] == u) and kv_full[sk].done(u & 1):
                        if slot[sk] != ("K", j):
                            stale.append(("K", j))
                        commits.append(s_full[q])
                        last_s[q] = j
                        if not uses(j, o) or last_s[o] >= j:
                            commits.append(kv_empty[sk])
                            rel[sk] = u + 1
                        pend[q] = j
                        nxt[q] = adv(j + 1, q)
                        prog = True
            yield prog

    def softmax(q):
        k = 0
        for j in range(n):
            ci = j % nci
            while not ci_full[ci].done((j // nci) & 1):
                yield False
            if uses(j, q):
                while not s_full[q].done(k & 1):
                    yield False
                p_full[q].arrive(4)
                k += 1
            ci_empty[ci].arrive(4)
            yield True

    roles = [loader(), mma(), softmax(0), softmax(1)]
    idle = 0
    while roles:
        while commits and rng.random() < 0.6:
            commits.pop(0).arrive()
        prog = False
        for r in list(roles):
            try:
                prog |= next(r)
            except StopIteration:
                roles.remove(r)
                prog = True
        idle = 0 if (prog or commits) else idle + 1
        if idle > 20 or stale:
            return False, stale
    return True, stale


def _patterns():
    rng = random.Random(11)
    pats = [[USE0 | USE1] * 40, [USE0] * 30, [USE0, USE1] * 20]
    for _ in range(60):
        n = rng.randint(1, 80)
        p0 = rng.random()
        pats.append([rng.choice([USE0, USE1, USE0 | USE1]) if rng.random() < p0 else USE0 | USE1 for _ in range(n)])
    # long one-sided runs: query tile 0 jumps far ahead of query tile 1
    pats.append([USE0 | USE1] + [USE1] * 50 + [USE0] + [USE1] * 7 + [USE0 | USE1])
    pats.append([USE0] * 3 + [USE1] * 40 + [USE0] * 3)
    return pats


@pytest.mark.parametrize("ns", [4, 8])
def test_protocol_never_deadlocks_or_reads_stale_slots(ns):
    for i, pat in enumerate(_patterns()):
        for seed in range(3):
            ok, stale = run(pat, ns=ns, seed=seed)
            assert ok and not stale, (i, pat, stale)


def test_unguarded_slot_test_reads_stale_data():
    # Without the per-slot release count, a query tile that looks several tiles ahead tests a slot
    # barrier two phases early and issues an MMA on the previous occupant of the slot.
    pat = [USE0 | USE1] + [USE1] * 50 + [USE0] + [USE1] * 7 + [USE0 | USE1]
    results = [run(pat, seed=s, guard=False) for s in range(5)]
    assert any(stale for _, stale in results)
