"""CPU model of the attention kernel's per-CTA barrier protocol: TMA producer, four column-info warps,
the in-order tcgen05 MMA issuer and eight softmax warps (two column halves x four TMEM lane
groups).  Random tile counts, random delays of every asynchronous completion (TMA landings, MMA
completions in issue order) and random rescale decisions are run against invariants:

- no deadlock;
- the K / V^T slot an MMA reads holds the tile the protocol says from the MMA's issue to its
  completion;
- the softmax reads S_u from its buffer and the column info of tile u, and reads its partner half's
  maximum of tile u;
- PV_u reads P_u complete in both halves and before S_{u+2} overwrites the buffer;
- an O rescale runs only after PV_{u-1} has completed and before PV_u is issued;
- the epilogue sees every PV applied.

The model mirrors the kernel's waits one for one (slot and ring indices, phase parities); it
exercises no GPU.  Barrier semantics: a phase completes when its arrival count is
reached; a parity test is true iff the barrier's current phase parity differs from the tested one."""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the phase expects"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


class Violation(AssertionError):
    pass


def check(cond, what):
    if not cond:
        raise Violation(what)


def run(n, nk=3, nv=3, nci=4, seed=0, rescale_p=0.2, swap_order=False, rescale_parity_shift=0,
        producer_skips_empty_wait=False):
    """n tiles, each K and V^T tile filled by one TMA copy.  Returns True when every role finished."""
    rng = random.Random(seed)
    k_full, k_empty = [Bar(1) for _ in range(nk)], [Bar(1) for _ in range(nk)]
    v_full, v_empty = [Bar(1) for _ in range(nv)], [Bar(1) for _ in range(nv)]
    ci_full, ci_empty = [Bar(4) for _ in range(nci)], [Bar(8) for _ in range(nci)]
    s_full, p_full, xm_bar = [Bar(1), Bar(1)], [Bar(8), Bar(8)], [Bar(8), Bar(8)]
    pv_done, o_final = Bar(1), Bar(1)
    kslot, vslot = [None] * nk, [None] * nv          # tile held by each slot
    sbuf = [None, None]                               # ("S", u) or ("P", u, set of (half, group))
    cinfo = [None] * nci
    xm = [[None, None], [None, None]]
    o_applied = [0]                                   # PVs applied to O
    rescale = [rng.random() < rescale_p for _ in range(n)]
    tma_events, mma_fifo = [], []                     # pending asynchronous completions

    # ---- producer (one thread) -------------------------------------------------------------
    def producer():
        for u in range(n):
            sk, sv = u % nk, u % nv
            while not producer_skips_empty_wait and not k_empty[sk].done(((u // nk) & 1) ^ 1):
                yield False
            tma_events.append(("k", sk, u))
            while not v_empty[sv].done(((u // nv) & 1) ^ 1):
                yield False
            tma_events.append(("v", sv, u))
            yield True

    def land(ev):
        kind, s, u = ev
        if kind == "k":
            kslot[s] = u
            k_full[s].arrive()            # the expect_tx arrival completes when the bytes land
        else:
            vslot[s] = u
            v_full[s].arrive()

    # ---- column-info warps -----------------------------------------------------------------
    def colinfo(w):
        for u in range(n):
            ci = u % nci
            while not ci_empty[ci].done(((u // nci) & 1) ^ 1):
                yield False
            cinfo[ci] = u
            ci_full[ci].arrive()
            yield True

    def ready(slot, u):
        return slot == u

    # ---- MMA issuer (one thread; operations complete in issue order) --------------------------
    def mma():
        def issue_s(u):
            sk = u % nk
            while not k_full[sk].done((u // nk) & 1):
                yield False
            check(ready(kslot[sk], u), f"S{u} issued on K slot {kslot[sk]}")
            mma_fifo.append(("S", u))
            yield True

        def issue_pv(v):
            sv = v % nv
            while not p_full[v & 1].done((v >> 1) & 1):
                yield False
            while not v_full[sv].done((v // nv) & 1):
                yield False
            check(ready(vslot[sv], v), f"PV{v} issued on V slot {vslot[sv]}")
            b = sbuf[v & 1]
            check(b is not None and b[0] == "P" and b[1] == v and len(b[2]) == 8, f"PV{v} issued on {b}")
            mma_fifo.append(("PV", v))
            yield True

        for u in range(n):
            if swap_order and u >= 1:
                yield from issue_pv(u - 1)
                yield from issue_s(u)
            else:
                yield from issue_s(u)
                if u >= 1:
                    yield from issue_pv(u - 1)
        if n:
            yield from issue_pv(n - 1)
        mma_fifo.append(("END", n))
        yield True

    def complete(op):
        kind, u = op
        if kind == "S":
            sk = u % nk
            check(ready(kslot[sk], u), f"S{u} completed on K slot {kslot[sk]}")
            b = sbuf[u & 1]
            check(b is None or (b[0] == "P" and o_applied[0] > b[1]), f"S{u} overwrote unread {b}")
            sbuf[u & 1] = ("S", u)
            s_full[u & 1].arrive()
            k_empty[sk].arrive()
        elif kind == "PV":
            sv = u % nv
            check(ready(vslot[sv], u), f"PV{u} completed on V slot {vslot[sv]}")
            b = sbuf[u & 1]
            check(b is not None and b[0] == "P" and b[1] == u and len(b[2]) == 8, f"PV{u} read {b}")
            check(o_applied[0] == u, f"PV{u} applied out of order")
            o_applied[0] = u + 1
            v_empty[sv].arrive()
            pv_done.arrive()
        else:
            o_final.arrive()

    # ---- softmax warps ----------------------------------------------------------------------
    def softmax(half, g):
        for u in range(n):
            ci, b = u % nci, u & 1
            while not ci_full[ci].done((u // nci) & 1):
                yield False
            while not s_full[b].done((u >> 1) & 1):
                yield False
            check(sbuf[b] == ("S", u) or (sbuf[b] and sbuf[b][0] == "P" and sbuf[b][1] == u), f"softmax {u} read {sbuf[b]}")
            check(cinfo[ci] == u, f"softmax {u} read column info of {cinfo[ci]}")
            if g == 0:
                xm[b][half] = u
            xm_bar[b].arrive()
            while not xm_bar[b].done((u >> 1) & 1):
                yield False
            check(xm[b][half ^ 1] == u, f"softmax {u} half {half} read partner max of {xm[b][half ^ 1]}")
            if sbuf[b][0] == "S":
                sbuf[b] = ("P", u, set())
            sbuf[b][2].add((half, g))
            if rescale[u] and u >= 1:
                par = ((u - 1) & 1) ^ rescale_parity_shift
                while not pv_done.done(par):
                    yield False
                check(o_applied[0] == u, f"rescale at {u} with {o_applied[0]} PVs applied")
            ci_empty[ci].arrive()
            p_full[b].arrive()
            yield True
        while not o_final.done(0):
            yield False
        check(o_applied[0] == n, "epilogue before every PV")

    roles = [producer(), mma()] + [colinfo(w) for w in range(4)] + [softmax(h, g) for h in (0, 1) for g in range(4)]
    idle = 0
    while roles:
        # fire some asynchronous completions: TMA landings in any order, MMAs in issue order
        while tma_events and rng.random() < 0.5:
            land(tma_events.pop(rng.randrange(len(tma_events))))
        while mma_fifo and rng.random() < 0.5:
            complete(mma_fifo.pop(0))
        prog = False
        for r in rng.sample(roles, len(roles)):
            try:
                prog |= next(r)
            except StopIteration:
                roles.remove(r)
                prog = True
        idle = 0 if (prog or tma_events or mma_fifo) else idle + 1
        if idle > 50:
            return False
    while mma_fifo:
        complete(mma_fifo.pop(0))
    return True


def _lengths():
    rng = random.Random(11)
    return [0, 1, 2, 3, 7, 40] + [rng.randint(1, 60) for _ in range(40)]


@pytest.mark.parametrize("nk", [3, 6])
def test_protocol_finishes_and_keeps_every_invariant(nk):
    for n in _lengths():
        for seed in range(3):
            assert run(n, nk=nk, nv=nk, seed=seed), (n, seed)


def test_issuing_pv_before_the_next_s_still_holds():
    # the issue order S_u, PV_{u-1} is the kernel's; PV_{u-1}, S_u is also safe (only slower)
    for seed in range(5):
        assert run(24, seed=seed, swap_order=True)


def test_wrong_rescale_parity_is_caught():
    # waiting for the PV completion of the wrong phase either deadlocks or rescales too early
    bad = 0
    for seed in range(20):
        try:
            ok = run(30, seed=seed, rescale_p=0.5, rescale_parity_shift=1)
        except Violation:
            ok = False
        bad += not ok
    assert bad > 0


def test_model_detects_a_slot_reused_too_early():
    # a producer that skips the empty-slot wait overwrites a K tile before its MMA has consumed it
    caught = 0
    for seed in range(10):
        try:
            ok = run(20, nk=2, nv=2, seed=seed, producer_skips_empty_wait=True)
        except AssertionError:
            ok = False
        caught += not ok
    assert caught > 0
