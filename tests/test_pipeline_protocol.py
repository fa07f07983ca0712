"""CPU model of the attention kernel's per-CTA barrier protocol: TMA producer, two column-info warps,
the in-order tcgen05 MMA issuer and two softmax warpgroups of four warps (TMEM lane groups), the
first taking the even-numbered tiles and the second the odd-numbered ones.  Random tile counts,
random delays of every asynchronous completion (TMA landings, MMA completions in issue order) and
random rescale decisions are run against invariants:

- no deadlock;
- the K / V^T slot an MMA reads holds the tile the protocol says from the MMA's issue to its
  completion;
- the softmax of tile u reads S_u from its buffer and the column info of tile u;
- the running offset a warpgroup starts tile u from is the one settled after tile u - 1 by the
  other warpgroup (the decision chain), never an older or a newer one;
- PV_u reads P_u complete (all four warps of its warpgroup) and before S_{u+2} overwrites the buffer;
- an O rescale runs only after PV_{u-1} has completed and before PV_u is issued;
- the epilogue sees every PV applied and both warpgroups' final row sums.

The model mirrors the kernel's waits one for one (slot and ring indices, phase parities); it
exercises no GPU.  Barrier semantics: a phase completes when its arrival count is reached; a parity
test is true iff the barrier's current phase parity differs from the tested one."""
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
        producer_skips_empty_wait=False, dec_parity_shift=0, dec_skips_wait=False):
    """n tiles, each K and V^T tile filled by one TMA copy.  Returns True when every role finished."""
    rng = random.Random(seed)
    k_full, k_empty = [Bar(1) for _ in range(nk)], [Bar(1) for _ in range(nk)]
    v_full, v_empty = [Bar(1) for _ in range(nv)], [Bar(1) for _ in range(nv)]
    ci_full, ci_empty = [Bar(2) for _ in range(nci)], [Bar(4) for _ in range(nci)]
    s_full, p_full, dec_full = [Bar(1), Bar(1)], [Bar(4), Bar(4)], [Bar(4), Bar(4)]
    pv_done, o_final, xl_bar = Bar(1), Bar(1), Bar(8)
    kslot, vslot = [None] * nk, [None] * nv          # tile held by each slot
    sbuf = [None, None]                               # ("S", u) or ("P", u, set of lane groups)
    cinfo = [[None, None] for _ in range(nci)]        # tile whose columns each column-info warp wrote
    sdec = [None] * 4                                 # per lane group: tile whose decision is stored
    xl = [[None] * 4, [None] * 4]                     # per warpgroup and lane group: final row sums posted
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

    # ---- column-info warps (each writes its half of every tile's columns) ----------------------
    def colinfo(w):
        for u in range(n):
            ci = u % nci
            while not ci_empty[ci].done(((u // nci) & 1) ^ 1):
                yield False
            cinfo[ci][w] = u
            ci_full[ci].arrive()
            yield True

    # ---- MMA issuer (one thread; operations complete in issue order) --------------------------
    def mma():
        def issue_s(u):
            sk = u % nk
            while not k_full[sk].done((u // nk) & 1):
                yield False
            check(kslot[sk] == u, f"S{u} issued on K slot {kslot[sk]}")
            mma_fifo.append(("S", u))
            yield True

        def issue_pv(v):
            sv = v % nv
            while not p_full[v & 1].done((v >> 1) & 1):
                yield False
            while not v_full[sv].done((v // nv) & 1):
                yield False
            check(vslot[sv] == v, f"PV{v} issued on V slot {vslot[sv]}")
            b = sbuf[v & 1]
            check(b is not None and b[0] == "P" and b[1] == v and len(b[2]) == 4, f"PV{v} issued on {b}")
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
            check(kslot[sk] == u, f"S{u} completed on K slot {kslot[sk]}")
            b = sbuf[u & 1]
            check(b is None or (b[0] == "P" and o_applied[0] > b[1]), f"S{u} overwrote unread {b}")
            sbuf[u & 1] = ("S", u)
            s_full[u & 1].arrive()
            k_empty[sk].arrive()
        elif kind == "PV":
            sv = u % nv
            check(vslot[sv] == u, f"PV{u} completed on V slot {vslot[sv]}")
            b = sbuf[u & 1]
            check(b is not None and b[0] == "P" and b[1] == u and len(b[2]) == 4, f"PV{u} read {b}")
            check(o_applied[0] == u, f"PV{u} applied out of order")
            o_applied[0] = u + 1
            v_empty[sv].arrive()
            pv_done.arrive()
        else:
            o_final.arrive()

    # ---- softmax warps: warpgroup wg takes tiles u with u % 2 == wg ---------------------------
    def softmax(wg, g):
        for u in range(n):
            if u % 2 != wg:
                continue
            ci, b = u % nci, u & 1
            while not ci_full[ci].done((u // nci) & 1):
                yield False
            while not s_full[b].done((u >> 1) & 1):
                yield False
            check(sbuf[b] == ("S", u) or (sbuf[b] and sbuf[b][0] == "P" and sbuf[b][1] == u),
                  f"softmax {u} read {sbuf[b]}")
            check(cinfo[ci] == [u, u], f"softmax {u} read column info of {cinfo[ci]}")
            yield True                                # scale, mask and the tile maximum happen here
            if u > 0:
                par = (((u - 1) >> 1) & 1) ^ dec_parity_shift
                while not dec_skips_wait and not dec_full[wg ^ 1].done(par):
                    yield False
                check(sdec[g] == u - 1, f"tile {u} started from the decision of tile {sdec[g]}")
            sdec[g] = u
            dec_full[wg].arrive()
            yield True                                # exponentials, P written
            if sbuf[b][0] == "S":
                sbuf[b] = ("P", u, set())
            sbuf[b][2].add(g)
            ci_empty[ci].arrive()
            if rescale[u] and u >= 1:
                par = ((u - 1) & 1) ^ rescale_parity_shift
                while not pv_done.done(par):
                    yield False
                check(o_applied[0] == u, f"rescale at {u} with {o_applied[0]} PVs applied")
            p_full[b].arrive()
            yield True
        while not o_final.done(0):
            yield False
        check(o_applied[0] == n, "epilogue before every PV")
        xl[wg][g] = True
        xl_bar.arrive()
        while not xl_bar.done(0):
            yield False
        check(xl[wg ^ 1][g], "epilogue read the other warpgroup's row sum before it was posted")

    roles = [producer(), mma()] + [colinfo(w) for w in range(2)] + [softmax(w, g) for w in (0, 1) for g in range(4)]
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
    return [0, 1, 2, 3, 4, 5, 7, 40] + [rng.randint(1, 60) for _ in range(40)]


@pytest.mark.parametrize("nk", [3, 6])
def test_protocol_finishes_and_keeps_every_invariant(nk):
    for n in _lengths():
        for seed in range(3):
            assert run(n, nk=nk, nv=nk, seed=seed), (n, seed)


def test_issuing_pv_before_the_next_s_still_holds():
    # the issue order S_u, PV_{u-1} is the kernel's; PV_{u-1}, S_u is also safe (only slower)
    for seed in range(5):
        assert run(24, seed=seed, swap_order=True)


def _caught(**kw):
    bad = 0
    for seed in range(20):
        try:
            ok = run(30, seed=seed, **kw)
        except AssertionError:
            ok = False
        bad += not ok
    return bad


def test_wrong_rescale_parity_is_caught():
    # waiting for the PV completion of the wrong phase either deadlocks or rescales too early
    assert _caught(rescale_p=0.5, rescale_parity_shift=1) > 0


def test_wrong_decision_parity_or_a_skipped_decision_wait_is_caught():
    # starting a tile from a decision of the wrong phase, or without waiting for it at all, reads an
    # offset that is not the previous tile's
    assert _caught(dec_parity_shift=1) > 0
    assert _caught(dec_skips_wait=True) > 0


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
