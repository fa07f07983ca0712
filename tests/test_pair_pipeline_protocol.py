"""CPU model of the barrier protocol of the pair attention kernel (attn_pair_kernel): TMA producer, two
column-info warps, the in-order tcgen05 MMA issuer and two softmax warpgroups (one per query tile, four
TMEM lane groups each) walking one tile list whose entries each carry the use bits of one or both query
tiles.  Random lists, random delays of every asynchronous completion (TMA landings in any order, MMAs
in issue order) and random rescale decisions are run against invariants:

- no deadlock;
- the K / V^T slot an MMA reads holds the entry the protocol says from the MMA's issue to its
  completion;
- the softmax of tile t reads S_t of the entry it is at, and the column info of that entry for as long
  as it uses it;
- PV_t(j) reads P_t(j) complete in all four lane groups, and S_t(j+1) overwrites P_t(j) only after
  PV_t(j) has completed;
- an O_t rescale after the wait for S_t(j) finds every earlier PV_t complete;
- the epilogue of tile t sees every PV_t applied.

The model mirrors the kernel's waits one for one (slot and ring indices, phase parities); it exercises
no GPU.  Barrier semantics: a phase completes when its arrival count is reached; a parity test is true
iff the barrier's current phase parity differs from the tested one."""
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


def run(entries, nk=2, nv=2, nci=4, seed=0, rescale_p=0.2, s_before_pv=False, skip_without_ci_wait=False):
    """entries: list of (use0, use1), at least one true each.  Returns True when every role finished."""
    rng = random.Random(seed)
    n = len(entries)
    k_full, k_empty = [Bar(1) for _ in range(nk)], [Bar(1) for _ in range(nk)]
    v_full, v_empty = [Bar(1) for _ in range(nv)], [Bar(1) for _ in range(nv)]
    ci_full, ci_empty = [Bar(2) for _ in range(nci)], [Bar(8) for _ in range(nci)]
    s_full, p_full = [Bar(1), Bar(1)], [Bar(4), Bar(4)]
    q_ready, o_final = Bar(8), Bar(1)
    kslot, vslot = [None] * nk, [None] * nv
    sbuf = [None, None]                    # per query tile: ("S", u) or ("P", u, set of lane groups)
    cinfo = [None] * nci
    applied = [[], []]                     # entries whose PV_t has completed, in order
    used = [[u for u in range(n) if entries[u][t]] for t in (0, 1)]
    rescale = [[rng.random() < rescale_p for _ in range(n)] for _ in (0, 1)]
    tma_events, fifo = [], []

    def producer():
        for u in range(n):
            sk, sv = u % nk, u % nv
            while not k_empty[sk].done(((u // nk) & 1) ^ 1):
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
            k_full[s].arrive()
        else:
            vslot[s] = u
            v_full[s].arrive()

    def colinfo():
        for u in range(n):
            ci = u % nci
            while not ci_empty[ci].done(((u // nci) & 1) ^ 1):
                yield False
            cinfo[ci] = u
            ci_full[ci].arrive()
            yield True

    def mma():
        cnt, pend = [0, 0], [False, False]
        while not q_ready.done(0):
            yield False

        def issue_pv(t, ent):
            while not p_full[t].done((cnt[t] - 1) & 1):
                yield False
            sv = ent % nv
            while not v_full[sv].done((ent // nv) & 1):
                yield False
            check(vslot[sv] == ent, f"PV_{t}({ent}) issued on V slot holding {vslot[sv]}")
            b = sbuf[t]
            check(b is not None and b[0] == "P" and b[1] == ent and len(b[2]) == 4, f"PV_{t}({ent}) issued on {b}")
            fifo.append(("PV", t, ent))
            yield True

        def issue_s(t, u):
            fifo.append(("S", t, u))
            fifo.append(("commit_s", t, None))
            cnt[t] += 1
            pend[t] = True

        for u in range(n):
            sk = u % nk
            k_ready, any_pv = False, False
            for t in (0, 1):
                uses = entries[u][t]
                if s_before_pv and uses:
                    # planted error: S_t(u) before PV_t(u - 1)
                    if not k_ready:
                        while not k_full[sk].done((u // nk) & 1):
                            yield False
                        k_ready = True
                    had = pend[t]
                    issue_s(t, u)
                    if had:
                        yield from issue_pv(t, u - 1)
                        any_pv = True
                    continue
                if pend[t]:
                    yield from issue_pv(t, u - 1)
                    pend[t] = False
                    any_pv = True
                if uses:
                    if not k_ready:
                        while not k_full[sk].done((u // nk) & 1):
                            yield False
                        k_ready = True
                    check(kslot[sk] == u, f"S({u}) issued on K slot holding {kslot[sk]}")
                    issue_s(t, u)
            if any_pv:
                fifo.append(("commit_v", (u - 1) % nv, None))
            fifo.append(("commit_k", sk, None))
            yield True
        any_pv = False
        for t in (0, 1):
            if pend[t]:
                yield from issue_pv(t, n - 1)
                any_pv = True
        if any_pv:
            fifo.append(("commit_v", (n - 1) % nv, None))
        fifo.append(("end", None, None))
        yield True

    def complete(op):
        kind, a, b = op
        if kind == "S":
            t, u = a, b
            check(kslot[u % nk] == u, f"S_{t}({u}) completed on K slot holding {kslot[u % nk]}")
            prev = sbuf[t]
            check(prev is None or (prev[0] == "P" and applied[t] and applied[t][-1] == prev[1]),
                  f"S_{t}({u}) overwrote {prev} before its PV completed")
            sbuf[t] = ("S", u)
        elif kind == "PV":
            t, u = a, b
            check(vslot[u % nv] == u, f"PV_{t}({u}) completed on V slot holding {vslot[u % nv]}")
            s = sbuf[t]
            check(s is not None and s[0] == "P" and s[1] == u and len(s[2]) == 4, f"PV_{t}({u}) read {s}")
            applied[t].append(u)
        elif kind == "commit_s":
            s_full[a].arrive()
        elif kind == "commit_v":
            v_empty[a].arrive()
        elif kind == "commit_k":
            k_empty[a].arrive()
        else:
            o_final.arrive()

    def softmax(t, g):
        q_ready.arrive()
        yield True
        j = 0
        for u in range(n):
            ci = u % nci
            if not (skip_without_ci_wait and not entries[u][t]):
                while not ci_full[ci].done((u // nci) & 1):
                    yield False
            if not entries[u][t]:
                ci_empty[ci].arrive()
                yield True
                continue
            check(cinfo[ci] == u, f"softmax {t} at {u} read column info of {cinfo[ci]}")
            while not s_full[t].done(j & 1):
                yield False
            s = sbuf[t]
            check(s == ("S", u) or (s and s[0] == "P" and s[1] == u), f"softmax {t} at {u} read {s}")
            check(cinfo[ci] == u, f"softmax {t} at {u}: column info replaced by {cinfo[ci]} while in use")
            if s[0] == "S":
                sbuf[t] = ("P", u, set())
            sbuf[t][2].add(g)
            ci_empty[ci].arrive()
            if rescale[t][u] and j >= 1:
                check(len(applied[t]) == j, f"O_{t} rescale at tile {j} with {len(applied[t])} PVs applied")
            p_full[t].arrive()
            j += 1
            yield True
        while not o_final.done(0):
            yield False
        check(applied[t] == used[t], f"epilogue {t} saw PVs {applied[t]} of {used[t]}")

    roles = [producer(), mma(), colinfo(), colinfo()] + [softmax(t, g) for t in (0, 1) for g in range(4)]
    idle = 0
    while roles:
        while tma_events and rng.random() < 0.5:
            land(tma_events.pop(rng.randrange(len(tma_events))))
        while fifo and rng.random() < 0.5:
            complete(fifo.pop(0))
        prog = False
        for r in rng.sample(roles, len(roles)):
            try:
                prog |= bool(next(r))
            except StopIteration:
                roles.remove(r)
                prog = True
        idle = 0 if (prog or tma_events or fifo) else idle + 1
        if idle > 50:
            return False
    while fifo:
        complete(fifo.pop(0))
    return True


def _lists(rng, count):
    out = [[], [(True, False)], [(False, True)], [(True, True)] * 3]
    for _ in range(count):
        n = rng.randint(1, 40)
        mode = rng.random()
        if mode < 0.5:   # mostly shared, as on video rows
            out.append([(True, True) if rng.random() < 0.85 else ((True, False) if rng.random() < 0.5 else (False, True))
                        for _ in range(n)])
        else:            # sparse-like: independent selections
            lst = []
            for _ in range(n):
                a, b = rng.random() < 0.5, rng.random() < 0.5
                lst.append((a, b) if (a or b) else (True, False))
            out.append(lst)
    return out


@pytest.mark.parametrize("nk,nv", [(2, 2), (3, 2), (2, 3)])
def test_pair_protocol_finishes_and_keeps_every_invariant(nk, nv):
    rng = random.Random(5)
    for i, entries in enumerate(_lists(rng, 40)):
        for seed in range(2):
            assert run(entries, nk=nk, nv=nv, seed=seed + 10 * i), (entries, seed)


def test_long_runs_of_one_tile_only():
    # one query tile idle for many entries (the tail pair whose second block is past the rows)
    for seed in range(4):
        assert run([(True, False)] * 30, seed=seed)
        assert run([(False, True)] * 9 + [(True, True)] * 9 + [(True, False)] * 9, seed=seed)


def test_s_before_pv_is_caught():
    # issuing S_t(u) before PV_t(u - 1) lets S overwrite an unread P (or a rescale see a PV missing)
    caught = 0
    for seed in range(20):
        try:
            ok = run([(True, True)] * 12, seed=seed, rescale_p=0.5, s_before_pv=True)
        except AssertionError:
            ok = False
        caught += not ok
    assert caught > 0


def test_skipping_without_the_column_info_wait_is_caught():
    # an idle tile arriving on ci_empty before the entry's column info exists breaks the phase count
    caught = 0
    for seed in range(20):
        try:
            ok = run([(True, False)] * 10 + [(True, True)] * 4, seed=seed, skip_without_ci_wait=True)
        except AssertionError:
            ok = False
        caught += not ok
    assert caught > 0
