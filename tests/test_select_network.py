"""CPU model of the register-resident bitonic network of the sparse selection kernel (one warp per query
block, M keys per lane): lane l starts with candidates i * 32 + l, the network runs on element
e = l M + i, exchanging across lanes (shuffle by lane ^ j / M) when the partner distance j is at least M
and inside the lane otherwise.  The model mirrors the kernel's loops and direction tests one for one; it
checks that the result is the ascending order for every M the kernel is built for, with padded slots.

The top-128 selection (keep <= 128) is modelled the same way: chunks of 128 candidates, 4 per lane
(lane l holds candidates 4 l .. 4 l + 3 of the chunk), each sorted by the network; the running list A
and a sorted chunk B combine as min(A[e], B[127 - e]) (B read from lane 31 - l, register 3 - i) and one
merge network; the first keep keys must equal the first keep of the full sort."""
import random

import pytest


def network(keys_by_lane, M):
    a = [list(v) for v in keys_by_lane]          # a[lane][i]
    n = 32 * M
    k = 2
    while k <= n:
        j = k >> 1
        while j >= M:
            lm = j // M
            new = [row[:] for row in a]
            for lane in range(32):
                take_min = ((lane & lm) == 0) == (((lane * M) & k) == 0)
                for i in range(M):
                    o = a[lane ^ lm][i]
                    new[lane][i] = min(o, a[lane][i]) if take_min else max(o, a[lane][i])
            a = new
            j >>= 1
        j = M // 2
        while j > 0:
            if j < k:
                for lane in range(32):
                    for i in range(M):
                        if i & j:
                            continue
                        up = ((lane * M + i) & k) == 0
                        x, y = a[lane][i], a[lane][i ^ j]
                        sw = (x > y) == up
                        a[lane][i], a[lane][i ^ j] = (y, x) if sw else (x, y)
            j >>= 1
        k <<= 1
    return [a[e // M][e % M] for e in range(n)]


@pytest.mark.parametrize("M", [8, 16, 32])
def test_network_sorts_with_padding(M):
    rng = random.Random(M)
    pad = (1 << 64) - 1
    for n_cand in (1, 2, 31, 32 * M // 2 + 3, 32 * M):
        scores = [rng.randrange(0, 50) for _ in range(n_cand)]          # many ties: the index decides
        keys = [(s << 32) | c for c, s in enumerate(scores)]
        lanes = [[keys[i * 32 + l] if i * 32 + l < n_cand else pad for i in range(M)] for l in range(32)]
        assert network(lanes, M) == sorted(keys) + [pad] * (32 * M - n_cand)


def merge_network(a, M):
    """Sorts a bitonic sequence held as a[lane][i], element e = lane * M + i (the kernel's merge)."""
    a = [row[:] for row in a]
    j = 16 * M
    while j >= M:
        lm = j // M
        new = [row[:] for row in a]
        for lane in range(32):
            take_min = (lane & lm) == 0
            for i in range(M):
                o = a[lane ^ lm][i]
                new[lane][i] = min(o, a[lane][i]) if take_min else max(o, a[lane][i])
        a = new
        j >>= 1
    j = M // 2
    while j > 0:
        for lane in range(32):
            for i in range(M):
                if i & j:
                    continue
                x, y = a[lane][i], a[lane][i ^ j]
                a[lane][i], a[lane][i ^ j] = (x, y) if x < y else (y, x)
        j >>= 1
    return a


def top128(keys, pad):
    """The kernel's chunked selection: returns the 128 smallest keys ascending."""
    a = None
    for c0 in range(0, len(keys), 128):
        chunk = keys[c0:c0 + 128]
        lanes = [[chunk[l * 4 + i] if l * 4 + i < len(chunk) else pad for i in range(4)] for l in range(32)]
        srt = network(lanes, 4)
        t = [[srt[l * 4 + i] for i in range(4)] for l in range(32)]
        if a is None:
            a = t
            continue
        a = [[min(a[l][i], t[l ^ 31][3 - i]) for i in range(4)] for l in range(32)]
        a = merge_network(a, 4)
    return [a[e // 4][e % 4] for e in range(128)]


def test_top128_equals_the_full_sort():
    rng = random.Random(5)
    pad = (1 << 64) - 1
    for n_cand in (1, 7, 83, 128, 129, 200, 331, 548, 1024):
        for trial in range(3):
            scores = [rng.randrange(0, 40 if trial else 1 << 20) for _ in range(n_cand)]
            keys = [(s << 32) | c for c, s in enumerate(scores)]
            want = sorted(keys) + [pad] * max(0, 128 - n_cand)
            assert top128(keys, pad) == want[:128], (n_cand, trial)


def test_top128_model_catches_an_unreversed_chunk():
    # pairing A[e] with B[e] instead of B[127 - e] loses kept keys: the model must notice
    rng = random.Random(9)
    keys = [(rng.randrange(0, 1 << 20) << 32) | c for c in range(331)]
    pad = (1 << 64) - 1
    lanes0 = [[keys[l * 4 + i] for i in range(4)] for l in range(32)]
    s0 = network(lanes0, 4)
    a = [[s0[l * 4 + i] for i in range(4)] for l in range(32)]
    chunk = keys[128:256]
    s1 = network([[chunk[l * 4 + i] for i in range(4)] for l in range(32)], 4)
    t = [[s1[l * 4 + i] for i in range(4)] for l in range(32)]
    wrong = merge_network([[min(a[l][i], t[l][i]) for i in range(4)] for l in range(32)], 4)
    assert [wrong[e // 4][e % 4] for e in range(128)] != sorted(keys[:256])[:128]
