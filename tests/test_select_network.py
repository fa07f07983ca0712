"""CPU model of the register-resident bitonic network of the sparse selection kernel (one warp per query
block, M keys per lane): lane l starts with candidates i * 32 + l, the network runs on element
e = l M + i, exchanging across lanes (shuffle by lane ^ j / M) when the partner distance j is at least M
and inside the lane otherwise.  The model mirrors the kernel's loops and direction tests one for one; it
checks that the result is the ascending order for every M the kernel is built for, with padded slots."""
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
