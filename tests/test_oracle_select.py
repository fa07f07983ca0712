"""Pins for the oracle's sparse block selection: exact small-integer cases, order pins, ties, 100 % keep."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import select as sel


def test_block_means_sequential_order():
    # [2^24, 1 x 126, -2^24]: adding in ascending row order loses every +1 (2^24 + 1 rounds back to 2^24
    # under half-even), so the fp32 mean is exactly 0; any other summation order keeps some of them.
    x = np.zeros((128, 1), np.float32)
    x[0, 0] = 2.0 ** 24
    x[1:127, 0] = 1.0
    x[127, 0] = -(2.0 ** 24)
    assert sel.block_means(x)[0, 0] == 0.0
    assert float(x[:, 0].astype(np.float64).sum()) == 126.0


def test_block_means_ragged_last_block():
    x = np.arange(300, dtype=np.float32)[:, None]
    m = sel.block_means(x)
    assert m.shape == (3, 1)
    assert list(m[:, 0]) == [63.5, 191.5, (256 + 299) / 2]


def test_fma_chain_single_rounding_and_channel_order():
    # qmean = [a, -a], kmean = [a, a] with a = 1 + 2^-12:
    # acc0 = fmaf(a, a, 0) = RN(1 + 2^-11 + 2^-24) = 1 + 2^-11 (half-ulp tie to even)
    # acc1 = fmaf(-a, a, acc0) = -(1 + 2^-11 + 2^-24) + (1 + 2^-11) = -2^-24 exactly (one rounding)
    a = np.float32(1 + 2.0 ** -12)
    q = np.array([[a, -a]], np.float32)
    k = np.array([[a, a]], np.float32)
    assert sel.scores(q, k)[0, 0] == np.float32(-(2.0 ** -24))
    # reversed channel order would give +2^-24, separate multiply-then-add would give 0
    assert sel.scores(q[:, ::-1], k[:, ::-1])[0, 0] == np.float32(2.0 ** -24)


def test_exact_small_integer_case_against_rationals():
    rng = np.random.default_rng(5)
    H, D, nq, lh, nk = 2, 16, 256, 384, 512
    q = rng.integers(-1, 2, (nq, H, D)).astype(np.float32)     # |q mean| <= 1, step 2^-7
    kc = rng.integers(-3, 4, (nk, H, D)).astype(np.float32)
    k8 = rng.integers(-12, 13, (H, lh, D)).astype(np.int8)     # k~ in [-3, 3], mean step 2^-9
    ks = np.full((H, lh), 0.25, np.float32)
    # every partial dot product is a multiple of 2^-16 below 48 in magnitude: exact in fp32
    got, score = sel.select(q, k8, ks, kc, 0.25)
    for h in range(H):
        kfull = np.concatenate([k8[h].astype(np.int64) * Fraction(1, 4), kc[:, h].astype(np.int64)])
        qm = [sum(Fraction(int(v)) for v in q[b * 128:(b + 1) * 128, h, c]) / 128 for b in range(2) for c in range(D)]
        qm = np.asarray(qm, object).reshape(2, D)
        kblocks = [kfull[j * 128:(j + 1) * 128] for j in range(len(kfull) // 128)]
        km = [[sum(blk[:, c]) / 128 for c in range(D)] for blk in kblocks]
        for b in range(2):
            exact = [sum(qm[b][c] * km[j][c] for c in range(D)) for j in range(len(km))]
            assert [float(v) for v in exact] == list(score[h, b])     # every step was exact in fp32
            order = sorted(range(len(exact)), key=lambda j: (-exact[j], j))
            assert list(got[h, b]) == order[:2]                        # ceil(7 * 0.25) = 2


def test_ties_pick_lower_index_and_full_keep():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((128, 1, 8)).astype(np.float32)
    blk = rng.standard_normal((128, 1, 8)).astype(np.float32)
    kc = np.concatenate([blk, blk, -blk, blk])            # candidates 0,1,3 identical
    k8 = np.zeros((1, 0, 8), np.int8)
    ks = np.zeros((1, 0), np.float32)
    s_top, sc = sel.select(q, k8, ks, kc, 0.5)
    assert sc[0, 0, 0] == sc[0, 0, 1] == sc[0, 0, 3]
    if sc[0, 0, 0] > sc[0, 0, 2]:
        assert list(s_top[0, 0]) == [0, 1]
    else:
        assert list(s_top[0, 0]) == [2, 0]
    s_all, _ = sel.select(q, k8, ks, kc, 1.0)
    assert sorted(s_all[0, 0]) == [0, 1, 2, 3]


@pytest.mark.parametrize("n,f,k", [(331, 0.25, 83), (80, 0.25, 20), (1, 0.25, 1), (7, 0.25, 2), (10, 1.0, 10), (0, 0.25, 0)])
def test_keep_count(n, f, k):
    assert sel.keep_count(n, f) == k


def test_nan_scores_rank_as_minus_infinity():
    # One inf query channel: its block mean is inf, so candidate scores become inf, -inf or NaN
    # (inf * 0 in the fmaf chain).  The order is total: NaN ranks as -inf, ties by lower index.
    q = np.ones((128, 1, 2), np.float32)
    q[5, 0, 0] = np.inf
    blocks = [(0.0, 5.0), (-1.0, 0.0), (1.0, 0.0), (0.0, 0.0), (-2.0, 0.0)]   # NaN, -inf, inf, NaN, -inf
    kc = np.concatenate([np.tile(np.array(b, np.float32), (128, 1))[:, None, :] for b in blocks])
    k8 = np.zeros((1, 0, 2), np.int8)
    ks = np.zeros((1, 0), np.float32)
    s_all, sc = sel.select(q, k8, ks, kc, 1.0)
    s = sc[0, 0]
    assert np.isnan(s[0]) and np.isnan(s[3]) and s[1] == -np.inf and s[4] == -np.inf and s[2] == np.inf
    assert list(s_all[0, 0]) == [2, 0, 1, 3, 4]
    s_half, _ = sel.select(q, k8, ks, kc, 0.5)
    assert list(s_half[0, 0]) == [2, 0, 1]
