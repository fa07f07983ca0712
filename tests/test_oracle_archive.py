"""Pins for the oracle's archive of evicted frames and the selection of the retained history (reading in
oracle/ring.py; hyphentech.top config table: at most 18 history latent frames on the GPU, earlier
history archived to CPU).  Expected histories are built from the original inputs, quantised afresh."""
import collections

import numpy as np
import pytest

from oracle.quant import quantize
from oracle.ring import OracleCache

T, H, D = 5, 2, 16


def _frames(n, seed=0):
    rng = np.random.default_rng(seed)
    return [(rng.standard_normal((T, H, D)).astype(np.float32), rng.standard_normal((T, H, D)).astype(np.float32))
            for _ in range(n)]


def _expected(frames, order):
    k = np.concatenate([frames[g][0] for g in order])
    v = np.concatenate([frames[g][1] for g in order])
    qk, sk = quantize(k)
    qv, sv = quantize(v)
    return qk.transpose(1, 0, 2), sk.T, qv.transpose(1, 0, 2), sv.T


def _rollout_with_archive(W=3, segs=(2, 3, 1, 4)):
    frames = _frames(sum(segs))
    c = OracleCache(H, D, T, W, W, 1)
    archive, g = {}, 0
    for n in segs:
        for e in c.evicted_by(n):                # archive what the append is about to drop
            archive[e] = c.archive(e)
        k = np.concatenate([frames[g + f][0] for f in range(n)])
        v = np.concatenate([frames[g + f][1] for f in range(n)])
        before = c.retained_frames()
        c.append(k, v, n)
        g += n
        dropped = [e for e in before if e not in c.retained_frames()]
        assert sorted(dropped) == sorted(e for e in before if e in archive)
    return c, frames, archive


def test_evicted_by_matches_a_sliding_window():
    c, frames, archive = _rollout_with_archive()
    # every appended frame except the retained ones went through the archive first (frames that an
    # append writes and drops at once -- older than the window within one segment -- are never retained)
    assert c.retained_frames() == [7, 8, 9]
    assert sorted(archive) == [0, 1, 2, 3, 4, 5]
    dq = collections.deque(range(10), maxlen=3)
    assert c.retained_frames() == list(dq)


def test_select_current_frames_in_order_changes_nothing():
    c, frames, archive = _rollout_with_archive()
    before = c.history()
    c.select(c.retained_frames(), {})
    for a, b in zip(before, c.history()):
        assert np.array_equal(a, b)


def test_select_archived_frames_restores_their_codes():
    c, frames, archive = _rollout_with_archive()
    order = [1, 8, 4]                            # two archived frames around a retained one, in this order
    c.select(order, archive)
    assert c.retained_frames() == order
    for got, want in zip(c.history(), _expected(frames, order)):
        assert np.array_equal(got, want)


def test_appends_after_a_selection_slide_from_the_selected_list():
    c, frames, archive = _rollout_with_archive()
    c.select([0, 5], archive)
    extra = _frames(2, seed=9)
    c.append(np.concatenate([f[0] for f in extra]), np.concatenate([f[1] for f in extra]), 2)
    assert c.retained_frames() == [5, 10, 11]
    frames = frames + extra
    for got, want in zip(c.history(), _expected(frames, [5, 10, 11])):
        assert np.array_equal(got, want)


def test_selection_errors():
    c, frames, archive = _rollout_with_archive()
    with pytest.raises(ValueError):
        c.select([1, 2, 3, 4], archive)          # more than W frames
    with pytest.raises(ValueError):
        c.select([8, 8], archive)                # a repeated frame
    with pytest.raises(KeyError):
        c.select([6], {})                        # neither retained nor given
    full = OracleCache(H, D, T, 0, 10, 1)
    with pytest.raises(ValueError):
        full.select([], {})                      # no window: the full history is always kept
