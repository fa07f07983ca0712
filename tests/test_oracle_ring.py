"""Pins for the oracle's history ring: brute-force sliding-window simulation, invariants."""
import collections

import numpy as np
import pytest

from oracle.quant import quantize
from oracle.ring import OracleCache, CapacityError


def _rollout(W, C, T=5, H=2, D=64, segs=(3, 2, 4, 1, 5), head=(4, 0, 3, 2, 1), seed=0):
    rng = np.random.default_rng(seed)
    cache = OracleCache(H, D, T, W, C, sum(head) + 1)
    sim = collections.deque(maxlen=W if W > 0 else None)   # textbook sliding window of frames
    heads = []
    for F, hl in zip(segs, head):
        k = rng.standard_normal((F * T, H, D)).astype(np.float32)
        v = rng.standard_normal((F * T, H, D)).astype(np.float32)
        hk = rng.standard_normal((hl, H, D)).astype(np.float32) if hl else None
        hv = rng.standard_normal((hl, H, D)).astype(np.float32) if hl else None
        cache.append(k, v, F, hk, hv)
        for f in range(F):
            sim.append((k[f * T:(f + 1) * T], v[f * T:(f + 1) * T]))
        if hl:
            heads.append((hk, hv))
        yield cache, list(sim), heads


@pytest.mark.parametrize("W,C", [(3, 3), (3, 7), (4, 4), (18, 18), (0, 40)])
def test_history_matches_deque_simulation(W, C):
    for cache, frames, heads in _rollout(W, C):
        hk8, hks, hv8, hvs = cache.history()
        assert hk8.shape[1] == len(frames) * cache.T
        if frames:
            k = np.concatenate([f[0] for f in frames])     # [Lh, H, D]
            v = np.concatenate([f[1] for f in frames])
            qk, sk = quantize(k)
            qv, sv = quantize(v)
            assert np.array_equal(hk8, qk.transpose(1, 0, 2)) and np.array_equal(hks, sk.T)
            assert np.array_equal(hv8, qv.transpose(1, 0, 2)) and np.array_equal(hvs, sv.T)
        pk8, pks, pv8, pvs = cache.prior_heads()
        if heads:
            qk, sk = quantize(np.concatenate([h[0] for h in heads]))
            assert np.array_equal(pk8, qk.transpose(1, 0, 2)) and np.array_equal(pks, sk.T)


def test_window_invariant_newest_frames():
    for cache, frames, _ in _rollout(4, 6):
        r = cache.retained_frames()
        assert len(r) <= 4
        assert r == list(range(cache.frames_appended - len(r), cache.frames_appended))


def test_physical_layout_does_not_change_history():
    a = list(_rollout(3, 3))[-1][0]
    b = list(_rollout(3, 11))[-1][0]
    for x, y in zip(a.history(), b.history()):
        assert np.array_equal(x, y)


def test_tiny_config_eviction_schedule():
    # 2-frame segments, window 4: after segment 2 the window holds frames 0..3;
    # segment 3's own append evicts frames 0 and 1.  With window 3 segment 3 already misses frame 0.
    c = OracleCache(2, 64, 24, 4, 4, 48)
    z = np.zeros((48, 2, 64), np.float32)
    c.append(z, z, 2)
    c.append(z, z, 2)
    assert c.retained_frames() == [0, 1, 2, 3]
    c.append(z, z, 2)
    assert c.retained_frames() == [2, 3, 4, 5]
    c3 = OracleCache(2, 64, 24, 3, 3, 48)
    c3.append(z, z, 2)
    c3.append(z, z, 2)
    assert c3.retained_frames() == [1, 2, 3]


def test_capacity_errors_leave_state_unchanged():
    c = OracleCache(1, 64, 2, 0, 3, 2)
    z = np.zeros((4, 1, 64), np.float32)
    c.append(z, z, 2)
    with pytest.raises(CapacityError):
        c.append(z, z, 2)
    assert c.frames_appended == 2
    h = np.zeros((3, 1, 64), np.float32)
    with pytest.raises(CapacityError):
        c.append(z[:2], z[:2], 1, h, h)
    assert c.frames_appended == 2 and c.head_used == 0
