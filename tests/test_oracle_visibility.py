"""Pins for the oracle's visibility rule and tile classes: closed-form counts and a token-level brute force."""
import json
import os

import numpy as np
import pytest

from int8_kv_cache_action_b200.workloads import CONFIGS, SegmentText, Tail, small_config
from oracle import visibility as vis


def _counts(cfg):
    hist_frames = sum(p.n_frames for p in cfg.prior)
    if cfg.window_frames:
        hist_frames = min(hist_frames, cfg.window_frames)
    lh = hist_frames * cfg.tokens_per_frame
    lp = sum(p.head_len for p in cfg.prior)
    return vis.visible_counts(lh, lp, cfg.n_query, cfg.tokens_per_frame, cfg.current)


@pytest.mark.parametrize("name,expected", [
    # history + current video + description head + one 64-token tail, from the configs' sizes
    ("C1", 7020 + 3120 + 256 + 64),
    ("C2", 15840 + 26400 + 768 + 64),
    ("C4", 158400 + 26400 + 7 * 768 + 64),
])
def test_closed_form_visible_counts(name, expected):
    c = _counts(CONFIGS[name])
    assert c.min() == expected and c.max() == expected


def test_c2_last_window_is_clipped_and_every_frame_sees_one_tail():
    cur = CONFIGS["C2"].current
    assert [(t.f0, t.f1) for t in cur.tails][-1] == (28, 30)
    for t in range(30):
        assert sum(1 for a in cur.tails if a.f0 <= t < a.f1) == 1


def _brute_rollout(T, W, segs):
    """Token-level record of a rollout: every token ever produced, with who may see it.

    Rule in words: a query of segment s at frame t sees (a) video frames of earlier segments that are
    among the newest W frames produced before s (all if W == 0), (b) every description head of segments
    <= s, (c) all video of segment s, (d) tails of segment s whose window contains t.
    Returns, for the last segment, the visibility matrix [Nq, keys] with keys ordered as
    [history (age order), earlier heads, current video, current head, current tails].
    """
    frames_before = []
    for si, seg in enumerate(segs[:-1]):
        frames_before += [(si, f) for f in range(seg.n_frames)]
    kept = frames_before if W == 0 else frames_before[-W:] if W else []
    keys = []
    for (si, f) in kept:
        keys += [("hist", si, f)] * T
    for si, seg in enumerate(segs[:-1]):
        keys += [("head", si, None)] * seg.head_len
    cur = segs[-1]
    s = len(segs) - 1
    keys += [("video", s, None)] * (cur.n_frames * T)
    keys += [("head", s, None)] * cur.head_len
    for a in cur.tails:
        keys += [("tail", s, (a.f0, a.f1))] * a.len
    nq = cur.n_frames * T
    m = np.zeros((nq, len(keys)), bool)
    for i in range(nq):
        t = i // T
        for j, (kind, seg_of_key, extra) in enumerate(keys):
            if kind in ("hist", "head", "video"):
                m[i, j] = True
            elif kind == "tail":
                m[i, j] = seg_of_key == s and extra[0] <= t < extra[1]
    return m, len(kept) * T


@pytest.mark.parametrize("name", ["C0", "C0w3"])
def test_brute_force_tiny(name):
    cfg = CONFIGS[name]
    segs = list(cfg.prior) + [cfg.current]
    m, lh = _brute_rollout(cfg.tokens_per_frame, cfg.window_frames, segs)
    lp = sum(p.head_len for p in cfg.prior)
    lo, hi = vis.key_windows(lh, lp, cfg.n_query, cfg.current)
    t = (np.arange(cfg.n_query) // cfg.tokens_per_frame)[:, None]
    assert np.array_equal(m, (lo[None] <= t) & (t < hi[None]))
    assert lh == (96 if cfg.window_frames == 4 else 72)   # window 3 already drops frame 0 before segment 3


def _class_from_matrix(m, regions):
    nq = m.shape[0]
    out = []
    for b in range(0, nq, 128):
        row = []
        base = 0
        for n in regions:
            for s in range(0, n, 128):
                blk = m[b:b + 128, base + s: base + min(s + 128, n)]
                row.append(1 if blk.all() else (0 if not blk.any() else 2))
            base += n
        out.append(row)
    return np.asarray(out, np.int8)


@pytest.mark.parametrize("cfg", [
    small_config(),
    small_config(tokens_per_frame=70, n_frames=5, tails=((64, 0, 1), (100, 1, 4), (5, 4, 5), (130, 2, 3))),
    small_config(tokens_per_frame=33, n_frames=7, window=0, prior_frames=(2, 5), tails=()),
])
def test_class_map_against_brute_force(cfg):
    segs = list(cfg.prior) + [cfg.current]
    m, lh = _brute_rollout(cfg.tokens_per_frame, cfg.window_frames, segs)
    lp = sum(p.head_len for p in cfg.prior)
    got = vis.class_map(lh, lp, cfg.n_query, cfg.tokens_per_frame, cfg.current)
    want = _class_from_matrix(m, vis.region_lengths(lh, lp, cfg.n_query, cfg.current))
    assert np.array_equal(got, want)
    assert (got == vis.PARTIAL).any() or not cfg.current.tails


def test_prompt_structure_whole_segment_action_visible_everywhere():
    # papers.ananclaw.com prompt example: one action spanning the whole 30-frame segment
    with open(os.path.join(os.path.dirname(__file__), "golden", "prompt_two_segments.json")) as f:
        g = json.load(f)
    (f0, f1), = g["_expected_windows"][0]
    text = SegmentText(30, 8, (Tail(5, f0, f1),))
    c = vis.visible_counts(0, 0, 30 * 4, 4, text)
    assert np.all(c == 30 * 4 + 8 + 5)
    cm = vis.class_map(0, 0, 30 * 4, 4, text)
    assert np.all(cm == vis.FULL)
