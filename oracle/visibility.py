"""Segment-causal, action-aware visibility.  Test infrastructure (see package header).

Follows fluxbbs.com "架构": attention is bidirectional inside a segment and a
segment sees only itself and earlier segments (segment-causal); each segment's
text is split into one description head, visible across segments, and action
tails, each tied to one action and its time window and visible only inside its
own segment, locked to that window.  papers.ananclaw.com "这是什么" restates the
same split (descriptive context persists, action instructions only act inside
their time window).

For a query of the current segment at segment-local latent frame t the keys
are, in this order (the "regions"):
  0  retained history video tokens (age order)      -- always visible
  1  description heads of earlier segments           -- always visible
  2  current-segment video tokens                    -- always visible (bidirectional)
  3  current-segment text: head tokens               -- always visible
                           tail a tokens             -- visible iff f0_a <= t < f1_a
Action tails of earlier segments are never cached, so never visible.
Windows are half-open and counted in segment-local latent frames (reading).

Each key carries a window [lo, hi); it is visible to frame t iff lo <= t < hi.

Text query rows (the text stream of the double-stream joint attention, papers.ananclaw.com "这是什么"
component list).  The pages state who may see the text, not what the text sees; the reading adopted
keeps the action lock in both directions and the description head free of actions:
  * a description-head row of the current segment sees the retained history, earlier heads, all
    current-segment video and the current head, but no action tail of the segment: the head is cached
    and visible across segments, so a head that absorbed the tails would carry the segment's actions
    into later segments -- the cross-segment replay the action-aware mask exists to remove;
  * a row of tail a (window [f0, f1)) sees the retained history, earlier heads and the current head,
    the current-segment video frames t with f0 <= t < f1 (the mirror of "tail a is visible to frame t
    iff f0 <= t < f1"), and the tails b whose window shares a frame with a's
    (max(f0_b, f0) < min(f1_b, f1)),
    itself included (a tail with an empty window shares no frame, so it sees no tail and no video).
A text row with no visible key (possible only in degenerate layouts) has output 0.
"""
from __future__ import annotations

import numpy as np

ALWAYS_LO, ALWAYS_HI = 0, 1 << 30
TILE = 128
SKIP, FULL, PARTIAL = 0, 1, 2


def region_lengths(history_tokens, prior_head_tokens, n_query, text):
    return [history_tokens, prior_head_tokens, n_query, text.text_len]


def key_windows(history_tokens, prior_head_tokens, n_query, text):
    """(lo, hi) int64 arrays over all keys in region order."""
    n_always = history_tokens + prior_head_tokens + n_query + text.head_len
    lo = [np.full(n_always, ALWAYS_LO, np.int64)]
    hi = [np.full(n_always, ALWAYS_HI, np.int64)]
    for t in text.tails:
        lo.append(np.full(t.len, t.f0, np.int64))
        hi.append(np.full(t.len, t.f1, np.int64))
    return np.concatenate(lo), np.concatenate(hi)


def tiles(history_tokens, prior_head_tokens, n_query, text):
    """KV tiles: each region is cut into 128-key tiles from its first key; the last may be partial.

    Returns a list of (region, start_in_region, count, global_key_offset).
    """
    out = []
    base = 0
    for r, n in enumerate(region_lengths(history_tokens, prior_head_tokens, n_query, text)):
        for s in range(0, n, TILE):
            out.append((r, s, min(TILE, n - s), base + s))
        base += n
    return out


def class_map(history_tokens, prior_head_tokens, n_query, tokens_per_frame, text):
    """int8 [n_qblocks, n_tiles]: SKIP (no visible pair), FULL (all valid pairs visible) or PARTIAL.

    Only valid rows (< n_query) and valid keys of each tile count.  Rows of the
    same latent frame see the same keys, so pairs are counted per frame.
    """
    lo, hi = key_windows(history_tokens, prior_head_tokens, n_query, text)
    tl = tiles(history_tokens, prior_head_tokens, n_query, text)
    nqb = (n_query + TILE - 1) // TILE
    out = np.zeros((nqb, len(tl)), np.int8)
    for b in range(nqb):
        rows = np.arange(b * TILE, min((b + 1) * TILE, n_query))
        frames, counts = np.unique(rows // tokens_per_frame, return_counts=True)
        for j, (_, _, cnt, g0) in enumerate(tl):
            klo, khi = lo[g0:g0 + cnt], hi[g0:g0 + cnt]
            vis = 0
            for t, c in zip(frames, counts):
                vis += int(c) * int(np.count_nonzero((klo <= t) & (t < khi)))
            total = len(rows) * cnt
            out[b, j] = FULL if vis == total else (SKIP if vis == 0 else PARTIAL)
    return out


def visible_counts(history_tokens, prior_head_tokens, n_query, tokens_per_frame, text):
    """Number of visible keys for every query row (int64 [n_query])."""
    lo, hi = key_windows(history_tokens, prior_head_tokens, n_query, text)
    t = np.arange(n_query) // tokens_per_frame
    frames = np.unique(t)
    per_frame = {int(f): int(np.count_nonzero((lo <= f) & (f < hi))) for f in frames}
    return np.asarray([per_frame[int(x)] for x in t], np.int64)


def visible_mask_row(lo, hi, frame):
    return (lo <= frame) & (frame < hi)


def text_row_kinds(text):
    """Per text row: (is_head, f0, f1); f0 = f1 = 0 for head rows."""
    out = [(True, 0, 0)] * text.head_len
    for t in text.tails:
        out += [(False, t.f0, t.f1)] * t.len
    return out


def text_query_mask(history_tokens, prior_head_tokens, n_query, tokens_per_frame, text):
    """bool [text_len, n_keys] over the keys in region order (history, earlier heads, current video,
    current head, current tails): which keys each current-segment text row sees."""
    lo, hi = key_windows(history_tokens, prior_head_tokens, n_query, text)
    n_keys = lo.shape[0]
    c0 = history_tokens + prior_head_tokens              # first current-video key
    t0 = c0 + n_query + text.head_len                    # first tail key
    video_frame = np.arange(n_query) // tokens_per_frame
    m = np.zeros((text.text_len, n_keys), bool)
    for i, (is_head, f0, f1) in enumerate(text_row_kinds(text)):
        m[i, :c0] = True                                 # retained history and earlier heads
        m[i, c0 + n_query:t0] = True                     # the current description head
        if is_head:
            m[i, c0:c0 + n_query] = True                 # every current video frame, no tail
        else:
            m[i, c0:c0 + n_query] = (f0 <= video_frame) & (video_frame < f1)
            m[i, t0:] = np.maximum(lo[t0:], f0) < np.minimum(hi[t0:], f1)   # tails sharing a frame
    return m
