"""INT8 history ring with an N-latent-frame sliding window.  Test infrastructure (see package header).

Follows fluxbbs.com "架构" (each finished segment's text and video K/V go into a
cache that the next segment reuses), "单卡 4090 怎么做到的" second technique
(retained history limited to 18 frames, "temporal_context" sampling) and the
hyphentech.top config table (the GPU keeps at most 18 history latent frames,
older history leaves the GPU; the standard setting keeps full history).

Readings adopted where the pages are silent:
  * frames carry a global latent index g = 0, 1, 2, ... over the rollout and
    live in ring slot g mod C (C = capacity in frames);
  * with a window W the retained frames are the newest W, the same for every
    query of the next segment (the budget limits history only, hyphentech.top
    "官方运行限制");  W = 0 means full history;
  * appending an F-frame segment writes only its frames f >= F - W (the others
    would leave the window at once);
  * description heads go to a separate store and are never evicted by the
    frame window (they are "always visible across segments");
  * action tails are never cached (they are visible only inside their own
    segment).

Archive and selection (hyphentech.top config table: the GPU keeps at most 18
history latent frames, earlier history is archived to CPU).  The pages say only
that; the reading adopted:
  * a frame that leaves the window can first be copied out of the cache as it
    stands (its INT8 codes and scales), its "record";
  * the retained history can be set to any list of at most W frames, each one
    either retained now or given by its record, in the order the list gives
    (that order is the history's age order for every later step);
  * later appends add their frames at the new end and drop from the old end,
    the same sliding window as before.
"""
from __future__ import annotations

import numpy as np

from .quant import quantize


class CapacityError(ValueError):
    pass


class OracleCache:
    def __init__(self, heads, head_dim, tokens_per_frame, window_frames, capacity_frames, head_store_tokens):
        self.H, self.D, self.T = heads, head_dim, tokens_per_frame
        self.W, self.C, self.HS = window_frames, capacity_frames, head_store_tokens
        if self.W > 0 and self.C < self.W:
            raise CapacityError("capacity below window")
        n = self.C * self.T
        self.k8 = np.zeros((self.H, n, self.D), np.int8)
        self.v8 = np.zeros((self.H, n, self.D), np.int8)
        self.ks = np.zeros((self.H, n), np.float32)
        self.vs = np.zeros((self.H, n), np.float32)
        self.hk8 = np.zeros((self.H, self.HS, self.D), np.int8)
        self.hv8 = np.zeros((self.H, self.HS, self.D), np.int8)
        self.hks = np.zeros((self.H, self.HS), np.float32)
        self.hvs = np.zeros((self.H, self.HS), np.float32)
        self.frames_appended = 0
        self.head_used = 0
        self.segments = 0
        self.retained = []            # global indices of the retained frames, age order
        self.store = {}               # global index -> record (k8 [H,T,D], ks [H,T], v8, vs) of retained frames

    # -- state -----------------------------------------------------------------------------
    def retained_frames(self):
        """Global indices of the retained history frames, oldest first."""
        return list(self.retained)

    def history_tokens(self) -> int:
        return len(self.retained_frames()) * self.T

    # -- append ----------------------------------------------------------------------------
    def append(self, k, v, n_frames, head_k=None, head_v=None):
        """k, v: float32 [n_frames*T, H, D] (exact bf16 values); head_k/v: [head_len, H, D] or None."""
        T = self.T
        head_len = 0 if head_k is None else head_k.shape[0]
        if k.shape[0] != n_frames * T:
            raise ValueError("token count")
        if self.W == 0 and self.frames_appended + n_frames > self.C:
            raise CapacityError("ring capacity")
        if self.head_used + head_len > self.HS:
            raise CapacityError("head store capacity")
        keep = n_frames if self.W == 0 else min(n_frames, self.W)
        for f in range(n_frames - keep, n_frames):
            g = self.frames_appended + f
            slot = g % self.C
            src = slice(f * T, (f + 1) * T)
            dst = slice(slot * T, (slot + 1) * T)
            qk, sk = quantize(k[src])          # [T, H, D], [T, H]
            qv, sv = quantize(v[src])
            self.k8[:, dst] = qk.transpose(1, 0, 2)
            self.v8[:, dst] = qv.transpose(1, 0, 2)
            self.ks[:, dst] = sk.T
            self.vs[:, dst] = sv.T
            self.store[g] = (qk.transpose(1, 0, 2).copy(), sk.T.copy(), qv.transpose(1, 0, 2).copy(), sv.T.copy())
            self.retained.append(g)
            if self.W > 0 and len(self.retained) > self.W:
                self.store.pop(self.retained.pop(0))
        if head_len:
            qk, sk = quantize(head_k)
            qv, sv = quantize(head_v)
            dst = slice(self.head_used, self.head_used + head_len)
            self.hk8[:, dst] = qk.transpose(1, 0, 2)
            self.hv8[:, dst] = qv.transpose(1, 0, 2)
            self.hks[:, dst] = sk.T
            self.hvs[:, dst] = sv.T
        self.frames_appended += n_frames
        self.head_used += head_len
        self.segments += 1

    # -- views -----------------------------------------------------------------------------
    def history(self):
        """Age-ordered retained history: (k8 [H,Lh,D], ks [H,Lh], v8, vs)."""
        if not self.retained:
            return (np.zeros((self.H, 0, self.D), np.int8), np.zeros((self.H, 0), np.float32),
                    np.zeros((self.H, 0, self.D), np.int8), np.zeros((self.H, 0), np.float32))
        recs = [self.store[g] for g in self.retained]
        return tuple(np.concatenate([r[i] for r in recs], axis=1) for i in range(4))

    # -- archive and selection ---------------------------------------------------------------
    def archive(self, g):
        """Record of retained frame g: copies of (k8 [H,T,D], ks [H,T], v8, vs)."""
        if g not in self.store:
            raise ValueError(f"frame {g} is not retained")
        return tuple(x.copy() for x in self.store[g])

    def evicted_by(self, n_frames):
        """Retained frames (oldest first) that an append of n_frames would drop from the window."""
        if self.W == 0:
            return []
        drop = len(self.retained) + min(n_frames, self.W) - self.W
        return self.retained[:max(0, drop)]

    def select(self, frames, records):
        """Make `frames` (global indices, age order, at most W, no repeats) the retained history; a frame
        not retained now is taken from records[g]."""
        frames = list(frames)
        if self.W == 0 or len(frames) > self.W or len(set(frames)) != len(frames):
            raise ValueError("selection needs a window, at most W frames, no repeats")
        store = {}
        for g in frames:
            store[g] = self.store[g] if g in self.store else tuple(np.asarray(x).copy() for x in records[g])
        self.store, self.retained = store, frames

    def prior_heads(self):
        u = self.head_used
        return self.hk8[:, :u], self.hks[:, :u], self.hv8[:, :u], self.hvs[:, :u]
