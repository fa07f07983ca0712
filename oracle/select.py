"""Block-sparse candidate selection.  Test infrastructure (see package header).

The pages (fluxbbs.com "单卡 4090 怎么做到的", fourth technique) fix only that
the first two denoising steps use dense attention and later steps keep 25 % of
the candidate video blocks.  Everything below is this project's own definition
of which blocks those are ("parity vs the real system: unpinned"):

  * query blocks: 128 consecutive current-segment video rows (last may be short);
  * candidate blocks: the retained history, age order, cut into 128-token blocks
    from its first token, followed by the current segment's video tokens cut the
    same way; candidate index = history blocks 0..Nh-1 then current Nh..Nh+Nc-1;
  * pooled vectors, per head and channel, in fp32 with a fixed order:
        history key  k~ = float(q8) * s          (one fp32 multiply)
        current key  k~ = float(bf16)
        query        q~ = float(bf16)
        sum over the block's valid tokens in ascending order from +0.0f,
        mean = sum / n_valid                      (fp32 IEEE division);
  * score = fmaf chain over channels (see csrc/oracle_score.c);
  * keep k = ceil(n * keep_frac) blocks (clamped to [1, n]), ordered by score
    descending then candidate index ascending;
  * the order is total: a NaN score (an inf or NaN input reaches the means)
    ranks as -inf, and -0 ranks equal to +0, so every candidate has exactly
    one rank (ties between them go to the lower index like any other tie).
Text, description heads and in-window action tails are always kept.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from . import build as _build

TILE = 128
_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _lib.oracle_scores_fmaf.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        _lib.oracle_scores_fmaf.restype = None
    return _lib


def block_means(x: np.ndarray) -> np.ndarray:
    """x: float32 [N, D] -> float32 [ceil(N/128), D]; sequential fp32 sums, then one division."""
    x = np.asarray(x, np.float32)
    n, d = x.shape
    nb = (n + TILE - 1) // TILE
    acc = np.zeros((nb, d), np.float32)
    for r in range(TILE):                      # add row r of every block, in ascending row order
        rows = np.arange(nb) * TILE + r
        ok = rows < n
        acc[ok] = (acc[ok] + x[rows[ok]]).astype(np.float32)
    nvalid = np.minimum(TILE, n - np.arange(nb) * TILE).astype(np.float32)
    return (acc / nvalid[:, None]).astype(np.float32)


def dequant_f32(q8: np.ndarray, s: np.ndarray) -> np.ndarray:
    """float(q8) * s in fp32 (one rounding)."""
    return (q8.astype(np.float32) * s.astype(np.float32)[..., None]).astype(np.float32)


def scores(qmean: np.ndarray, kmean: np.ndarray) -> np.ndarray:
    lib = _load()
    qm = np.ascontiguousarray(qmean, np.float32)
    km = np.ascontiguousarray(kmean, np.float32)
    out = np.empty((qm.shape[0], km.shape[0]), np.float32)
    lib.oracle_scores_fmaf(qm.shape[0], km.shape[0], qm.shape[1],
                           qm.ctypes.data, km.ctypes.data, out.ctypes.data)
    return out


def rank_key(s: np.ndarray) -> np.ndarray:
    """Score as a ranking key: NaN -> -inf (and -0 == +0, as float comparison already has it)."""
    s = np.asarray(s, np.float64)
    return np.where(np.isnan(s), -np.inf, s)


def keep_count(n: int, keep_frac: float) -> int:
    if n == 0:
        return 0
    k = math.ceil(n * float(np.float32(keep_frac)))
    return max(1, min(n, k))


def select(q: np.ndarray, hist_k8: np.ndarray, hist_ks: np.ndarray, k_cur: np.ndarray, keep_frac: float):
    """Per head and query block, the kept candidate indices in rank order.

    q, k_cur: float32 [N, H, D] (exact bf16 values); hist_k8 int8 [H, Lh, D]; hist_ks float32 [H, Lh].
    Returns (sel int32 [H, n_qb, k], score float32 [H, n_qb, n_cand]).
    """
    n, H, D = q.shape
    nqb = (n + TILE - 1) // TILE
    nh = (hist_k8.shape[1] + TILE - 1) // TILE
    nc = (k_cur.shape[0] + TILE - 1) // TILE
    ncand = nh + nc
    k = keep_count(ncand, keep_frac)
    sel = np.zeros((H, nqb, k), np.int32)
    sc = np.zeros((H, nqb, ncand), np.float32)
    for h in range(H):
        qm = block_means(q[:, h, :])
        parts = []
        if hist_k8.shape[1]:
            parts.append(block_means(dequant_f32(hist_k8[h], hist_ks[h])))
        parts.append(block_means(k_cur[:, h, :]))
        km = np.concatenate(parts, axis=0)
        s = scores(qm, km)
        sc[h] = s
        idx = np.arange(ncand)
        for b in range(nqb):
            order = np.lexsort((idx, -rank_key(s[b])))   # primary: score desc; then index asc
            sel[h, b] = order[:k]
    return sel, sc
