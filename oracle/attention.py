"""Masked attention over the INT8 history, prior description heads, the current segment and its text.

Test infrastructure (see package header).  Follows fluxbbs.com "架构" (segment-
causal + action-aware attention) and "单卡 4090 怎么做到的" (INT8 storage with
float scales, BF16 compute; block-sparse mode).  Computed plainly in fp64:

    for head h, query row i at latent frame t = i // T:
        k^_j = q8_j * s_j  (exact, fp64) for cached keys, the bf16 value otherwise
        s_ij = (q_i . k^_j) * scale          over the visible keys j
        O_i  = sum_j softmax_j(s_ij) v^_j,   LSE_i = log sum_j exp(s_ij)

Readings adopted: the score scale is the caller's `scale` (1/sqrt(d) by default,
the standard choice; the pages give none); keys and queries enter after any
positional encoding; only video query rows are computed.  In sparse mode the
history and current-video keys are restricted to the blocks kept for the row's
query block and head (see select.py); text and prior heads are always kept.

The matrix products use numpy's fp64 matmul as a library primitive; the
softmax is the textbook max-subtracted form.
"""
from __future__ import annotations

import numpy as np

from .quant import dequantize
from .visibility import key_windows, text_query_mask, TILE


def _keys_for_head(cache, h, k_cur, v_cur, k_txt, v_txt):
    hk8, hks, hv8, hvs = cache.history()
    pk8, pks, pv8, pvs = cache.prior_heads()
    K = np.concatenate([dequantize(hk8[h], hks[h]), dequantize(pk8[h], pks[h]),
                        k_cur[:, h, :].astype(np.float64), k_txt[:, h, :].astype(np.float64)], axis=0)
    V = np.concatenate([dequantize(hv8[h], hvs[h]), dequantize(pv8[h], pvs[h]),
                        v_cur[:, h, :].astype(np.float64), v_txt[:, h, :].astype(np.float64)], axis=0)
    return K, V


def attention(cache, q, k_cur, v_cur, k_txt, v_txt, text, scale, rows=None, sel=None, row_batch=256):
    """Returns (out float64 [len(rows), H, D], lse float64 [H, len(rows)]).

    q, k_cur, v_cur: float32 [Nq, H, D]; k_txt, v_txt: float32 [Lt, H, D] (exact bf16 values).
    sel: None (dense) or int32 [H, n_qblocks, k] kept candidate blocks (sparse).
    """
    nq, H, D = q.shape
    T = cache.T
    rows = np.arange(nq) if rows is None else np.asarray(rows, np.int64)
    Lh = cache.history_tokens()
    Lp = cache.head_used
    lo, hi = key_windows(Lh, Lp, nq, text)
    nkv = lo.shape[0]
    # candidate block id of every key (-1 = not a candidate, i.e. always kept in sparse mode)
    cand = np.full(nkv, -1, np.int64)
    nh = (Lh + TILE - 1) // TILE
    cand[:Lh] = np.arange(Lh) // TILE
    cand[Lh + Lp:Lh + Lp + nq] = nh + np.arange(nq) // TILE
    out = np.zeros((len(rows), H, D), np.float64)
    lse = np.zeros((H, len(rows)), np.float64)
    sc = float(scale)
    for h in range(H):
        K, V = _keys_for_head(cache, h, k_cur, v_cur, k_txt, v_txt)
        for r0 in range(0, len(rows), row_batch):
            rr = rows[r0:r0 + row_batch]
            Q = q[rr, h, :].astype(np.float64)
            S = (Q @ K.T) * sc
            t = (rr // T)[:, None]
            vis = (lo[None, :] <= t) & (t < hi[None, :])
            if sel is not None:
                kept = np.zeros((len(rr), nh + (nq + TILE - 1) // TILE + 1), bool)
                kept[:, -1] = True                       # index -1 -> always kept
                qb = rr // TILE
                for a, b in enumerate(qb):
                    kept[a, sel[h, b]] = True
                vis &= np.take_along_axis(kept, np.broadcast_to(cand, (len(rr), nkv)), axis=1)
            S = np.where(vis, S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            P = np.exp(S - m)
            l = P.sum(axis=1, keepdims=True)
            out[r0:r0 + len(rr), h, :] = (P @ V) / l
            lse[h, r0:r0 + len(rr)] = (m + np.log(l))[:, 0]
    return out, lse


def attention_text(cache, q_txt, k_cur, v_cur, k_txt, v_txt, text, scale, rows=None):
    """Text query rows of the current segment (visibility: visibility.text_query_mask), dense.

    q_txt: float32 [Lt, H, D].  Returns (out float64 [len(rows), H, D], lse float64 [H, len(rows)]); a
    row with no visible key has output 0 and LSE -inf.
    """
    lt, H, D = q_txt.shape
    nq = k_cur.shape[0]
    rows = np.arange(lt) if rows is None else np.asarray(rows, np.int64)
    vis = text_query_mask(cache.history_tokens(), cache.head_used, nq, cache.T, text)[rows]
    out = np.zeros((len(rows), H, D), np.float64)
    lse = np.full((H, len(rows)), -np.inf, np.float64)
    live = vis.any(axis=1)
    sc = float(scale)
    for h in range(H):
        K, V = _keys_for_head(cache, h, k_cur, v_cur, k_txt, v_txt)
        Q = q_txt[rows, h, :].astype(np.float64)
        S = np.where(vis, (Q @ K.T) * sc, -np.inf)
        m = np.where(live, S.max(axis=1), 0.0)[:, None]
        P = np.exp(S - m)
        l = P.sum(axis=1, keepdims=True)
        out[live, h, :] = ((P @ V) / np.where(l > 0, l, 1.0))[live]
        lse[h, live] = (m + np.log(np.where(l > 0, l, 1.0)))[live, 0]
    return out, lse
