"""Pin of the oracle's sparse-mode key restriction (fluxbbs.com "单卡 4090 怎么做到的", fourth technique:
after the first two denoising steps only a quarter of the candidate video blocks are attended to).

The oracle marks every key with the candidate block it belongs to and masks the keys of blocks that are
not kept.  Here the expected result is built a different way: for every query row the attended keys are
*gathered* -- the kept candidate blocks are enumerated region by region as explicit token ranges (history
blocks first, in age order, then current-segment blocks), followed by every earlier description head, the
current head and the action tails whose window holds the row's latent frame -- and torch's fp64
scaled_dot_product_attention runs over exactly that key set, with no mask at all.

The selection is written by hand, not taken from the ranking rule, and is chosen so that a wrong
candidate numbering shows: the history ends in a partial 128-token block, the two query blocks of one
attention CTA keep different sets, and each keeps one history block and one current block (in another
head, the opposite pairing).
"""
import numpy as np
import torch

from int8_kv_cache_action_b200.workloads import make_inputs, small_config
from oracle import attention as att
from oracle.quant import dequantize
from oracle.ring import OracleCache

TILE = 128


def _f32(t):
    return t.float().numpy()


def _candidate_ranges(n_hist, n_cur):
    """[(region, start, stop)] for candidate index 0, 1, ...: history blocks, then current blocks."""
    out = []
    for region, n in (("hist", n_hist), ("cur", n_cur)):
        start = 0
        while start < n:
            out.append((region, start, min(start + TILE, n)))
            start += TILE
    return out


def _gathered_reference(cache, inp, cfg, sel, scale):
    hk8, hks, hv8, hvs = cache.history()
    pk8, pks, pv8, pvs = cache.prior_heads()
    nq, H, _ = inp.q.shape
    T = cfg.tokens_per_frame
    seg = cfg.current
    cands = _candidate_ranges(hk8.shape[1], nq)
    out = np.zeros((nq, H, cfg.head_dim))
    lse = np.zeros((H, nq))
    for h in range(H):
        src_k = {"hist": torch.from_numpy(dequantize(hk8[h], hks[h])), "cur": inp.k_cur[:, h].double()}
        src_v = {"hist": torch.from_numpy(dequantize(hv8[h], hvs[h])), "cur": inp.v_cur[:, h].double()}
        head_k = torch.from_numpy(dequantize(pk8[h], pks[h]))
        head_v = torch.from_numpy(dequantize(pv8[h], pvs[h]))
        for i in range(nq):
            t = i // T
            ks, vs = [], []
            for c in sorted(int(x) for x in sel[h, i // TILE]):
                region, a, b = cands[c]
                ks.append(src_k[region][a:b])
                vs.append(src_v[region][a:b])
            ks.append(head_k)
            vs.append(head_v)
            at = seg.head_len
            ks.append(inp.k_txt[:at, h].double())
            vs.append(inp.v_txt[:at, h].double())
            for tail in seg.tails:
                if tail.f0 <= t < tail.f1:
                    ks.append(inp.k_txt[at:at + tail.len, h].double())
                    vs.append(inp.v_txt[at:at + tail.len, h].double())
                at += tail.len
            K, V = torch.cat(ks), torch.cat(vs)
            qi = inp.q[i, h].double()[None]
            o = torch.nn.functional.scaled_dot_product_attention(qi[None], K[None], V[None], scale=scale)[0, 0]
            out[i, h] = o.numpy()
            lse[h, i] = float(torch.logsumexp((qi @ K.T)[0] * scale, dim=0))
    return out, lse


def test_sparse_key_restriction_matches_gathered_attention():
    # 50-token frames, window 3 of 4 appended frames -> 150 history tokens = blocks [0, 128) and the
    # partial [128, 150); a 4-frame segment -> 200 queries = query blocks 0 and 1, current blocks
    # [0, 128) and [128, 200), i.e. candidates 0, 1 (history) and 2, 3 (current).
    cfg = small_config(heads=2, head_dim=64, tokens_per_frame=50, n_frames=4, window=3, prior_frames=(2, 2),
                       prior_head=10, head_len=12, tails=((8, 0, 2), (6, 2, 4)))
    inp = make_inputs(cfg)
    cache = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                        cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        cache.append(_f32(kv.k), _f32(kv.v), seg.n_frames, _f32(kv.head_k), _f32(kv.head_v))
    assert cache.history_tokens() == 150 and cfg.n_query == 200
    sel = np.array([[[1, 2], [0, 3]],          # head 0: block 0 keeps the partial history block + current 0
                    [[3, 0], [2, 1]]],         # head 1: the opposite pairing, listed out of order
                   np.int32)
    scale = 0.125
    got, got_lse = att.attention(cache, _f32(inp.q), _f32(inp.k_cur), _f32(inp.v_cur), _f32(inp.k_txt),
                                 _f32(inp.v_txt), cfg.current, scale, sel=sel)
    want, want_lse = _gathered_reference(cache, inp, cfg, sel, scale)
    assert np.abs(got - want).max() < 1e-12
    assert np.abs(got_lse - want_lse).max() < 1e-12
