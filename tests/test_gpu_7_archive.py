"""Archive of evicted frames and selection of the retained history through the C ABI (reading in nomas.h
and oracle/ring.py; hyphentech.top config table: at most 18 history latent frames on the GPU, earlier
history archived to CPU).  Records are compared byte for byte with the oracle's; after a selection the
retained history (in its new age order), the sparse selection over it and the attention are compared
with the oracle given the same selection, also after further appends; stale buffers are reported."""
import math

import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200 import _nomas as N
from int8_kv_cache_action_b200.workloads import make_inputs, small_config
from tests.helpers import TOL_MAX_ABS, TOL_MEAN_REL, attention_errors, f32

pytestmark = pytest.mark.gpu


def _record_parts(rec, H, T, D):
    b = rec.numpy()
    codes = H * T * D
    k8 = b[:codes].view(np.int8).reshape(H, T, D)
    v8 = b[codes:2 * codes].view(np.int8).reshape(H, T, D)
    ks = b[2 * codes:2 * codes + 4 * H * T].view(np.float32).reshape(H, T)
    vs = b[2 * codes + 4 * H * T:].view(np.float32).reshape(H, T)
    return k8, ks, v8, vs


def _rollout(cfg, inp):
    """Append the prior segments frame-window by frame-window, archiving every frame the next append
    would evict, on both sides.  Returns (gpu cache, oracle cache, gpu records, oracle records)."""
    from int8_kv_cache_action_b200.runtime import KVCache
    from oracle.ring import OracleCache
    gc = KVCache.for_config(cfg)
    oc = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                     cfg.head_store_tokens)
    grec, orec = {}, {}
    for seg, kv in zip(cfg.prior, inp.prior):
        ev = gc.evicted_by(seg.n_frames)
        assert ev == oc.evicted_by(seg.n_frames)
        for g in ev:
            grec[g] = gc.archive(g)
            orec[g] = oc.archive(g)
        hk = None if kv.head_k is None else kv.head_k.cuda()
        hv = None if kv.head_v is None else kv.head_v.cuda()
        gc.append(kv.k.cuda(), kv.v.cuda(), seg.n_frames, hk, hv)
        oc.append(f32(kv.k), f32(kv.v), seg.n_frames, f32(kv.head_k), f32(kv.head_v))
        assert gc.retained() == oc.retained_frames()
    torch.cuda.synchronize()
    return gc, oc, grec, orec


def _cfg():
    return small_config(tokens_per_frame=150, n_frames=3, prior_frames=(2, 3, 2, 3), window=4, heads=2)


def _check_history(gc, oc):
    k, v = gc.dequant()
    hk8, hks, hv8, hvs = oc.history()
    want_k = (hk8.astype(np.float32) * hks[..., None]).transpose(1, 0, 2)
    want_v = (hv8.astype(np.float32) * hvs[..., None]).transpose(1, 0, 2)
    assert np.array_equal(k.cpu().numpy(), want_k) and np.array_equal(v.cpu().numpy(), want_v)


def _check_attention(gc, oc, cfg, inp, mode):
    from int8_kv_cache_action_b200.runtime import mask_views, segment_text_of
    from oracle import attention as att
    from oracle import select as sel
    seg = segment_text_of(cfg.current)
    q, kc = inp.q.cuda(), inp.k_cur.cuda()
    buf, lay = gc.build_mask(seg, mode, 0.25, q, kc)
    out, _ = gc.attention(seg, buf, q, kc, inp.v_cur.cuda(), inp.k_txt.cuda(), inp.v_txt.cuda(), mode=mode)
    torch.cuda.synchronize()
    assert gc.status() == 0
    s = None
    if mode:
        hk8, hks, _, _ = oc.history()
        s, sc = sel.select(f32(inp.q), hk8, hks, f32(inp.k_cur), 0.25)
        mv = mask_views(buf, lay)
        assert np.array_equal(mv["sel"].cpu().numpy(), s)
    ref, _ = att.attention(oc, f32(inp.q), f32(inp.k_cur), f32(inp.v_cur), f32(inp.k_txt), f32(inp.v_txt),
                           cfg.current, 1.0 / math.sqrt(cfg.head_dim), sel=s)
    mx, mr = attention_errors(out.cpu().numpy(), ref)
    assert mx <= TOL_MAX_ABS and mr <= TOL_MEAN_REL, (mx, mr)


def test_archived_records_match_the_oracle_byte_for_byte():
    cfg = _cfg()
    gc, oc, grec, orec = _rollout(cfg, make_inputs(cfg))
    assert sorted(grec) == sorted(orec) and len(grec) >= 4
    for g in grec:
        for got, want in zip(_record_parts(grec[g], cfg.heads, cfg.tokens_per_frame, cfg.head_dim), orec[g]):
            assert np.array_equal(got.view(np.uint8), np.ascontiguousarray(want).view(np.uint8)), g


@pytest.mark.parametrize("mode", [0, 1])
def test_selected_history_matches_the_oracle_and_appends_continue(mode):
    cfg = _cfg()
    inp = make_inputs(cfg)
    gc, oc, grec, orec = _rollout(cfg, inp)
    ret = gc.retained()
    old = sorted(grec)
    order = [old[1], ret[-1], old[0], ret[0]]          # archived and retained frames, in a new age order
    gc.select(order, grec)
    oc.select(order, orec)
    assert gc.retained() == order
    _check_history(gc, oc)
    _check_attention(gc, oc, cfg, inp, mode)
    # an append after the selection slides from the selected list
    extra = inp.k_cur[:2 * cfg.tokens_per_frame], inp.v_cur[:2 * cfg.tokens_per_frame]
    gc.append(extra[0].cuda(), extra[1].cuda(), 2)
    oc.append(f32(extra[0]), f32(extra[1]), 2)
    assert gc.retained() == oc.retained_frames()
    _check_history(gc, oc)
    _check_attention(gc, oc, cfg, inp, mode)


def test_selection_errors_and_stale_buffers():
    from int8_kv_cache_action_b200.runtime import KVCache, segment_text_of
    cfg = _cfg()
    inp = make_inputs(cfg)
    gc, oc, grec, orec = _rollout(cfg, inp)
    ret = gc.retained()
    assert N.nomas_kv_select(gc.handle, [ret[0], ret[0]]) == N.NOMAS_EINVAL          # repeated frame
    assert N.nomas_kv_select(gc.handle, [sorted(grec)[0]]) == N.NOMAS_EINVAL         # no record for it
    assert N.nomas_kv_select(gc.handle, ret + [sorted(grec)[0]], [0] * 4 + [grec[sorted(grec)[0]].data_ptr()]) \
        == N.NOMAS_EINVAL                                                           # more than W frames
    full = KVCache(2, 64, 10, 0, 8, 1)
    assert N.nomas_kv_select(full.handle, []) == N.NOMAS_EUNSUPPORTED               # no window
    assert gc.retained() == ret                                                    # nothing changed
    # a mask and a workspace prepared before a selection are reported as stale after it
    seg = segment_text_of(cfg.current)
    q, kc, vc, kt, vt = (getattr(inp, n).cuda() for n in ("q", "k_cur", "v_cur", "k_txt", "v_txt"))
    buf, _ = gc.build_mask(seg)
    gc.select(list(reversed(ret)))
    gc.attention(seg, buf, q, kc, vc, kt, vt)
    assert gc.status() == N.NOMAS_EDEVICE
