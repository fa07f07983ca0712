"""GPU parity of the text query rows (NOMAS_MODE_TEXT; the reading is stated in nomas.h and in
oracle/visibility.py) through the C ABI: the class map of the text query blocks exactly, the attention
output within max-abs 1e-2 / mean-rel 2e-3 of the fp64 oracle and the LSE, all rows on small layouts
(an empty tail window and a text without head included) and sampled rows at full size."""
import math

import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, small_config
from tests.helpers import TOL_MAX_ABS, TOL_MEAN_REL, attention_errors, f32, gpu_cache, oracle_cache

pytestmark = pytest.mark.gpu

TEXT = 2


def _classes(m, regions):
    """Tile classes of a boolean [rows, keys] matrix: 128-row blocks x 128-key tiles of each region."""
    out = []
    for b in range(0, m.shape[0], 128):
        row, base = [], 0
        for n in regions:
            for s0 in range(0, n, 128):
                blk = m[b:b + 128, base + s0:base + min(s0 + 128, n)]
                row.append(1 if blk.all() else (0 if not blk.any() else 2))
            base += n
        out.append(row)
    return np.asarray(out, np.int8)


SMALL = [
    small_config(tokens_per_frame=100, n_frames=3, prior_frames=(3, 3), window=4),
    small_config(tokens_per_frame=33, n_frames=5, window=0, prior_frames=(2, 3),
                 tails=((20, 0, 2), (7, 2, 2), (130, 1, 5), (9, 4, 5))),
    small_config(tokens_per_frame=57, n_frames=4, head_dim=64, heads=3, head_len=0, window=3,
                 prior_frames=(2, 2), tails=((70, 0, 4), (64, 1, 2))),
]


def _run(cfg, rows=None):
    from int8_kv_cache_action_b200.runtime import mask_views, segment_text_of
    from oracle import attention as att
    from oracle import visibility as vis
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    oc = oracle_cache(cfg, inp)
    seg = segment_text_of(cfg.current)
    buf, lay = gc.build_mask(seg, TEXT)
    m = vis.text_query_mask(oc.history_tokens(), oc.head_used, cfg.n_query, cfg.tokens_per_frame, cfg.current)
    want_cls = _classes(m, vis.region_lengths(oc.history_tokens(), oc.head_used, cfg.n_query, cfg.current))
    assert np.array_equal(mask_views(buf, lay)["class"].cpu().numpy(), want_cls)
    d = {k: getattr(inp, k).cuda() for k in ("q_txt", "k_cur", "v_cur", "k_txt", "v_txt")}
    out, lse = gc.attention(seg, buf, d["q_txt"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"], mode=TEXT,
                            want_lse=True)
    torch.cuda.synchronize()
    assert gc.status() == 0
    rows = np.arange(cfg.current.text_len) if rows is None else rows
    ref, ref_lse = att.attention_text(oc, f32(inp.q_txt), f32(inp.k_cur), f32(inp.v_cur), f32(inp.k_txt),
                                      f32(inp.v_txt), cfg.current, 1.0 / math.sqrt(cfg.head_dim), rows=rows)
    got = out.cpu().numpy()[rows]
    assert np.isfinite(got).all()
    mx, mr = attention_errors(got, ref)
    assert mx <= TOL_MAX_ABS and mr <= TOL_MEAN_REL, (mx, mr)
    live = np.isfinite(ref_lse)
    gl = lse.cpu().numpy()[:, rows]
    assert np.abs(gl[live] - ref_lse[live]).max() <= 2e-3
    dead = ~live.all(axis=0)
    assert np.all(got[dead] == 0)          # rows with no visible key


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"T{c.tokens_per_frame}_d{c.head_dim}_h{c.current.head_len}")
def test_text_rows_small_all_rows(cfg, attn_kernel):
    _run(cfg)


@pytest.mark.parametrize("name", ["C1", "C2"])
def test_text_rows_full_size_sampled(name):
    cfg = CONFIGS[name]
    rng = np.random.default_rng(5)
    lt, hl = cfg.current.text_len, cfg.current.head_len
    rows = {0, hl - 1, hl, lt - 1} | set(rng.integers(0, lt, 60).tolist())
    rows |= {hl + 64 * a for a in range(len(cfg.current.tails))}          # first row of every tail
    _run(cfg, np.asarray(sorted(rows), np.int64))


@pytest.mark.parametrize("shares", [2, 3, 8])
@pytest.mark.parametrize("cfg", SMALL[:2], ids=lambda c: f"T{c.tokens_per_frame}_h{c.current.head_len}")
def test_text_rows_split_lists(cfg, shares, attn_kernel):
    # each key list cut into 2, 3 or 8 shares (some of them empty at this size) and merged
    from int8_kv_cache_action_b200 import _nomas as N
    prev = N.nomas_set_text_split(shares)
    try:
        _run(cfg)
    finally:
        N.nomas_set_text_split(prev)


def test_video_rows_unchanged_by_a_text_call():
    # a text-mode call between two video calls leaves the video output bitwise identical
    from int8_kv_cache_action_b200.runtime import segment_text_of
    cfg = SMALL[0]
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    seg = segment_text_of(cfg.current)
    d = {k: getattr(inp, k).cuda() for k in ("q", "q_txt", "k_cur", "v_cur", "k_txt", "v_txt")}
    vb, _ = gc.build_mask(seg)
    a, _ = gc.attention(seg, vb, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"])
    tb, _ = gc.build_mask(seg, TEXT)
    gc.attention(seg, tb, d["q_txt"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"], mode=TEXT)
    b, _ = gc.attention(seg, vb, d["q"], d["k_cur"], d["v_cur"], d["k_txt"], d["v_txt"])
    torch.cuda.synchronize()
    assert torch.equal(a, b) and gc.status() == 0
