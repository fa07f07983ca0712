"""GPU parity of nomas_mask_build: tile classes (exact), sparse scores and kept blocks (bit-exact), and
the per-CTA tile lists derived from them."""
import dataclasses
import numpy as np
import pytest
import torch

from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, small_config
from tests.helpers import f32, gpu_cache, oracle_cache

pytestmark = pytest.mark.gpu

DENSE = [CONFIGS["C0"], CONFIGS["C0w3"], small_config(), small_config(tokens_per_frame=33, n_frames=7, window=0,
                                                                        prior_frames=(2, 5), tails=()),
         small_config(tokens_per_frame=70, n_frames=5, tails=((64, 0, 1), (100, 1, 4), (5, 4, 5), (130, 2, 3))),
         CONFIGS["C1"], CONFIGS["C2"], CONFIGS["C4"]]


def _seg(cfg):
    from int8_kv_cache_action_b200.runtime import segment_text_of
    return segment_text_of(cfg.current)


def _expected_dense_lists(cls):
    nqb, nt = cls.shape
    out = []
    for p in range(0, nqb, 2):
        c0 = cls[p]
        c1 = cls[p + 1] if p + 1 < nqb else np.zeros(nt, np.int8)
        out.append([(j, int(c0[j]), int(c1[j])) for j in range(nt) if c0[j] or c1[j]])
    return out


@pytest.mark.parametrize("cfg", DENSE, ids=lambda c: c.name + f"_w{c.window_frames}")
def test_class_map_and_dense_lists(cfg):
    from int8_kv_cache_action_b200.runtime import mask_views
    from oracle import visibility as vis
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    oc = oracle_cache(cfg, inp)
    seg = _seg(cfg)
    buf, lay = gc.build_mask(seg)
    mv = mask_views(buf, lay)
    want = vis.class_map(oc.history_tokens(), oc.head_used, cfg.n_query, cfg.tokens_per_frame, cfg.current)
    got = mv["class"].cpu().numpy()
    assert np.array_equal(got, want)
    counts = mv["count"].cpu().numpy()
    lists = mv["list"].cpu().numpy()
    tl = vis.tiles(oc.history_tokens(), oc.head_used, cfg.n_query, cfg.current)
    for p, exp in enumerate(_expected_dense_lists(want)):
        assert counts[p] == len(exp)
        for e, (j, c0, c1) in zip(lists[p, :counts[p]], exp):
            region, start, cnt, _ = tl[j]
            assert e[3] == j and (e[0] & 3) == region and e[1] == start and e[2] == cnt
            assert bool(e[0] & 4) == bool(c0) and bool(e[0] & 8) == bool(c1)
            assert bool(e[0] & 16) == (bool(c0) and (c0 == 2 or cnt < 128))
            assert bool(e[0] & 32) == (bool(c1) and (c1 == 2 or cnt < 128))
    assert gc.status() == 0


SPARSE = [small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4),
          small_config(tokens_per_frame=97, n_frames=5, prior_frames=(4, 4), window=5, head_dim=64),
          small_config(tokens_per_frame=150, n_frames=3, prior_frames=(3, 3), window=4, keep_frac=1.0),
          CONFIGS["C3r"], CONFIGS["C3"],
          # keep <= 128 takes the chunked top-128 selection (C3r, C3, the small shapes, and 548
          # candidates in five chunks, the last one ragged); larger keeps the full sorts: 158
          # candidates (keys in registers, 8 per lane), C3 at half keep (16 per lane), 548 (32 per
          # lane) and 1173 candidates (shared memory)
          small_config("wide", tokens_per_frame=100, n_frames=300, prior_frames=(400,), window=400, keep_frac=0.2),
          small_config("k158", tokens_per_frame=100, n_frames=100, prior_frames=(100,), window=100, heads=2,
                       keep_frac=0.9),
          dataclasses.replace(CONFIGS["C3"], keep_frac=0.5, name="C3half"),
          small_config("wide", tokens_per_frame=100, n_frames=300, prior_frames=(400,), window=400),
          small_config("wider", tokens_per_frame=100, n_frames=300, prior_frames=(700, 500), window=1200, heads=1)]


@pytest.mark.parametrize("cfg", SPARSE, ids=lambda c: c.name + f"_T{c.tokens_per_frame}_k{c.keep_frac}")
def test_sparse_selection_bit_exact(cfg):
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import mask_views
    from oracle import select as sel
    inp = make_inputs(cfg)
    gc = gpu_cache(cfg, inp)
    oc = oracle_cache(cfg, inp)
    q, kc = inp.q.cuda(), inp.k_cur.cuda()
    buf, lay = gc.build_mask(_seg(cfg), N.NOMAS_MODE_SPARSE, cfg.keep_frac, q, kc)
    mv = mask_views(buf, lay)
    hk8, hks, _, _ = oc.history()
    want_sel, want_score = sel.select(f32(inp.q), hk8, hks, f32(inp.k_cur), cfg.keep_frac)
    got_score = mv["score"].cpu().numpy()
    assert np.array_equal(got_score.view(np.uint32), want_score.view(np.uint32))
    assert np.array_equal(mv["sel"].cpu().numpy(), want_sel)
    # lists: kept candidates of either query block, in index order, with the right use bits
    counts, lists = mv["count"].cpu().numpy(), mv["list"].cpu().numpy()
    n_pairs = (lay["n_qblocks"] + 1) // 2
    nh = lay["n_hist_tiles"]
    for h in range(cfg.heads):
        for p in range(n_pairs):
            ent = lists[h * n_pairs + p, :counts[h * n_pairs + p]]
            vid = [e for e in ent if (e[0] & 3) in (0, 2)]
            s0 = set(want_sel[h, 2 * p].tolist())
            s1 = set(want_sel[h, 2 * p + 1].tolist()) if 2 * p + 1 < lay["n_qblocks"] else set()
            cands = [e[3] if (e[0] & 3) == 0 else e[3] - lay["n_head_tiles"] for e in vid]
            assert cands == sorted(s0 | s1)
            for e, c in zip(vid, cands):
                assert bool(e[0] & 4) == (c in s0) and bool(e[0] & 8) == (c in s1)
            assert sum(1 for e in ent if (e[0] & 3) == 1) == lay["n_head_tiles"]
    assert gc.status() == 0
