"""Shared test helpers: build the CUDA cache and the oracle cache from the same seeded inputs."""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

from int8_kv_cache_action_b200.workloads import Config, Inputs, make_inputs

TOL_MAX_ABS = 1e-2      # attention: max |o - o_ref| over compared elements
TOL_MEAN_REL = 2e-3     # attention: sum |o - o_ref| / sum |o_ref|


def f32(t):
    return None if t is None else t.float().cpu().numpy()


def oracle_cache(cfg: Config, inp: Inputs):
    from oracle.ring import OracleCache
    oc = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                     cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        oc.append(f32(kv.k), f32(kv.v), seg.n_frames, f32(kv.head_k), f32(kv.head_v))
    return oc


def gpu_cache(cfg: Config, inp: Inputs, device="cuda"):
    from int8_kv_cache_action_b200.runtime import KVCache
    gc = KVCache.for_config(cfg, device)
    for seg, kv in zip(cfg.prior, inp.prior):
        hk = None if kv.head_k is None else kv.head_k.to(device)
        hv = None if kv.head_v is None else kv.head_v.to(device)
        gc.append(kv.k.to(device), kv.v.to(device), seg.n_frames, hk, hv)
    return gc


def to_device(inp: Inputs, device="cuda"):
    return {k: getattr(inp, k).to(device) for k in ("q", "k_cur", "v_cur", "k_txt", "v_txt")}


def attention_errors(out, ref):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(out - ref)
    return float(err.max()), float(err.sum() / max(np.abs(ref).sum(), 1e-300))


def sample_rows(cfg: Config, n_random=200, seed=7):
    """Rows covering every latent frame's first and last row, 128-block edges and random rows."""
    nq, T = cfg.n_query, cfg.tokens_per_frame
    rows = set()
    for f in range(cfg.current.n_frames):
        rows.update({f * T, f * T + T - 1})
    for b in range(0, nq, 128):
        if (b // 128) % 4 == 0 or b + 128 >= nq:
            rows.update({b, min(b + 127, nq - 1)})
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, nq, n_random).tolist())
    rows.add(nq - 1)
    return np.asarray(sorted(rows), np.int64)


def rn32(x: Fraction) -> Fraction:
    """Round a rational below the fp32 overflow threshold to the nearest fp32 (subnormals included),
    ties to even."""
    if x == 0:
        return Fraction(0)
    neg = x < 0
    x = -x if neg else x
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if x < Fraction(2) ** e:
        e -= 1
    assert e <= 127, "overflow"
    e = max(e, -126)                                    # the subnormal grid is 2^-149
    m = x / Fraction(2) ** (e - 23)
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl & 1):
        fl += 1
    r = Fraction(fl) * Fraction(2) ** (e - 23)
    return -r if neg else r
