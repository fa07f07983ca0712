"""Seeded synthetic workloads for the segment-causal INT8-KV attention path.

This module holds shapes and random draws only: no quantisation, visibility,
selection or attention arithmetic lives here, so both the CUDA path and the
CPU oracle can be fed from it without sharing any of the method's code.

Shapes follow the Hy-Nomas pages:
  * 16 heads x 128 head dim in the DiT ("Segment-autoregressive DiT" bullet of
    the model-card component list, papers.ananclaw.com "这是什么");
  * DCAE-V f32t4c32 latent -> 1280x704 gives a 40x22 grid = 880 tokens per
    latent frame, 480x832 gives 15x26 = 390 (same component list; the
    single-GPU section of that page uses 480x832);
  * 30 latent frames per 5 s segment (Diffusers call with
    segment_latent_lengths=[30, 30], same page, "Diffusers" section);
  * text up to 1280 tokens (fluxbbs.com "训练流程", stage three);
  * an 18-latent-frame history window on one GPU (fluxbbs.com
    "单卡 4090 怎么做到的", second technique; hyphentech.top config table).

Inputs are fp32 N(0,1) draws from a seeded CPU generator, rounded once to
bf16.  In the reduced and production shapes, 3 of the 128 channels per head
(2 %, chosen by a seeded permutation, independently for q and for k) are
scaled by 20 in every q and K source, to stress the per-token INT8 scales.
Seeds are 42 + 100 * cfg + tensor_id (42 is the pages' default sampling seed).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

# tensor ids used in the seed formula
TID_Q, TID_KCUR, TID_VCUR, TID_KHIST, TID_VHIST, TID_KTXT, TID_VTXT, TID_OUTLIER, TID_KHEAD, TID_VHEAD, TID_QTXT = range(11)


@dataclass(frozen=True)
class Tail:
    """One action tail: `len` tokens visible to query latent frames [f0, f1) of its own segment."""
    len: int
    f0: int
    f1: int


@dataclass(frozen=True)
class SegmentText:
    """Text layout of one segment: a description head followed by action tails."""
    n_frames: int
    head_len: int
    tails: Tuple[Tail, ...] = ()

    @property
    def text_len(self) -> int:
        return self.head_len + sum(t.len for t in self.tails)


@dataclass(frozen=True)
class Config:
    name: str
    cfg_id: int
    heads: int
    head_dim: int
    tokens_per_frame: int
    window_frames: int            # 0 = unbounded (full history)
    capacity_frames: int          # ring slots
    head_store_tokens: int        # INT8 description-head store capacity
    prior: Tuple[SegmentText, ...]  # segments appended before the current one (their heads go to the store)
    current: SegmentText
    outliers: bool
    mode: int = 0                 # 0 dense, 1 sparse
    keep_frac: float = 0.25
    description: str = ""

    @property
    def n_query(self) -> int:
        return self.current.n_frames * self.tokens_per_frame

    def seed(self, tid: int) -> int:
        return 42 + 100 * self.cfg_id + tid


def _windows(n_tails: int, width: int, n_frames: int) -> Tuple[Tail, ...]:
    return tuple(Tail(64, min(width * a, n_frames), min(width * a + width, n_frames)) for a in range(n_tails))


def _c0(window: int) -> Config:
    seg = SegmentText(2, 16, (Tail(8, 0, 1), Tail(8, 1, 2)))
    return Config(
        name=f"tiny_w{window}", cfg_id=0, heads=2, head_dim=64, tokens_per_frame=24,
        window_frames=window, capacity_frames=window, head_store_tokens=3 * 16,
        prior=(seg, seg), current=seg, outliers=False,
        description="tiny: 2 heads x 64, 3 segments of 2 latent frames of a 4x6 grid, "
                    f"16-token head + 2 tails of 8, history window {window} frames")


def _c1(mode: int = 0) -> Config:
    cur = SegmentText(8, 256, tuple(Tail(64, 2 * a, 2 * a + 2) for a in range(4)))
    prior = tuple(SegmentText(8, 0) for _ in range(3))   # 24 frames -> 18 retained (ring wraps)
    return Config(
        name="reduced_480x832" + ("_sparse" if mode else ""), cfg_id=1 if not mode else 3,
        heads=16, head_dim=128, tokens_per_frame=390, window_frames=18, capacity_frames=18,
        head_store_tokens=256, prior=prior, current=cur, outliers=True, mode=mode,
        description="480x832 -> 15x26 = 390 tokens/frame, 8-frame segment (3120 queries), "
                    "18-frame INT8 history (7020 tokens), 256 head + 4 tails x 64")


def _c2(mode: int = 0) -> Config:
    cur = SegmentText(30, 768, _windows(8, 4, 30))
    prior = (SegmentText(30, 0),)                        # 30 frames -> 18 retained (ring wraps)
    return Config(
        name="production_1280x704" + ("_sparse" if mode else ""), cfg_id=2 if not mode else 3,
        heads=16, head_dim=128, tokens_per_frame=880, window_frames=18, capacity_frames=18,
        head_store_tokens=768, prior=prior, current=cur, outliers=True, mode=mode,
        description="1280x704 -> 40x22 = 880 tokens/frame, 30-frame segment (26400 queries), "
                    "18-frame INT8 history (15840 tokens), 768 head + 8 tails x 64 over 4-frame windows")


def _c4() -> Config:
    cur = SegmentText(30, 768, _windows(8, 4, 30))
    prior = tuple(SegmentText(30, 768) for _ in range(6))
    return Config(
        name="full_history_7th_of_7", cfg_id=4, heads=16, head_dim=128, tokens_per_frame=880,
        window_frames=0, capacity_frames=7 * 30, head_store_tokens=7 * 768,
        prior=prior, current=cur, outliers=True,
        description="7th segment of a 7-segment 1280x704 rollout, history not windowed: "
                    "158400 INT8 history tokens + 6 prior 768-token heads")


CONFIGS = {
    "C0": _c0(4),
    "C0w3": _c0(3),
    "C1": _c1(0),
    "C2": _c2(0),
    "C3": _c2(1),
    "C3r": _c1(1),
    "C4": _c4(),
}


def small_config(name: str = "small", *, heads=2, head_dim=128, tokens_per_frame=100, n_frames=3,
                 window=4, prior_frames=(3, 3), prior_head=40, head_len=40,
                 tails=((24, 0, 1), (30, 1, 3), (20, 2, 3)), outliers=True, mode=0, keep_frac=0.25,
                 cfg_id=5) -> Config:
    """A parity-sized config: several tiles per region and ragged tails everywhere."""
    cur = SegmentText(n_frames, head_len, tuple(Tail(*t) for t in tails))
    prior = tuple(SegmentText(f, prior_head) for f in prior_frames)
    cap = window if window > 0 else sum(prior_frames) + n_frames
    hs = prior_head * len(prior_frames) + head_len
    return Config(name=name, cfg_id=cfg_id, heads=heads, head_dim=head_dim,
                  tokens_per_frame=tokens_per_frame, window_frames=window, capacity_frames=cap,
                  head_store_tokens=max(hs, 1), prior=prior, current=cur, outliers=outliers,
                  mode=mode, keep_frac=keep_frac)


# ----------------------------------------------------------------------------------------------
# random draws
# ----------------------------------------------------------------------------------------------

def _randn_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    return x.to(torch.bfloat16).to(device)


def outlier_channels(cfg: Config) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-head outlier channel sets for q and for k: int64 [H, n_out] each."""
    n_out = int(round(0.02 * cfg.head_dim))
    g = torch.Generator(device="cpu").manual_seed(cfg.seed(TID_OUTLIER))
    qc = torch.stack([torch.randperm(cfg.head_dim, generator=g)[:n_out] for _ in range(cfg.heads)])
    kc = torch.stack([torch.randperm(cfg.head_dim, generator=g)[:n_out] for _ in range(cfg.heads)])
    return qc, kc


def _scale_outliers(x: torch.Tensor, chans: torch.Tensor) -> torch.Tensor:
    """Multiply channels chans[h] of head h by 20 (x is [tokens, H, D] bf16); exact in bf16 up to rounding."""
    xf = x.float()
    for h in range(chans.shape[0]):
        xf[:, h, chans[h]] *= 20.0
    return xf.to(torch.bfloat16)


@dataclass
class SegmentKV:
    k: torch.Tensor            # [F*T, H, D] bf16
    v: torch.Tensor
    head_k: Optional[torch.Tensor]   # [head_len, H, D] bf16 or None
    head_v: Optional[torch.Tensor]


@dataclass
class Inputs:
    cfg: Config
    q: torch.Tensor            # [Nq, H, D]
    k_cur: torch.Tensor
    v_cur: torch.Tensor
    k_txt: torch.Tensor        # [Lt, H, D]
    v_txt: torch.Tensor
    prior: List[SegmentKV] = field(default_factory=list)
    q_txt: Optional[torch.Tensor] = None   # [Lt, H, D]: text query rows (the text stream of the joint attention)


def make_inputs(cfg: Config, device="cpu", seed_offset: int = 0) -> Inputs:
    """Draw every tensor of a config.  `seed_offset` shifts all seeds (one independent problem per rank)."""
    H, D, T = cfg.heads, cfg.head_dim, cfg.tokens_per_frame
    off = seed_offset * 1000

    def s(tid):
        return cfg.seed(tid) + off

    nq = cfg.n_query
    lt = cfg.current.text_len
    q = _randn_bf16((nq, H, D), s(TID_Q))
    kc = _randn_bf16((nq, H, D), s(TID_KCUR))
    vc = _randn_bf16((nq, H, D), s(TID_VCUR))
    kt = _randn_bf16((lt, H, D), s(TID_KTXT))
    vt = _randn_bf16((lt, H, D), s(TID_VTXT))
    qt = _randn_bf16((lt, H, D), s(TID_QTXT))
    hist_tokens = sum(p.n_frames for p in cfg.prior) * T
    head_tokens = sum(p.head_len for p in cfg.prior)
    kh = _randn_bf16((hist_tokens, H, D), s(TID_KHIST))
    vh = _randn_bf16((hist_tokens, H, D), s(TID_VHIST))
    khd = _randn_bf16((head_tokens, H, D), s(TID_KHEAD))
    vhd = _randn_bf16((head_tokens, H, D), s(TID_VHEAD))
    if cfg.outliers:
        qch, kch = outlier_channels(cfg)
        q = _scale_outliers(q, qch)
        qt = _scale_outliers(qt, qch)
        kc = _scale_outliers(kc, kch)
        kt = _scale_outliers(kt, kch)
        kh = _scale_outliers(kh, kch)
        khd = _scale_outliers(khd, kch)
    prior = []
    t0 = h0 = 0
    for p in cfg.prior:
        n = p.n_frames * T
        prior.append(SegmentKV(kh[t0:t0 + n].to(device), vh[t0:t0 + n].to(device),
                               khd[h0:h0 + p.head_len].to(device) if p.head_len else None,
                               vhd[h0:h0 + p.head_len].to(device) if p.head_len else None))
        t0 += n
        h0 += p.head_len
    return Inputs(cfg, q.to(device), kc.to(device), vc.to(device), kt.to(device), vt.to(device), prior,
                  qt.to(device))


def attention_flops(cfg: Config, visible_keys_per_row_sum: int) -> float:
    """Algorithmic attention FLOPs: 4 * d * H * sum over rows of visible keys (QK^T and PV)."""
    return 4.0 * cfg.head_dim * cfg.heads * float(visible_keys_per_row_sum)


APPEND_BYTES_PER_TOKEN_HEAD = lambda d: 2 * (2 * d) + 2 * d + 2 * 4   # K,V bf16 read + int8 write + 2 fp32 scales


def n_blocks(n: int, b: int = 128) -> int:
    return (n + b - 1) // b


__all__ = ["Tail", "SegmentText", "Config", "CONFIGS", "small_config", "Inputs", "SegmentKV",
           "make_inputs", "outlier_channels", "attention_flops", "APPEND_BYTES_PER_TOKEN_HEAD", "n_blocks"]
