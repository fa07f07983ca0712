"""Host-side helpers for a segment's text layout (description head + action tails).

The offline prompt format on papers.ananclaw.com ("离线 prompt JSON 格式") gives each segment and
each contained action a start and end time as MM:SS.mmm.  The same page's Diffusers example uses 30
latent frames for a 5-second segment (24 FPS, temporal compression 4), i.e. 6 latent frames per
second.  An action's window in segment-local latent frames is taken as
    f0 = floor((t_start - segment_start) * 6),  f1 = ceil((t_end - segment_start) * 6),
clipped to the segment; the window is half-open.  This conversion is this library's reading: the
pages state the time format and the frame rate, not the rounding.
"""
from __future__ import annotations

from fractions import Fraction
from typing import List, Tuple

LATENT_FPS = Fraction(24, 4)


def parse_time(s: str) -> Fraction:
    """'MM:SS.mmm' -> seconds (exact)."""
    mm, rest = s.split(":")
    sec, _, ms = rest.partition(".")
    ms = (ms + "000")[:3]
    return Fraction(int(mm) * 60 + int(sec)) + Fraction(int(ms), 1000)


def _floor(x: Fraction) -> int:
    return x.numerator // x.denominator


def _ceil(x: Fraction) -> int:
    return -((-x.numerator) // x.denominator)


def segment_frames(seg: dict) -> int:
    return _ceil((parse_time(seg["end_time"]) - parse_time(seg["start_time"])) * LATENT_FPS)


def action_windows(seg: dict) -> List[Tuple[int, int]]:
    """Latent-frame windows [f0, f1) of a segment's contained actions."""
    s0 = parse_time(seg["start_time"])
    n = segment_frames(seg)
    out = []
    for a in seg.get("contained_actions", []):
        f0 = _floor((parse_time(a["start_time"]) - s0) * LATENT_FPS)
        f1 = _ceil((parse_time(a["end_time"]) - s0) * LATENT_FPS)
        out.append((max(0, min(n, f0)), max(0, min(n, f1))))
    return out
