"""Full-dimensional routing policies of NanoKV-Fast (Table 7: "Full-dimensional
routing in the deployed NanoKV-Fast configurations"), as the token ranges and
head flags that nanokv_attend_routed takes.  Host-side helpers, no GPU work.

The pages describe the deployed policies in latent frames: a number of recent
frames, one periodic anchor per N older frames (or per fewer on listed
layers), sink frames at the start of the rollout, a per-layer fallback that
reads every history token full-dim, and sensitive head-layer pairs kept at
full dimension.  Readings taken where the table is silent:
  * a frame is `frame_tokens` consecutive history tokens, frame 0 the oldest;
    the last frame may be partial;
  * "recent" frames are the last `recent` frames of the history;
  * "sink" frames are the first `sinks` frames;
  * among the frames that are not recent, an anchor is every frame whose
    index is a multiple of `anchor_every` (the first frame of each group).
"""
from __future__ import annotations

import math


def frames_to_ranges(frames, T: int, frame_tokens: int) -> list[tuple[int, int]]:
    """Sorted, merged (start, count) token ranges covering the given frames,
    clipped to the T history tokens."""
    out: list[tuple[int, int]] = []
    for f in sorted(set(frames)):
        s = f * frame_tokens
        e = min(T, s + frame_tokens)
        if s >= e:
            continue
        if out and out[-1][0] + out[-1][1] == s:
            out[-1] = (out[-1][0], e - out[-1][0])
        else:
            out.append((s, e - s))
    return out


def frame_policy(T: int, frame_tokens: int, recent: int = 0, sinks: int = 0, anchor_every: int = 0,
                 full_layer: bool = False) -> list[tuple[int, int]]:
    """History token ranges read full-dim under a Table 7 policy: the `sinks`
    first frames, the `recent` last frames, one anchor per `anchor_every`
    older frames, or every token when the layer falls back to full dimension."""
    if T <= 0:
        return []
    if full_layer:
        return [(0, T)]
    n = math.ceil(T / frame_tokens)
    older = max(0, n - recent)
    frames = set(range(min(sinks, n))) | set(range(older, n))
    if anchor_every > 0:
        frames |= {f for f in range(older) if f % anchor_every == 0}
    return frames_to_ranges(frames, T, frame_tokens)


def full_mask(ranges, T: int):
    """Boolean mask [T] of the tokens the ranges route full-dim."""
    import numpy as np
    m = np.zeros(T, dtype=bool)
    for s, c in ranges:
        m[s:s + c] = True
    return m
