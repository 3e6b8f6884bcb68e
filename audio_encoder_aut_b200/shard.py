"""Window-aligned sharding of a batch across GPUs (host logic, no collectives).

The forward has no exchange across windows: a window is whole 100-frame chunks
of one request and attention never crosses a window (aut_encoder page, module
docstring; openarchlab "1A . AuT Audio Encoder", section 4, window isolation),
and every other step is per token.  So a batch splits exactly along window
boundaries: whole requests, or a long request cut at multiples of
n_window_infer frames.  Pieces are assigned to ranks longest-first onto the
least-loaded rank (LPT), by token count.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True, order=True)
class Piece:
    request: int   # index in the batch
    frame0: int    # first frame of the piece inside its request
    frames: int    # frames in the piece


def _tokens(frames: int) -> int:
    """Token count of a frame span that starts on a chunk boundary."""
    full, rem = divmod(frames, 100)
    t = rem
    for _ in range(3):
        t = (t + 1) // 2 if t > 0 else 0
    return 13 * full + t


def pieces(lens, n_window_infer: int, max_frames: int | None = None) -> list[Piece]:
    """Cut requests longer than `max_frames` (rounded down to whole windows)
    at window boundaries; shorter requests stay whole."""
    out = []
    step = None
    if max_frames is not None:
        step = max(n_window_infer, (max_frames // n_window_infer) * n_window_infer)
    for r, n in enumerate(lens):
        if n <= 0:
            continue
        if step is None or n <= step:
            out.append(Piece(r, 0, n))
        else:
            for f0 in range(0, n, step):
                out.append(Piece(r, f0, min(step, n - f0)))
    return out


def assign(ps: list[Piece], world: int) -> list[list[Piece]]:
    """Longest-processing-time-first assignment of pieces to `world` ranks."""
    loads = [0] * world
    shards = [[] for _ in range(world)]
    for p in sorted(ps, key=lambda p: (-_tokens(p.frames), p.request, p.frame0)):
        k = min(range(world), key=lambda i: (loads[i], i))
        shards[k].append(p)
        loads[k] += _tokens(p.frames)
    for s in shards:
        s.sort(key=lambda p: (p.request, p.frame0))
    return shards


def reassemble(lens, shards, outputs):
    """Concatenate per-rank outputs (rows of each rank's pieces, in its shard
    order) back into the unsharded packed order: requests in input order,
    pieces in frame order."""
    rows = {}
    for shard, out in zip(shards, outputs):
        at = 0
        for p in shard:
            n = _tokens(p.frames)
            rows[(p.request, p.frame0)] = out[at:at + n]
            at += n
    keys = sorted(rows)
    import numpy as np
    return np.concatenate([rows[k] for k in keys], axis=0) if keys else None
